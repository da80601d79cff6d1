// k_attn_bucket_tc.cu -- bucket-major attention tiles on the 5th-generation
// tensor cores (tcgen05 MMA with TMEM accumulators; sm_100a).
//
// Same tiles and results as bucket_attn_kernel (k_attn_bucket.cu; method
// citations there): a tile is one bucket, or one run of consecutive queries'
// sinks and windows, with up to 16 queries and one KV head.  Here the tile's
// 16 queries x 8 query heads are the 128 rows of one MMA (a row per TMEM
// lane), and the tile's keys stream through in 64-key stages:
//
//   S  = Q K^T   M = 128, N = 64 keys, K = d      (TMEM, three buffers)
//   P  = exp2(S * scale * log2 e - m)            (softmax warps, bf16 into the
//                                                 first 32 columns of S's buffer)
//   O += P V     M = 128, N = d, K = 64 keys      (A = P read from TMEM; TMEM,
//                                                 two accumulators)
//
// Warp roles (16 warps):
//   warp 0     planner: claims work items (two ahead) and copies each tile's
//              description (bucket_tile_records_kernel) and member lists into
//              shared memory, prefetched to registers one item ahead;
//   warps 1-2, 13-14  loaders: gather every stage's K and V rows of the KV
//              head (16 keys per warp) with 16-byte cp.async into
//              128-byte-swizzled planes (the layout the MMA descriptors name);
//              completion lands on mbarriers;
//   warp 3     allocates TMEM; lane 0 issues the S MMAs and their commits;
//   warp 15    lane 0 issues the P V MMAs and their commits (its own thread,
//              so a P V is never queued behind the issue of later S MMAs);
//   warp 12    Q loader: the tile's Q rows, as soon as its Q buffer is free;
//   warps 4-7  softmax: thread = row = TMEM lane; reads its 64 scores of a
//              stage, masks keys outside its query's ranges, keeps the
//              running max (raised lazily: O and the sum are rescaled only
//              when the max grows by more than 2^8), writes its P row back to
//              TMEM over the scores, and at the end of the tile hands the
//              row's (max, sum) on;
//   warps 8-11 epilogue: write each row's partial (O row / sum as bf16, and
//              the fp32 max and sum) from one of two TMEM accumulators (tiles
//              alternate), overlapping the next tile's softmax; softmax and
//              epilogue keep what they need of a description in registers.
// Q and tile descriptions are double-buffered across work items and the K/V
// ring continues across them, so loads of the next tile overlap this one.  An
// S buffer (and the P in it) is released by the commit of its P V MMA, so the
// softmax never waits for the tensor cores except to rescale O.
// Every wait is bounded; on a timeout the CTA records DEV_TIMEOUT, all roles
// leave, outstanding copies and MMAs are waited for, and TMEM is freed.
#include <limits.h>
#include <math.h>

#include "attn_bucket.cuh"
#include "lsa_internal.cuh"
#include "ptx.cuh"

namespace lsa {

constexpr int TB_M = 128;            // MMA rows: BA_Q queries x 8 query heads
constexpr int TB_N = 64;             // keys per stage
constexpr int TB_OPEN_MAX = 2048;    // members of one bucket a tile can hold (block size bound)
#ifndef LSA_TB_SB
#define LSA_TB_SB 3
#endif
constexpr int TB_SB = LSA_TB_SB;     // S buffers in TMEM: S runs up to TB_SB - 1 stages ahead of P V
constexpr uint32_t TB_COL_O = TB_SB * 64;   // first TMEM column of the two O accumulators
static_assert(TB_COL_O + 256 <= 512, "TMEM: S buffers and two O accumulators in 512 columns");
#ifndef LSA_TB_LOADERS
#define LSA_TB_LOADERS 4     // K/V loader warps (2 or 4)
#endif
constexpr int TB_NL = LSA_TB_LOADERS;
static_assert(TB_NL == 2 || TB_NL == 4, "K/V loader warps");
constexpr int TB_KPW = 64 / TB_NL;                // keys of a stage per loader warp
constexpr int TB_PVW = 11 + TB_NL;                // the P V MMA issuer's warp
constexpr int TB_THREADS = 32 * (12 + TB_NL);     // 16 warps with four loaders
constexpr uint32_t TB_WAIT = 1u << 22;

// Polls each bounded wait of the tile kernel's roles makes before it gives up
// (and, times 8, the MMA issuer's polls without progress).  A test hook
// (lsa_set_wait_limit) lowers it to make the waits run out; the drain of the
// MMAs in flight on the way out always allows TB_WAIT.
__device__ uint32_t g_tb_wait = TB_WAIT;

#ifndef LSA_TB_QB
#define LSA_TB_QB 2          // Q buffers (2: the next tile's Q loads during this tile)
#endif
#ifndef LSA_TB_NS_MAX
#define LSA_TB_NS_MAX 4      // K/V stages when shared memory allows (else 3)
#endif

template <int D, int NS, int QB>
struct TbCfg {
    static constexpr int CH = D / 8;                    // 16-byte chunks per row
    static constexpr int Q_PLANE = TB_M * 128;          // 64 dims of 128 rows
    static constexpr int Q_BYTES = (D / 64) * Q_PLANE;
    static constexpr int KV_PLANE = TB_N * 128;         // 64 dims of 64 keys
    static constexpr int K_BYTES = (D / 64) * KV_PLANE;
    static constexpr int STAGE = 2 * K_BYTES;           // K then V
    static constexpr int OFF_Q = 0;                     // QB buffers
    static constexpr int OFF_KV = OFF_Q + QB * Q_BYTES; // NS stages
    static constexpr int OFF_BAR = OFF_KV + NS * STAGE;
    static constexpr int NBAR = 16 + 3 * TB_SB + 2 * NS;
    static constexpr int OFF_ML = OFF_BAR + NBAR * 8;      // [2][128] (max, sum) per row
    static constexpr int OFF_LISTS = OFF_ML + 2 * TB_M * 8;   // then 4 member lists of G ints
    // dynamic shared memory for a block of G pooled groups (+ alignment slack)
    static constexpr int bytes(int G) { return OFF_LISTS + 4 * ((G + 3) & ~3) * 4 + 1024; }
    static constexpr uint32_t KSTEPS = D / 16;
    // kind::f16, fp32 accumulate, bf16 A and B, M = 128
    static constexpr uint32_t IDESC_S =
        (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(TB_N >> 3) << 17) | ((uint32_t)(TB_M >> 4) << 24);
    static constexpr uint32_t IDESC_PV = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) /* B MN-major */ |
                                         ((uint32_t)(D >> 3) << 17) | ((uint32_t)(TB_M >> 4) << 24);
};

// ---- tcgen05 wrappers --------------------------------------------------------
__device__ __forceinline__ uint64_t tb_desc(uint32_t smem_addr, uint32_t lbo, uint32_t sbo)
{
    return (uint64_t)((smem_addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) /* tcgen05 descriptor */ |
           (2ull << 61) /* 128-byte swizzle */;
}

__device__ __forceinline__ void tb_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                       uint32_t idesc, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

// D (+)= A B with A (M x 16, bf16 pairs per 32-bit column, row m in lane m)
// read from TMEM at column a_tmem.
__device__ __forceinline__ void tb_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

__device__ __forceinline__ void tb_commit(uint64_t* bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     ptx::smem_addr(bar))
                 : "memory");
}

__device__ __forceinline__ void tb_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tb_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tb_ld32(uint32_t taddr, float* v)
{
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
        "%12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, "
        "%29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
          "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
          "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
}

// Two 32-column TMEM loads in flight, one wait.
__device__ __forceinline__ void tb_ld64(uint32_t taddr, float* v)
{
    uint32_t r[64];
#pragma unroll
    for (int h = 0; h < 2; ++h)
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
            "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
            "%28, %29, %30, %31}, [%32];"
            : "=r"(r[32 * h + 0]), "=r"(r[32 * h + 1]), "=r"(r[32 * h + 2]), "=r"(r[32 * h + 3]),
              "=r"(r[32 * h + 4]), "=r"(r[32 * h + 5]), "=r"(r[32 * h + 6]), "=r"(r[32 * h + 7]),
              "=r"(r[32 * h + 8]), "=r"(r[32 * h + 9]), "=r"(r[32 * h + 10]), "=r"(r[32 * h + 11]),
              "=r"(r[32 * h + 12]), "=r"(r[32 * h + 13]), "=r"(r[32 * h + 14]), "=r"(r[32 * h + 15]),
              "=r"(r[32 * h + 16]), "=r"(r[32 * h + 17]), "=r"(r[32 * h + 18]), "=r"(r[32 * h + 19]),
              "=r"(r[32 * h + 20]), "=r"(r[32 * h + 21]), "=r"(r[32 * h + 22]), "=r"(r[32 * h + 23]),
              "=r"(r[32 * h + 24]), "=r"(r[32 * h + 25]), "=r"(r[32 * h + 26]), "=r"(r[32 * h + 27]),
              "=r"(r[32 * h + 28]), "=r"(r[32 * h + 29]), "=r"(r[32 * h + 30]), "=r"(r[32 * h + 31])
            : "r"(taddr + 32u * h));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int j = 0; j < 64; ++j) v[j] = __uint_as_float(r[j]);
}

// 2^x by the hardware approximation (flush-to-zero; 2^-inf = +0).
__device__ __forceinline__ float ex2_approx(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ void tb_st32(uint32_t taddr, const float* v)
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
        "%28, %29, %30, %31, %32};" ::"r"(taddr),
        "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
        "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
        "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
        "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
        "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
        "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
        "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
        "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
        "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
        "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
        "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
        : "memory");
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tb_st32u(uint32_t taddr, const uint32_t* v)
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
        "%28, %29, %30, %31, %32};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
        "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
        "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]),
        "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]),
        "r"(v[29]), "r"(v[30]), "r"(v[31])
        : "memory");
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

template <int D, int NS, int QB>
__global__ void __launch_bounds__(TB_THREADS, 1) bucket_attn_tc_kernel(BaArgs a)
{
    using C = TbCfg<D, NS, QB>;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem = (unsigned char*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* info_full = bars;          // [2]
    uint64_t* info_empty = bars + 2;     // [2]
    uint64_t* q_full = bars + 4;         // [2]
    uint64_t* q_empty = bars + 6;        // [2]
    uint64_t* s_full = bars + 8;                    // [TB_SB]
    uint64_t* s_empty = s_full + TB_SB;             // [TB_SB] (committed after the buffer's P V)
    uint64_t* p_full = s_empty + TB_SB;             // [TB_SB]
    uint64_t* o_full = p_full + TB_SB;              // [2] (two O accumulators, by item parity)
    uint64_t* o_empty = o_full + 2;                 // [2]
    uint64_t* ml_full = o_empty + 2;                // [2]
    uint64_t* ml_empty = ml_full + 2;               // [2]
    uint64_t* kv_full = ml_empty + 2;               // [NS]
    float2* ml = reinterpret_cast<float2*>(smem + C::OFF_ML);   // [2][TB_M]
    uint64_t* kv_empty = kv_full + NS;
    const int lcap = (a.ix.G + 3) & ~3;  // ints per member list
    int32_t* lists = reinterpret_cast<int32_t*>(smem + C::OFF_LISTS);
    // [0, 2): open-member lists of the two item buffers; [2, 4): closed-member lists
    auto open_list = [&](int ib) { return lists + ib * lcap; };
    auto mem_list = [&](int ib) { return lists + (2 + ib) * lcap; };
    __shared__ TileInfo ti[2];
    __shared__ uint32_t tmem_slot;
    __shared__ volatile int abort_flag;
    __shared__ int cnt_s[1];
    __shared__ uint64_t fin_bar;
    __shared__ uint64_t fin_bar2;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const IndexView& ix = a.ix;
    const int p = ix.p;
    const int lp = ((p & (p - 1)) == 0) ? __ffs(p) - 1 : -1;
    const int64_t n_work = (a.n_wt + a.P.ctr[CTR_TILES]) * a.Hkv;

    if (tid == 0) {
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(&info_full[i], 1);
            ptx::mbar_init(&info_empty[i], 11 + TB_NL);   // 4 softmax, 4 epilogue, 2 MMA issuers, K/V loaders, Q loader
            ptx::mbar_init(&o_full[i], 1);
            ptx::mbar_init(&o_empty[i], 4);
            ptx::mbar_init(&ml_full[i], 4);
            ptx::mbar_init(&ml_empty[i], 4);
            ptx::mbar_init(&q_full[i], 32);        // every Q-loader lane's cp.async arrival
            ptx::mbar_init(&q_empty[i], 1);
        }
        for (int i = 0; i < TB_SB; ++i) {
            ptx::mbar_init(&s_full[i], 1);
            ptx::mbar_init(&s_empty[i], 1);
            ptx::mbar_init(&p_full[i], 4);
        }
        for (int s = 0; s < NS; ++s) {
            ptx::mbar_init(&kv_full[s], 32 * TB_NL);
            ptx::mbar_init(&kv_empty[s], 1);
        }
        ptx::mbar_init(&fin_bar, 1);
        ptx::mbar_init(&fin_bar2, 1);
        abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 3) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(
                         ptx::smem_addr(&tmem_slot))
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tb_fence_before();
    __syncthreads();
    tb_fence_after();
    const uint32_t tmem = tmem_slot;
    const uint32_t wl = g_tb_wait;

    // Bounded waits.  wait1: one thread.  waitw: every lane of a warp polls
    // (each gets the barrier's acquire) and the warp agrees on the outcome,
    // so that warp-collective instructions after it are never divergent.
    auto fail = [&](uint32_t where) {
        abort_flag = 1;
        dev_error(ix.status, DEV_TIMEOUT, where);
    };
    auto wait1 = [&](uint64_t* bar, uint32_t parity, uint32_t where) -> bool {
        if (abort_flag) return false;
        if (ptx::mbar_wait_bounded(bar, parity, wl)) return true;
        fail(where);
        return false;
    };
    auto waitw = [&](uint64_t* bar, uint32_t parity, uint32_t where) -> bool {
        bool ok = !abort_flag && ptx::mbar_wait_bounded(bar, parity, wl);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok && lane == 0) fail(where);
        return ok;
    };

    if (warp == 0) {
        // ============================ planner ============================
        // Claims work items and brings each tile's description and member
        // lists into shared memory.  Its global reads are software-pipelined
        // so that the wait for a free description buffer hides them: the
        // claim runs two items ahead; the description and the first
        // 32 x PF_MEM member ids of the next item are in registers before the
        // wait.
        constexpr int REC_V = TILE_REC_BYTES / 16;     // a record is 28 x 16 bytes, a lane each
        constexpr int PF_MEM = 4;
        const uint4* recs = reinterpret_cast<const uint4*>(a.P.recs);
        auto claim = [&]() -> int {
            int wv = 0;
            if (lane == 0) wv = atomicAdd(a.P.ctr + CTR_WORK, 1);
            return wv;   // meaningful in lane 0
        };
        auto load_rec = [&](int64_t w) -> uint4 {
            uint4 r = make_uint4(0u, 0u, 0u, 0u);
            if (w < n_work && lane < REC_V) r = recs[(w / a.Hkv) * REC_V + lane];
            return r;
        };
        // a 32-bit field of a record spread over the lanes (warp-uniform call)
        auto rec_u32 = [&](const uint4& r, int off) -> uint32_t {
            const int c = (off >> 2) & 3;
            const uint32_t v = c == 0 ? r.x : c == 1 ? r.y : c == 2 ? r.z : r.w;
            return __shfl_sync(0xffffffffu, v, off >> 4);
        };
        auto load_mem = [&](const uint4& r, int64_t w, int32_t* m) {
#pragma unroll
            for (int u = 0; u < PF_MEM; ++u) m[u] = 0;
            if (w >= n_work || (int)rec_u32(r, (int)offsetof(TileInfo, kind)) != 1) return;
            const int o0 = (int)rec_u32(r, (int)offsetof(TileInfo, o0));
            const int ng = (int)rec_u32(r, (int)offsetof(TileInfo, nclosed)) / p;
            const int64_t b = (int64_t)(((uint64_t)rec_u32(r, (int)offsetof(TileInfo, b) + 4) << 32) |
                                        rec_u32(r, (int)offsetof(TileInfo, b)));
            const int32_t* mem_g = ix.members + b * ix.NP + o0;
#pragma unroll
            for (int u = 0; u < PF_MEM; ++u)
                if (lane + 32 * u < ng) m[u] = mem_g[lane + 32 * u];
        };
        int64_t w_cur = __shfl_sync(0xffffffffu, claim(), 0);
        int c_next = claim();
        uint4 rec_cur = load_rec(w_cur);
        int32_t mem_cur[PF_MEM];
        load_mem(rec_cur, w_cur, mem_cur);
        for (int i = 0;; ++i) {
            const int ib = i & 1;
            const uint32_t iph = (uint32_t)((i >> 1) & 1);
            TileInfo& T = ti[ib];
            const int64_t w_nxt = __shfl_sync(0xffffffffu, c_next, 0);
            if (w_cur < n_work) c_next = claim();
            const uint4 rec_nxt = load_rec(w_nxt);
            if (!waitw(&info_empty[ib], iph ^ 1u, 100u)) break;
            if (w_cur >= n_work) {
                if (lane == 0) {
                    T.n_st = -1;
                    ptx::mbar_arrive(&info_full[ib]);
                }
                break;
            }
            if (lane < REC_V) reinterpret_cast<uint4*>(&T)[lane] = rec_cur;
            __syncwarp();
            if (lane == 0) T.h = (int)(w_cur % a.Hkv);
            if (T.kind == 1) {
                int32_t* mem_l = mem_list(ib);
                const int ng = T.nclosed / p;
#pragma unroll
                for (int u = 0; u < PF_MEM; ++u)
                    if (lane + 32 * u < ng) mem_l[lane + 32 * u] = mem_cur[u];
                const int32_t* mem_g = ix.members + T.b * ix.NP + T.o0;
                for (int x = 32 * PF_MEM + lane; x < ng; x += 32) mem_l[x] = mem_g[x];
                if (T.any_open) {
                    int32_t* open_l = open_list(ib);
                    ba_open_list(ix, a.n_blk, T.b, T.g, lane, 32, cnt_s, open_l, [] { __syncwarp(); });
                }
            }
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&info_full[ib]);
            w_cur = w_nxt;
            rec_cur = rec_nxt;
            load_mem(rec_cur, w_cur, mem_cur);
        }
    } else if (warp == 12) {
        // ============================ Q loader ============================
        // The tile's Q rows (row r = query r / hpg, head r % hpg; rows of empty
        // query positions are zero), as soon as the tile is described and its
        // Q buffer is free.
        for (int i = 0;; ++i) {
            const int ib = i & 1;
            const uint32_t iph = (uint32_t)((i >> 1) & 1);
            const TileInfo& T = ti[ib];
            if (!waitw(&info_full[ib], iph, 130u)) break;
            if (T.n_st < 0) break;
            const int qb = i % QB;
            if (!waitw(&q_empty[qb], (uint32_t)(((i / QB) & 1) ^ 1), 140u)) break;
            unsigned char* qs = smem + C::OFF_Q + qb * C::Q_BYTES;
            // Query q's hpg head rows are contiguous (hpg * D bf16) and fill MMA
            // rows q*hpg .. q*hpg+hpg-1.  Rows of empty query positions are
            // not loaded: every key of such a row is masked, so whatever the
            // buffer holds there never reaches a partial.
            const int per_q = a.hpg * C::CH;               // 16-byte chunks per query
            for (int q = 0; q < BA_Q; ++q) {
                if (T.slot[q] < 0) continue;
                const __nv_bfloat16* src_q = a.Q + ((size_t)T.row[q] * a.Hq + (size_t)T.h * a.hpg) * D;
                for (int x = lane; x < per_q; x += 32) {
                    const int hh = x / C::CH, c = x % C::CH;   // C::CH is a power of two
                    const int r = q * a.hpg + hh;
                    ptx::cp_async16(qs + (c >> 3) * C::Q_PLANE + r * 128 + (((c & 7) ^ (r & 7)) << 4),
                                    src_q + (size_t)hh * D + c * 8);
                }
            }
            ptx::cp_async_mbar_arrive(&q_full[qb]);
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&info_empty[ib]);   // done with ti[ib]
        }
        asm volatile("cp.async.wait_all;" ::: "memory");
    } else if (warp < 3 || (warp >= 13 && warp < TB_PVW)) {
        // ============================ loaders ============================
        // Gather every stage's K and V rows of the KV head (tokens from the
        // shared-memory member lists).
        const int lw = (warp < 3) ? warp - 1 : warp - 11;   // warps 1, 2, 13, 14
        int64_t gs = 0;
        for (int i = 0;; ++i) {
            const int ib = i & 1;
            const uint32_t iph = (uint32_t)((i >> 1) & 1);
            const TileInfo& T = ti[ib];
            if (!waitw(&info_full[ib], iph, 105u)) break;
            const int n_st = T.n_st;
            if (n_st < 0) break;
            const int32_t* mem_l = mem_list(ib);
            const int32_t* open_l = open_list(ib);

            // ---- K / V stages ----
            const size_t tstride = (size_t)a.Hkv * D;
            const __nv_bfloat16* Kb = a.K + ((size_t)T.b * ix.T_cap * a.Hkv + T.h) * D;
            const __nv_bfloat16* Vb = a.V + ((size_t)T.b * ix.T_cap * a.Hkv + T.h) * D;
            bool stop = false;
            for (int s = 0; s < n_st; ++s, ++gs) {
                const int slot = (int)(gs % NS);
                if (!waitw(&kv_empty[slot], (uint32_t)(((gs / NS) & 1) ^ 1), 120u)) {
                    stop = true;
                    break;
                }
                // this lane's key of the stage: one token per lane, shared by
                // shuffles; rows past the tile's last key are zero-filled without
                // a read (every query masks them, and 0 x 0 adds nothing to O)
                const int k = T.kbeg + s * TB_N + TB_KPW * lw + lane;
                int32_t tok = -1;
                if (lane < TB_KPW && k < T.kend) {
                    const int64_t t64 = ba_token(T, k, p, lp, mem_l, open_l);
                    tok = (int32_t)t64;
                    if (t64 < 0 || t64 >= ix.T_cap) {
                        dev_error(ix.status, DEV_BAD_INDEX, (uint32_t)t64);
                        tok = 0;
                    }
                }
                unsigned char* ks = smem + C::OFF_KV + slot * C::STAGE;
                constexpr int KPI = 32 / C::CH;       // keys per warp instruction
#pragma unroll 4
                for (int j = 0; j < TB_KPW / KPI; ++j) {
                    const int kl = KPI * j + lane / C::CH;        // key inside this warp's share
                    const int c = lane % C::CH;
                    const int32_t tk = __shfl_sync(0xffffffffu, tok, kl);
                    const int kr = TB_KPW * lw + kl;              // row inside the stage
                    const int soff = (c >> 3) * C::KV_PLANE + kr * 128 + (((c & 7) ^ (kr & 7)) << 4);
                    const bool real = tk >= 0;
                    const size_t goff = real ? (size_t)tk * tstride + c * 8 : 0;
                    ptx::cp_async16_zfill(ks + soff, Kb + goff, real ? 16u : 0u);
                    ptx::cp_async16_zfill(ks + C::K_BYTES + soff, Vb + goff, real ? 16u : 0u);
                }
                ptx::cp_async_mbar_arrive(&kv_full[slot]);
            }
            if (stop) break;
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&info_empty[ib]);   // done with ti[ib]
        }
        asm volatile("cp.async.wait_all;" ::: "memory");
    } else if (warp == 3) {
        // ========================= S MMA issuer ==========================
        // S = Q K^T of every stage in order, as soon as the stage's K/V rows
        // have landed, the item's Q is in and the S buffer's previous P V is
        // done (so S runs up to TB_SB - 1 stages ahead of P V).
        if (lane == 0) {
            int64_t gs = 0;
            const uint32_t q_base = ptx::smem_addr(smem + C::OFF_Q);
            const uint32_t kv_base = ptx::smem_addr(smem + C::OFF_KV);
            for (int i = 0;; ++i) {
                const int ib = i & 1;
                const uint32_t iph = (uint32_t)((i >> 1) & 1);
                if (!wait1(&info_full[ib], iph, 250u)) break;
                const int nS = ti[ib].n_st;
                ptx::mbar_arrive(&info_empty[ib]);
                if (nS < 0) break;
                const int qb = i % QB;
                if (!wait1(&q_full[qb], (uint32_t)((i / QB) & 1), 251u)) break;
                bool stop = false;
                for (int s = 0; s < nS; ++s, ++gs) {
                    const int slot = (int)(gs % NS);
                    const int sb = (int)(gs % TB_SB);
                    if (!wait1(&kv_full[slot], (uint32_t)((gs / NS) & 1), 252u) ||
                        !wait1(&s_empty[sb], (uint32_t)(((gs / TB_SB) & 1) ^ 1), 253u)) {
                        stop = true;
                        break;
                    }
                    tb_fence_after();
                    ptx::fence_proxy_async();   // the loaders' cp.async rows, to the async proxy
                    const uint64_t qd = tb_desc(q_base + qb * C::Q_BYTES, 16, 1024);
                    const uint64_t kd = tb_desc(kv_base + slot * C::STAGE, 16, 1024);
#pragma unroll
                    for (int kk = 0; kk < (int)C::KSTEPS; ++kk) {
                        // k-step kk: plane kk / 4, +32 bytes per step inside the row
                        const uint64_t qo = (uint64_t)(((kk >> 2) * C::Q_PLANE + (kk & 3) * 32) >> 4);
                        const uint64_t ko = (uint64_t)(((kk >> 2) * C::KV_PLANE + (kk & 3) * 32) >> 4);
                        tb_mma(tmem + sb * TB_N, qd + qo, kd + ko, C::IDESC_S, kk > 0 ? 1u : 0u);
                    }
                    tb_commit(&s_full[sb]);
                    if (s == nS - 1) tb_commit(&q_empty[qb]);
                }
                if (stop) break;
            }
            // nothing this thread issued may still run on the tensor cores at exit
            tb_commit(&fin_bar);
            ptx::mbar_wait_bounded(&fin_bar, 0, TB_WAIT);
        }
    } else if (warp == TB_PVW) {
        // ======================== P V MMA issuer =========================
        // O += P V of every stage in order, as soon as its P is in TMEM (and,
        // for an item's first stage, its O accumulator has been read out).
        // A thread of its own, so that a P V never waits behind the issue of
        // later stages' S MMAs.  Its commits release the stage's K/V slot and
        // S buffer, and after an item's last stage hand O to the epilogue.
        if (lane == 0) {
            int64_t gP = 0;
            const uint32_t kv_base = ptx::smem_addr(smem + C::OFF_KV);
            for (int i = 0;; ++i) {
                const int ib = i & 1;
                const uint32_t iph = (uint32_t)((i >> 1) & 1);
                if (!wait1(&info_full[ib], iph, 270u)) break;
                const int n = ti[ib].n_st;
                ptx::mbar_arrive(&info_empty[ib]);
                if (n < 0) break;
                if (!wait1(&o_empty[ib], iph ^ 1u, 271u)) break;
                bool stop = false;
                for (int s = 0; s < n; ++s, ++gP) {
                    const int sbP = (int)(gP % TB_SB);
                    const int slot = (int)(gP % NS);
                    if (!wait1(&p_full[sbP], (uint32_t)((gP / TB_SB) & 1), 272u)) {
                        stop = true;
                        break;
                    }
                    // the softmax threads' TMEM stores of P are ordered before
                    // their arrivals on p_full
                    tb_fence_after();
                    const uint32_t t_o = tmem + TB_COL_O + 128 * ib;
                    const uint64_t vd =
                        tb_desc(kv_base + slot * C::STAGE + C::K_BYTES, C::KV_PLANE, 1024);
#pragma unroll
                    for (int kk = 0; kk < TB_N / 16; ++kk)   // 16 keys = 8 TMEM columns of P
                        tb_mma_ts(t_o, tmem + sbP * TB_N + kk * 8, vd + (uint64_t)(kk * 128),
                                  C::IDESC_PV, (s > 0 || kk > 0) ? 1u : 0u);
                    tb_commit(&kv_empty[slot]);
                    tb_commit(&s_empty[sbP]);
                    if (s == n - 1) tb_commit(&o_full[ib]);
                }
                if (stop) break;
            }
            tb_commit(&fin_bar2);
            ptx::mbar_wait_bounded(&fin_bar2, 0, TB_WAIT);
        }
    } else if (warp < 8) {
        // ============================ softmax ============================
        const int r = 32 * (warp & 3) + lane;               // row = TMEM lane
        const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
        int64_t gs = 0;
        for (int i = 0;; ++i) {
            const int ib = i & 1;
            const uint32_t iph = (uint32_t)((i >> 1) & 1);
            if (!waitw(&info_full[ib], iph, 300u)) break;
            const TileInfo& T = ti[ib];
            const int n_st = T.n_st;
            if (n_st < 0) {
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&info_empty[ib]);
                break;
            }
            const int q = r / a.hpg;
            const bool live = q < BA_Q && T.slot[q] >= 0;
            const QRange rg = live ? T.rng[q] : QRange{0, 0, 0, 0};
            const int kbeg = T.kbeg;
            // what the row needs of the description is in registers: release it
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&info_empty[ib]);
            float m_run = -INFINITY, l = 0.f;
            bool stop = false;
            for (int s = 0; s < n_st; ++s, ++gs) {
                const int sb = (int)(gs % TB_SB);
                if (!waitw(&s_full[sb], (uint32_t)((gs / TB_SB) & 1), 310u)) {
                    stop = true;
                    break;
                }
                tb_fence_after();
                float v[TB_N];
                tb_ld64(tmem + lane_base + sb * TB_N, v);

                const int kb = kbeg + s * TB_N;
                // keys of this stage the row's query reads, as a 64-bit mask
                uint64_t keep = 0;
                if (live) {
                    auto bits = [&](int lo, int hi) -> uint64_t {
                        int x = lo - kb, y = hi - kb;
                        x = x < 0 ? 0 : (x > TB_N ? TB_N : x);
                        y = y < 0 ? 0 : (y > TB_N ? TB_N : y);
                        if (y <= x) return 0ull;
                        const uint64_t up = (y == TB_N) ? ~0ull : ((1ull << y) - 1ull);
                        return up & ~((1ull << x) - 1ull);
                    };
                    keep = bits(rg.lo0, rg.hi0) | bits(rg.lo1, rg.hi1);
                }
                // a row that reads none of the stage's keys takes P = 0 by an
                // infinite offset instead of masking every score
                const bool none = keep == 0ull;
                if (keep != ~0ull && !none) {
#pragma unroll
                    for (int j = 0; j < TB_N; ++j)
                        if (!((keep >> j) & 1ull)) v[j] = -INFINITY;
                }
                // row maximum of the raw scores (scale > 0), as a tree
                float t8[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    float m = v[u];
#pragma unroll
                    for (int j = u + 8; j < TB_N; j += 8) m = fmaxf(m, v[j]);
                    t8[u] = m;
                }
                const float mraw = fmaxf(fmaxf(fmaxf(t8[0], t8[1]), fmaxf(t8[2], t8[3])),
                                         fmaxf(fmaxf(t8[4], t8[5]), fmaxf(t8[6], t8[7])));
                const float mx = none ? -INFINITY : mraw * a.scale_log2;   // -inf stays -inf
                // Lazy running max: raised only on the item's first stage, from
                // nothing, or by more than 8 (a factor 2^8), so that O needs
                // rescaling rarely; P stays <= 2^8.
                bool resc = false;
                float alpha = 1.f;
                if (mx > m_run) {
                    if (s == 0 || m_run == -INFINITY) {
                        m_run = mx;
                    } else if (mx > m_run + 8.f) {
                        alpha = ex2_approx(m_run - mx);
                        m_run = mx;
                        resc = true;
                    }
                }
                const float mu = none ? INFINITY : ((m_run == -INFINITY) ? 0.f : m_run);
                uint32_t pk[TB_N / 2];
                float s4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int j = 0; j < TB_N / 2; ++j) {
                    // p = 2^(s * scale * log2(e) - m); a masked key gives 2^-inf = 0
                    const float p0 = ex2_approx(fmaf(v[2 * j], a.scale_log2, -mu));
                    const float p1 = ex2_approx(fmaf(v[2 * j + 1], a.scale_log2, -mu));
                    s4[j & 3] += p0 + p1;
                    pk[j] = ptx::pack_bf16(p0, p1);
                }
                const float sum = (s4[0] + s4[1]) + (s4[2] + s4[3]);
                l = l * alpha + sum;
                if (__any_sync(0xffffffffu, resc)) {
                    // O is quiet once the previous stage's P V MMA (the commit
                    // that released its S buffer) has completed
                    const int64_t gq = gs - 1;
                    if (!waitw(&s_empty[gq % TB_SB], (uint32_t)((gq / TB_SB) & 1), 320u)) {
                        stop = true;
                        break;
                    }
                    tb_fence_after();
#pragma unroll 1
                    for (int c = 0; c < D / 32; ++c) {
                        float o[32];
                        tb_ld32(tmem + lane_base + TB_COL_O + 128 * ib + c * 32, o);
#pragma unroll
                        for (int j = 0; j < 32; ++j) o[j] *= alpha;
                        tb_st32(tmem + lane_base + TB_COL_O + 128 * ib + c * 32, o);
                    }
                }
                // P over the first 32 columns of the scores' buffer
                tb_st32u(tmem + lane_base + sb * TB_N, pk);
                tb_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&p_full[sb]);
            }
            if (stop) break;
            // the row's (max, sum) for the epilogue warps, once they have read
            // the pair of two items ago
            if (!waitw(&ml_empty[ib], iph ^ 1u, 330u)) break;
            ml[ib * TB_M + r] = make_float2(m_run, l);
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&ml_full[ib]);
        }
    } else {
        // ============================ epilogue ============================
        // Warps 8-11 (TMEM lanes by warp % 4): each row's partial -- the
        // unnormalised O row, max and sum -- once the tile's last P V MMA is
        // done, while the softmax warps already work on the next tile.
        const int r = 32 * (warp & 3) + lane;
        const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
        for (int i = 0;; ++i) {
            const int ib = i & 1;
            const uint32_t iph = (uint32_t)((i >> 1) & 1);
            if (!waitw(&info_full[ib], iph, 400u)) break;
            const TileInfo& T = ti[ib];
            if (T.n_st < 0) break;
            const int q = r / a.hpg, hh = r % a.hpg;
            const int slot = (q < BA_Q) ? T.slot[q] : -1;
            const bool live = slot >= 0;
            const size_t ph = ((size_t)(live ? slot : 0) * a.Hq) + (size_t)T.h * a.hpg + hh;
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&info_empty[ib]);   // the rest is in registers
            if (!waitw(&ml_full[ib], iph, 410u) || !waitw(&o_full[ib], iph, 420u)) break;
            tb_fence_after();
            const float2 mlr = ml[ib * TB_M + r];
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&ml_empty[ib]);
            __nv_bfloat16* po = a.P.part_o + ph * D;
            // the row normalised by its own sum (a convex combination of V rows)
            const float inv = (mlr.y > 0.f) ? 1.f / mlr.y : 0.f;
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
                float o[32];
                tb_ld32(tmem + lane_base + TB_COL_O + 128 * ib + c * 32, o);
                if (live) {
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        reinterpret_cast<uint4*>(po + c * 32)[j] = make_uint4(
                            ptx::pack_bf16(o[8 * j] * inv, o[8 * j + 1] * inv),
                            ptx::pack_bf16(o[8 * j + 2] * inv, o[8 * j + 3] * inv),
                            ptx::pack_bf16(o[8 * j + 4] * inv, o[8 * j + 5] * inv),
                            ptx::pack_bf16(o[8 * j + 6] * inv, o[8 * j + 7] * inv));
                }
            }
            if (live) a.P.part_ml[ph] = mlr;
            tb_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&o_empty[ib]);
        }
    }
    tb_fence_before();
    __syncthreads();
    if (warp == 3) {
        tb_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem)
                     : "memory");
    }
}

cudaError_t set_tile_wait_polls(int64_t polls)
{
    const uint32_t v = (polls < 0 || polls > (int64_t)TB_WAIT) ? TB_WAIT : (uint32_t)polls;
    return cudaMemcpyToSymbol(g_tb_wait, &v, sizeof(v));
}

bool bucket_attn_tc_supported(int Hq, int Hkv, int d, int G)
{
    return (d == 64 || d == 128) && Hq % Hkv == 0 && Hq / Hkv <= 8 && G <= TB_OPEN_MAX;
}

// Shared memory the device grants one block (opt-in maximum).
static int smem_optin()
{
    int dev = 0, v = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
        return 0;
    return v;
}

template <int D, int NS, int QB>
static cudaError_t launch_tc_t(const BaArgs& a, int cap, cudaStream_t st)
{
    using C = TbCfg<D, NS, QB>;
    auto kern = bucket_attn_tc_kernel<D, NS, QB>;
    const int bytes = C::bytes(a.ix.G);
    // the limit is raised once per device, for the largest block served
    const int lim = C::bytes(TB_OPEN_MAX) < cap ? C::bytes(TB_OPEN_MAX) : cap;
    if (bytes > lim) return cudaErrorInvalidConfiguration;
    cudaError_t e = ensure_smem_attr((const void*)kern, lim);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, TB_THREADS, bytes);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    kern<<<(unsigned)(sm_count() * per_sm), TB_THREADS, bytes, st>>>(a);
    note_launch();
    return cudaGetLastError();
}

cudaError_t launch_bucket_attn_tc(const BaArgs& a, int d, cudaStream_t st)
{
    // the deeper K/V ring where the block's member lists leave room for it
    constexpr int STATIC_SMEM = 1024;   // tile descriptions, flags (928 bytes; upper bound)
    constexpr int NSX = LSA_TB_NS_MAX, QB = LSA_TB_QB;
    const int cap = smem_optin() - STATIC_SMEM;
    if (d == 128)
        return (TbCfg<128, NSX, QB>::bytes(a.ix.G) <= cap) ? launch_tc_t<128, NSX, QB>(a, cap, st)
                                                            : launch_tc_t<128, 3, QB>(a, cap, st);
    return (TbCfg<64, NSX, QB>::bytes(a.ix.G) <= cap) ? launch_tc_t<64, NSX, QB>(a, cap, st)
                                                       : launch_tc_t<64, 3, QB>(a, cap, st);
}

}  // namespace lsa
