// k_score_tc.cu -- tensor-core candidate nomination for bf16 indices
// (tcgen05 MMA, TMEM accumulators, TMA tile loads; sm_100a).
//
// Method: "Latent Sparse Attention: un indice gerarchico per contesti
// lunghi", paragraph on retrieval: each query is compared with the centroids
// to choose the buckets it reads.  This is the one dense contraction of the
// path: scores S = Q C^T with Q [queries][64] and C [buckets][64], both bf16,
// accumulated in fp32.
//
// These approximate scores are written as fp16 to a [queries][buckets] matrix
// in the selection workspace; select_fill_kernel (k_select.cu) nominates each
// query's candidates from its row and then ranks them with exact binary64
// scores.  At 10M context the matrix is 32768 x 40960 fp16 (2.7 GB), written
// once and read once.
//
// CTA = 128 queries of one sequence (one TMEM lane each), 6 warps:
//   warp 0     TMA producer: the query tile once, then TC_N-centroid tiles into
//              a TC_STAGES-deep shared-memory ring (128-byte swizzle);
//   warp 1     owns 2 x TC_N TMEM columns (two fp32 accumulators) and
//              issues tcgen05.mma (M=128, N=TC_N, K=16, four per tile);
//   warps 2-5  epilogue: tcgen05.ld 32 columns at a time, fp32 -> fp16, and
//              64-byte row segments straight to the score matrix.
// Every mbarrier wait is bounded; on a timeout the CTA records DEV_TIMEOUT in
// the index status word, stops waiting, and still frees its TMEM.
#include <cuda.h>

#include <cuda_fp16.h>

#include "lsa_internal.cuh"
#include "ptx.cuh"
#include "hooks.cuh"
#include "tmap.cuh"

namespace lsa {

constexpr int TC_M = 128;
#ifndef LSA_TC_N
#define LSA_TC_N 256         // centroids per tile (128 gives two CTAs per SM; measured slower)
#endif
constexpr int TC_N = LSA_TC_N;
constexpr int TC_TMEM_COLS = 2 * TC_N;                    // two fp32 accumulators
constexpr int TC_MIN_BLOCKS = (TC_N <= 128) ? 2 : 1;
constexpr int TC_STAGES = 4;
constexpr int TC_THREADS = 192;
constexpr uint32_t TC_WAIT = 1u << 22;

// Polls each bounded wait of the scorer's roles makes before it gives up.  A
// test hook (lsa_set_wait_limit) lowers it to make the waits run out; the
// drains on the way out always allow TC_WAIT.
__device__ uint32_t g_tc_wait = TC_WAIT;

constexpr int TC_Q_BYTES = TC_M * DL * 2;                 // 16 KB
constexpr int TC_C_BYTES = TC_N * DL * 2;                 // 32 KB per stage at N = 256
constexpr int TC_OFF_C = TC_Q_BYTES;
constexpr int TC_OFF_BAR = TC_OFF_C + TC_STAGES * TC_C_BYTES;
constexpr int TC_NBAR = 1 + 2 * TC_STAGES + 4 + 1;
constexpr int TC_OFF_MISC = TC_OFF_BAR + TC_NBAR * 8;
constexpr int TC_SMEM = TC_OFF_MISC + 64 + 1024;          // + alignment slack


// ---- tcgen05 / TMA wrappers -------------------------------------------------
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y,
                                            uint64_t* bar)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(ptx::smem_addr(dst)),
        "l"((uint64_t)map), "r"(ptx::smem_addr(bar)), "r"(x), "r"(y)
        : "memory");
}

__device__ __forceinline__ uint64_t sw128_desc(const void* smem_tile)
{
    const uint64_t a = ptx::smem_addr(smem_tile);
    return ((a >> 4) & 0x3FFFull)   // start address
           | (1ull << 16)           // leading byte offset (unused for 128B-swizzled K-major)
           | (64ull << 32)          // stride byte offset: 8 rows x 128 B = 1024 B
           | (1ull << 46)           // descriptor version (tcgen05)
           | (2ull << 61);          // 128-byte swizzle
}

// kind::f16 instruction descriptor: fp32 accumulate, bf16 A and B, both
// K-major, N = TC_N, M = 128.
constexpr uint32_t TC_IDESC = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(TC_N >> 3) << 17) |
                              ((uint32_t)(TC_M >> 4) << 24);

__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                         uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(TC_IDESC), "r"(accumulate));
}

__device__ __forceinline__ void mma_commit(uint64_t* bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     ptx::smem_addr(bar))
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v)
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

__device__ __forceinline__ int64_t tc_eligible(const IndexView& ix, int64_t n_blk, int64_t pos,
                                               int W)
{
    const int64_t hi = pos - W;
    if (hi < 0) return 0;
    const int64_t span = (int64_t)ix.p * ix.G;
    int64_t nb = hi / span + 1;
    if (nb > n_blk) nb = n_blk;
    return nb * ix.k;
}

__global__ void __launch_bounds__(TC_THREADS, TC_MIN_BLOCKS) score_topk_tc_kernel(
    const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmC, IndexView ix,
    int64_t n_blk, PosSrc pos, int64_t Nq, int W, SelectWs ws)
{
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem =
        (unsigned char*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);  // 1 KB aligned
    unsigned char* q_s = smem;
    unsigned char* c_s = smem + TC_OFF_C;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + TC_OFF_BAR);
    uint64_t* q_full = bars;
    uint64_t* full = bars + 1;
    uint64_t* empty = full + TC_STAGES;
    uint64_t* acc_full = empty + TC_STAGES;
    uint64_t* acc_empty = acc_full + 2;
    uint64_t* fin = acc_empty + 2;        // the MMA thread's last MMAs are done
    uint32_t* misc = reinterpret_cast<uint32_t*>(smem + TC_OFF_MISC);
    volatile uint32_t* tmem_slot = misc;        // [0]
    volatile uint32_t* abort_flag = misc + 1;   // [1]
    uint32_t* nb_max = misc + 2;                // [2]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t b = blockIdx.y;
    const int64_t q0 = (int64_t)blockIdx.x * TC_M;
    if (blockIdx.x == 0 && b == 0 && threadIdx.x == 0) *ws.fb_count = 0;
    {
        const int64_t cta = b * gridDim.x + blockIdx.x;
        for (int64_t x = cta * blockDim.x + threadIdx.x; x < ws.plan.n_zero;
             x += (int64_t)gridDim.x * gridDim.y * blockDim.x)
            ws.plan.zero[x] = 0;
    }

    if (threadIdx.x == 0) {
        ptx::mbar_init(q_full, 1);
        for (int s = 0; s < TC_STAGES; ++s) {
            ptx::mbar_init(&full[s], 1);
            ptx::mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            ptx::mbar_init(&acc_full[a], 1);
            ptx::mbar_init(&acc_empty[a], 4);
        }
        ptx::mbar_init(fin, 1);
        *abort_flag = 0;
        *nb_max = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         ptx::smem_addr((const void*)tmem_slot)), "n"(TC_TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    // per-row eligibility (epilogue threads own rows)
    int64_t nb_row = 0;
    int r = 0;
    bool row_valid = false;
    if (warp >= 2) {
        r = 32 * (warp & 3) + lane;
        row_valid = (q0 + r) < Nq;
        if (row_valid) nb_row = tc_eligible(ix, n_blk, pos.at(b, Nq, q0 + r), W);
    }
    __syncthreads();
    if (warp >= 2) atomicMax(nb_max, (uint32_t)nb_row);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int n_tiles = (int)((*nb_max + TC_N - 1) / TC_N);
    const uint32_t wl = g_tc_wait;

    if (warp == 0 && lane == 0 && n_tiles > 0) {
        // ---------------- TMA producer ----------------
        ptx::mbar_arrive_expect_tx(q_full, TC_Q_BYTES);
        tma_load_2d(q_s, &tmQ, 0, (int)(b * Nq + q0), q_full);
        int issued = 0;
        for (int t = 0; t < n_tiles; ++t) {
            const int s = t % TC_STAGES;
            const uint32_t ph = (uint32_t)((t / TC_STAGES) & 1);
            if (*abort_flag) break;
            if (!ptx::mbar_wait_bounded(&empty[s], ph ^ 1u, wl)) {
                *abort_flag = 1;
                dev_error(ix.status, DEV_TIMEOUT, 1000u + (uint32_t)t);
                break;
            }
            ptx::mbar_arrive_expect_tx(&full[s], TC_C_BYTES);
            tma_load_2d(c_s + s * TC_C_BYTES, &tmC, 0, (int)(b * ix.NBK + (int64_t)t * TC_N),
                        &full[s]);
            issued = t + 1;
        }
        if (*abort_flag) {
            // no copy may still be writing shared memory when the CTA exits:
            // the latest load of every stage (and the query tile) has landed,
            // or a bounded wait gives up on it
            ptx::mbar_wait_bounded(q_full, 0, TC_WAIT);
            for (int t = (issued > TC_STAGES ? issued - TC_STAGES : 0); t < issued; ++t)
                ptx::mbar_wait_bounded(&full[t % TC_STAGES], (uint32_t)((t / TC_STAGES) & 1),
                                       TC_WAIT);
        }
    } else if (warp == 1 && lane == 0 && n_tiles > 0) {
        // ---------------- MMA issuer ----------------
        bool ok = ptx::mbar_wait_bounded(q_full, 0, wl);
        if (!ok) {
            *abort_flag = 1;
            dev_error(ix.status, DEV_TIMEOUT, 2000u);
        }
        const uint64_t adesc = sw128_desc(q_s);
        for (int t = 0; ok && t < n_tiles; ++t) {
            const int s = t % TC_STAGES;
            const uint32_t ph = (uint32_t)((t / TC_STAGES) & 1);
            const int buf = t & 1;
            const uint32_t aph = (uint32_t)((t >> 1) & 1);
            if (*abort_flag) break;
            if (!ptx::mbar_wait_bounded(&full[s], ph, wl) ||
                !ptx::mbar_wait_bounded(&acc_empty[buf], aph ^ 1u, wl)) {
                *abort_flag = 1;
                dev_error(ix.status, DEV_TIMEOUT, 3000u + (uint32_t)t);
                break;
            }
            tc_fence_after();
            const uint64_t bdesc = sw128_desc(c_s + s * TC_C_BYTES);
            const uint32_t d = tmem + (uint32_t)(buf * TC_N);
#pragma unroll
            for (int kk = 0; kk < DL / 16; ++kk)
                mma_bf16(d, adesc + 2ull * kk, bdesc + 2ull * kk, kk > 0 ? 1u : 0u);
            mma_commit(&empty[s]);
            mma_commit(&acc_full[buf]);
        }
        // nothing of this CTA may still run on the tensor cores when TMEM is freed
        mma_commit(fin);
        ptx::mbar_wait_bounded(fin, 0, TC_WAIT);
    } else if (warp >= 2) {
        // ---------------- epilogue ----------------
        const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
        __half* srow = ws.scores + (b * Nq + q0 + r) * ws.score_ld;
        __half* crow = ws.cmax + (b * Nq + q0 + r) * (ws.score_ld / 32);
        for (int t = 0; t < n_tiles; ++t) {
            const int buf = t & 1;
            const uint32_t ph = (uint32_t)((t >> 1) & 1);
            if (*abort_flag) break;
            if (!ptx::mbar_wait_bounded(&acc_full[buf], ph, wl)) {
                *abort_flag = 1;
                dev_error(ix.status, DEV_TIMEOUT, 4000u + (uint32_t)t);
                break;
            }
            tc_fence_after();
            for (int c = 0; c < TC_N / 32; ++c) {
                float v[32];
                __syncwarp();
                tmem_ld32(tmem + lane_base + (uint32_t)(buf * TC_N + c * 32), v);
                const int64_t g0 = (int64_t)t * TC_N + c * 32;
                if (row_valid && g0 < nb_row) {
                    uint4 pk[4];
                    __half2* h = reinterpret_cast<__half2*>(pk);
                    float mx = -INFINITY;
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        if (g0 + j < nb_row) mx = fmaxf(mx, v[j]);
#pragma unroll
                    for (int j = 0; j < 16; ++j) h[j] = __floats2half2_rn(v[2 * j], v[2 * j + 1]);
                    uint4* dst = reinterpret_cast<uint4*>(srow + g0);
#pragma unroll
                    for (int j = 0; j < 4; ++j) dst[j] = pk[j];
                    // fp16 rounding is monotone: the rounded maximum is the
                    // maximum of the rounded scores of the chunk
                    crow[g0 / 32] = __float2half_rn(mx);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&acc_empty[buf]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "n"(TC_TMEM_COLS)
                     : "memory");
    }
}

// ---- host side ---------------------------------------------------------------
static bool make_rows64_bf16(CUtensorMap* m, const void* base, uint64_t rows, uint32_t box_rows)
{
    TmapEncodeFn enc = tmap_encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)DL, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)DL * 2};
    const cuuint32_t box[2] = {(cuuint32_t)DL, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool tc_scoring_available() { return true; }

cudaError_t set_score_wait_polls(int64_t polls)
{
    const uint32_t v = (polls < 0 || polls > (int64_t)TC_WAIT) ? TC_WAIT : (uint32_t)polls;
    return cudaMemcpyToSymbol(g_tc_wait, &v, sizeof(v));
}

cudaError_t launch_score_topk_tc(const IndexView& ix, int64_t n_blk, const void* latent_Q,
                                 PosSrc pos, int64_t Nq, int W, const SelectWs& ws,
                                 cudaStream_t st)
{
    if (ix.dtype != LSA_BF16) return cudaErrorInvalidValue;
    CUtensorMap tmQ, tmC;
    if (!make_rows64_bf16(&tmQ, latent_Q, (uint64_t)ix.B * Nq, TC_M) ||
        !make_rows64_bf16(&tmC, ix.cent_rt, (uint64_t)ix.B * ix.NBK, TC_N))
        return cudaErrorInvalidValue;
    cudaError_t e = ensure_smem_attr((const void*)score_topk_tc_kernel, TC_SMEM);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)((Nq + TC_M - 1) / TC_M), (unsigned)ix.B);
    score_topk_tc_kernel<<<grid, TC_THREADS, TC_SMEM, st>>>(tmQ, tmC, ix, n_blk, pos, Nq, W, ws);
    note_launch();
    return cudaGetLastError();
}

}  // namespace lsa
