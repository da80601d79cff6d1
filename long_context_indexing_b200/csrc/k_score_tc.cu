// k_score_tc.cu -- tensor-core candidate lists for bf16 indices (tcgen05 MMA,
// TMEM accumulators, TMA tile loads; sm_100a).
//
// Method: "Latent Sparse Attention: un indice gerarchico per contesti
// lunghi", paragraph on retrieval: each query is compared with the centroids
// to choose the buckets it reads.  This is the one dense contraction of the
// path: scores S = Q C^T with Q [queries][64] and C [buckets][64], both bf16,
// accumulated in fp32.
//
// No score matrix is written.  A work item is (sequence, 128-query tile,
// split), where a split is a contiguous range of centroid tiles; persistent
// CTAs (one per SM) take the items in a fixed round-robin order.  Three
// launches:
//   pass 1   (score_tc_kernel<1>) the epilogue writes, per query row, the
//            maximum of every group of gw consecutive eligible scores, rounded
//            down to fp16, as ordered 16-bit keys;
//   theta    (score_theta_kernel, a warp per row) picks theta, the m-th largest
//            of the row's group maxima over all splits: at least m scores of
//            the row are >= theta (each of the m groups holds one);
//   pass 2   (score_tc_kernel<2>) recomputes the scores and appends every
//            eligible score >= theta to the row's list for the split (bucket
//            id), up to the list's capacity.
// Every eligible bucket left out of a list scored below theta, or was an
// appended score that found the list full (the largest of those is kept), so
// tau = max(theta, largest lost score) bounds the approximate score of every
// bucket of the split that is not in the list.  A row with at most KCF
// eligible buckets lists them all (theta = -inf: the lists are complete).
// select_fill_kernel (k_select.cu) merges a row's lists, ranks the candidates
// with exact binary64 scores and proves the exact ranking against the largest
// tau, or sends the row to the exact fallback.
//
// CTA = 18 warps:
//   warp 0     TMA producer: each item's query tile (two buffers), then its
//              centroid tiles into a TC_STAGES-deep ring (128-byte swizzle);
//   warp 1     owns 2 x TC_N TMEM columns (two fp32 accumulators) and issues
//              tcgen05.mma (M = 128, N = TC_N, K = 16, four per tile);
//   warps 2-17 epilogue, four warps per TMEM lane quarter: thread = (query
//              row, a quarter of every tile's columns, 64 scores); tcgen05.ld
//              of 32-column pieces, several in flight before one wait.
// Every mbarrier wait is bounded; after a timeout the CTA records DEV_TIMEOUT
// in the index status word, the producer and the MMA thread stop, the
// epilogue runs through its remaining items without waiting (so its named
// barriers stay matched), copies and MMAs in flight are waited for, and TMEM
// is freed.
#include <cuda.h>

#include <cuda_fp16.h>

#include "lsa_internal.cuh"
#include "ptx.cuh"
#include "hooks.cuh"
#include "tmap.cuh"
#include "tc_common.cuh"

namespace lsa {

constexpr int TC_M = 128;
constexpr int TC_N = 256;                                 // centroids per tile
constexpr int TC_TMEM_COLS = 2 * TC_N;                    // two fp32 accumulators
constexpr int TC_STAGES = 4;
constexpr int TC_EPI_WARPS = 16;                          // 4 per TMEM lane quarter
constexpr int TC_COLS = TC_N / 4;                         // columns of a tile per epilogue thread
constexpr int TC_EPI_THREADS = 32 * TC_EPI_WARPS;
constexpr int TC_THREADS = 64 + TC_EPI_THREADS;           // producer, MMA, epilogue
constexpr uint32_t TC_WAIT = 1u << 22;

// Polls each bounded wait of the scorer's roles makes before it gives up.  A
// test hook (lsa_set_wait_limit) lowers it to make the waits run out; the
// drains on the way out always allow TC_WAIT.
__device__ uint32_t g_tc_wait = TC_WAIT;

constexpr int TC_Q_BYTES = TC_M * DL * 2;                 // 16 KB per query buffer
constexpr int TC_C_BYTES = TC_N * DL * 2;                 // 32 KB per ring stage
constexpr int TC_OFF_C = 2 * TC_Q_BYTES;
constexpr int TC_OFF_BAR = TC_OFF_C + TC_STAGES * TC_C_BYTES;
constexpr int TC_NBAR = 2 + 2 + 2 * TC_STAGES + 2 + 2 + 1;
constexpr int TC_OFF_MISC = TC_OFF_BAR + TC_NBAR * 8;
constexpr int TC_MISC_BYTES = TC_M * 4 + TC_EPI_THREADS * 4 + 64;
constexpr int TC_SMEM = TC_OFF_MISC + TC_MISC_BYTES + 1024;   // + alignment slack

// kind::f16 instruction descriptor: fp32 accumulate, bf16 A and B, both
// K-major, N = TC_N, M = 128.
constexpr uint32_t TC_IDESC = tc_idesc_bf16(TC_M, TC_N);

// One of 8 values by a 3-bit index (selects, no indexed registers).
__device__ __forceinline__ float pick8(const float* v, int e)
{
    const float a = (e & 1) ? v[1] : v[0], b = (e & 1) ? v[3] : v[2];
    const float c = (e & 1) ? v[5] : v[4], d = (e & 1) ? v[7] : v[6];
    const float ab = (e & 2) ? b : a, cd = (e & 2) ? d : c;
    return (e & 4) ? cd : ab;
}

// Named barrier of the epilogue warps only.
__device__ __forceinline__ void epi_sync()
{
    asm volatile("bar.sync 1, %0;" ::"n"(TC_EPI_THREADS) : "memory");
}

// Ordered 16-bit key of an fp16 value (larger value, larger key; never 0).
__device__ __forceinline__ uint32_t tc_half_key(__half h)
{
    const uint32_t u = __half_as_ushort(h);
    return (u & 0x8000u) ? (~u & 0xFFFFu) : (u | 0x8000u);
}

__device__ __forceinline__ float tc_key_value(uint32_t k)
{
    const uint16_t u = (k & 0x8000u) ? (uint16_t)(k & 0x7FFFu) : (uint16_t)(~k & 0xFFFFu);
    return __half2float(__ushort_as_half(u));
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

// Geometry of one work item, computed identically by every role.
struct TcItem {
    int64_t b, q0;      // sequence, first query of the tile
    int s;              // split
    int t0, t1;         // centroid tiles [t0, t1) of this item (t1 <= t0: nothing eligible)
};

// Every lane of the calling warp takes part (warp-collective).
__device__ __forceinline__ TcItem tc_item(int64_t it, const IndexView& ix, int64_t n_blk,
                                          const PosSrc& pos, int64_t Nq, int W, const TcSplit& sp)
{
    TcItem r;
    r.s = (int)(it % sp.n_split);
    const int64_t qt = it / sp.n_split;
    r.b = qt / sp.n_qt;
    r.q0 = (qt % sp.n_qt) * TC_M;
    const int lane = threadIdx.x & 31;
    unsigned nb = 0;
#pragma unroll
    for (int u = 0; u < TC_M / 32; ++u) {
        const int64_t q = r.q0 + lane + 32 * u;
        if (q < Nq) {
            const int64_t e = tc_eligible(ix, n_blk, pos.at(r.b, Nq, q), W);
            if ((unsigned)e > nb) nb = (unsigned)e;
        }
    }
    nb = __reduce_max_sync(0xffffffffu, nb);
    const int n_ct = (int)((nb + TC_N - 1) / TC_N);
    r.t0 = r.s * sp.tps;
    r.t1 = min(r.t0 + sp.tps, n_ct);
    return r;
}

template <int PASS>
__global__ void __launch_bounds__(TC_THREADS, 1) score_tc_kernel(
    const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmC, IndexView ix,
    int64_t n_blk, PosSrc pos, int64_t Nq, int W, SelectWs ws, TcSplit sp)
{
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem =
        (unsigned char*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);  // 1 KB aligned
    unsigned char* q_s = smem;                        // [2][TC_Q_BYTES]
    unsigned char* c_s = smem + TC_OFF_C;             // [TC_STAGES][TC_C_BYTES]
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + TC_OFF_BAR);
    uint64_t* q_full = bars;                  // [2]
    uint64_t* q_empty = bars + 2;             // [2]
    uint64_t* full = bars + 4;                // [TC_STAGES]
    uint64_t* empty = full + TC_STAGES;       // [TC_STAGES]
    uint64_t* acc_full = empty + TC_STAGES;   // [2]
    uint64_t* acc_empty = acc_full + 2;       // [2]
    uint64_t* fin = acc_empty + 2;            // the MMA thread's last MMAs are done
    int* rcnt = reinterpret_cast<int*>(smem + TC_OFF_MISC);                 // [TC_M]
    float* lostv = reinterpret_cast<float*>(smem + TC_OFF_MISC + TC_M * 4); // [TC_EPI_THREADS]
    uint32_t* misc = reinterpret_cast<uint32_t*>(smem + TC_OFF_MISC + TC_M * 4 + TC_EPI_THREADS * 4);
    volatile uint32_t* tmem_slot = misc;        // [0]
    volatile uint32_t* abort_flag = misc + 1;   // [1]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (PASS == 1) {
        if (blockIdx.x == 0 && threadIdx.x == 0) *ws.fb_count = 0;
        for (int64_t x = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; x < ws.plan.n_zero;
             x += (int64_t)gridDim.x * blockDim.x)
            ws.plan.zero[x] = 0;
    }

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(&q_full[i], 1);
            ptx::mbar_init(&q_empty[i], 1);
            ptx::mbar_init(&acc_full[i], 1);
            ptx::mbar_init(&acc_empty[i], TC_EPI_WARPS);
        }
        for (int s = 0; s < TC_STAGES; ++s) {
            ptx::mbar_init(&full[s], 1);
            ptx::mbar_init(&empty[s], 1);
        }
        ptx::mbar_init(fin, 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (threadIdx.x < TC_M) rcnt[threadIdx.x] = 0;
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         ptx::smem_addr((const void*)tmem_slot)), "n"(TC_TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t wl = g_tc_wait;

    // warp-uniform bounded wait: every lane polls, the warp agrees
    auto waitw = [&](uint64_t* bar, uint32_t parity, uint32_t where) -> bool {
        bool ok = (*abort_flag == 0) && ptx::mbar_wait_bounded(bar, parity, wl);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok && lane == 0 && *abort_flag == 0) {
            *abort_flag = 1;
            dev_error(ix.status, DEV_TIMEOUT, where);
        }
        return ok;
    };

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        int64_t gt = 0, qi = 0;
        bool stop = false;
        for (int64_t it = blockIdx.x; it < sp.n_items && !stop; it += gridDim.x) {
            const TcItem I = tc_item(it, ix, n_blk, pos, Nq, W, sp);
            if (I.t1 <= I.t0) continue;
            const int qb = (int)(qi & 1);
            if (!waitw(&q_empty[qb], (uint32_t)(((qi >> 1) & 1) ^ 1), 1000u)) break;
            if (lane == 0) {
                ptx::mbar_arrive_expect_tx(&q_full[qb], TC_Q_BYTES);
                tma_load_2d(q_s + qb * TC_Q_BYTES, &tmQ, 0, (int)(I.b * Nq + I.q0), &q_full[qb]);
            }
            ++qi;
            for (int t = I.t0; t < I.t1; ++t, ++gt) {
                const int s = (int)(gt % TC_STAGES);
                if (!waitw(&empty[s], (uint32_t)(((gt / TC_STAGES) & 1) ^ 1), 1100u)) {
                    stop = true;
                    break;
                }
                if (lane == 0) {
                    ptx::mbar_arrive_expect_tx(&full[s], TC_C_BYTES);
                    tma_load_2d(c_s + s * TC_C_BYTES, &tmC, 0,
                                (int)(I.b * ix.NBK + (int64_t)t * TC_N), &full[s]);
                }
            }
        }
        if (*abort_flag && lane == 0) {
            // no copy may still be writing shared memory when the CTA exits:
            // the latest load of every stage and query buffer has landed, or a
            // bounded wait gives up on it
            for (int64_t g = (gt > TC_STAGES ? gt - TC_STAGES : 0); g < gt; ++g)
                ptx::mbar_wait_bounded(&full[g % TC_STAGES], (uint32_t)((g / TC_STAGES) & 1),
                                       TC_WAIT);
            for (int64_t q = (qi > 2 ? qi - 2 : 0); q < qi; ++q)
                ptx::mbar_wait_bounded(&q_full[q & 1], (uint32_t)((q >> 1) & 1), TC_WAIT);
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        int64_t gt = 0, qi = 0;
        bool stop = false;
        for (int64_t it = blockIdx.x; it < sp.n_items && !stop; it += gridDim.x) {
            const TcItem I = tc_item(it, ix, n_blk, pos, Nq, W, sp);
            if (I.t1 <= I.t0) continue;
            const int qb = (int)(qi & 1);
            if (!waitw(&q_full[qb], (uint32_t)((qi >> 1) & 1), 2000u)) break;
            const uint64_t adesc = sw128_desc(q_s + qb * TC_Q_BYTES);
            ++qi;
            for (int t = I.t0; t < I.t1; ++t, ++gt) {
                const int s = (int)(gt % TC_STAGES);
                const int buf = (int)(gt & 1);
                if (!waitw(&full[s], (uint32_t)((gt / TC_STAGES) & 1), 2100u) ||
                    !waitw(&acc_empty[buf], (uint32_t)(((gt >> 1) & 1) ^ 1), 2200u)) {
                    stop = true;
                    break;
                }
                tc_fence_after();
                if (lane == 0) {
                    const uint64_t bdesc = sw128_desc(c_s + s * TC_C_BYTES);
                    const uint32_t d = tmem + (uint32_t)(buf * TC_N);
#pragma unroll
                    for (int kk = 0; kk < DL / 16; ++kk)
                        mma_bf16(d, adesc + 2ull * kk, bdesc + 2ull * kk, TC_IDESC, kk > 0 ? 1u : 0u);
                    mma_commit(&empty[s]);
                    mma_commit(&acc_full[buf]);
                }
                __syncwarp();
            }
            if (!stop && lane == 0) mma_commit(&q_empty[qb]);
            __syncwarp();
        }
        // nothing of this CTA may still run on the tensor cores when TMEM is freed
        if (lane == 0) {
            mma_commit(fin);
            ptx::mbar_wait_bounded(fin, 0, TC_WAIT);
        }
        __syncwarp();
    } else {
        // ---------------- epilogue ----------------
        const int et = threadIdx.x - 64;                  // 0 .. TC_EPI_THREADS - 1
        const int sl = (warp - 2) >> 2;                   // column slice of every tile
        const int r = 32 * (warp & 3) + lane;             // query row = TMEM lane
        const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
        const int gl = sp.gw_log2;                        // 2 .. 6
        const unsigned FULL = 0xffffffffu;
        int64_t gt = 0;
        for (int64_t it = blockIdx.x; it < sp.n_items; it += gridDim.x) {
            const TcItem I = tc_item(it, ix, n_blk, pos, Nq, W, sp);
            const bool row_valid = I.q0 + r < Nq;
            const int64_t row = I.b * Nq + I.q0 + r;
            const int64_t nb_row =
                row_valid ? tc_eligible(ix, n_blk, pos.at(I.b, Nq, I.q0 + r), W) : 0;
            const int64_t lslot = row * sp.n_split + I.s;
            if (I.t1 <= I.t0) {
                if (PASS == 2 && sl == 0 && row_valid) {
                    ws.lst_n[lslot] = 0;
                    ws.lst_tau[lslot] = -INFINITY;
                }
                continue;
            }
            const float theta = (PASS == 2 && row_valid) ? ws.theta[row] : -INFINITY;
            uint16_t* grow = ws.gmax + row * ws.n_grp;
            float lost = -INFINITY;
            const bool go = __all_sync(FULL, *abort_flag == 0);   // warp-uniform
            for (int t = I.t0; t < I.t1; ++t, ++gt) {
                const int buf = (int)(gt & 1);
                const bool ok = go && waitw(&acc_full[buf], (uint32_t)((gt >> 1) & 1), 4000u);
                if (ok) {
                    tc_fence_after();
                    float va[TC_COLS];
                    __syncwarp();
                    tmem_ld64(tmem + lane_base + (uint32_t)(buf * TC_N + sl * TC_COLS), va);
                    // the accumulator is in registers: hand it back before the work
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(&acc_empty[buf]);
                    const int64_t gh = (int64_t)t * TC_N + sl * TC_COLS;   // first column here
                    if (PASS == 1 && row_valid && gh < nb_row) {
                        // group maxima of the eligible scores, as fp16 keys
                        // rounded down (0 = no eligible score in the group)
                        if (gh + TC_COLS > nb_row) {
#pragma unroll
                            for (int j = 0; j < TC_COLS; ++j)
                                if (gh + j >= nb_row) va[j] = -INFINITY;
                        }
                        auto key = [](float x) -> uint32_t {
                            return x > -INFINITY ? tc_half_key(__float2half_rd(x)) : 0u;
                        };
                        float m32[2];
#pragma unroll
                        for (int c = 0; c < 2; ++c) {
                            const float* v = va + 32 * c;
                            float m16[16], m8[8], m4[4], m2[2];
#pragma unroll
                            for (int j = 0; j < 16; ++j) m16[j] = fmaxf(v[2 * j], v[2 * j + 1]);
#pragma unroll
                            for (int j = 0; j < 8; ++j) m8[j] = fmaxf(m16[2 * j], m16[2 * j + 1]);
#pragma unroll
                            for (int j = 0; j < 4; ++j) m4[j] = fmaxf(m8[2 * j], m8[2 * j + 1]);
#pragma unroll
                            for (int j = 0; j < 2; ++j) m2[j] = fmaxf(m4[2 * j], m4[2 * j + 1]);
                            m32[c] = fmaxf(m2[0], m2[1]);
                            const int64_t g0 = gh + 32 * c;
                            if (gl == 4) {
                                *reinterpret_cast<uint32_t*>(grow + (g0 >> 4)) =
                                    key(m2[0]) | (key(m2[1]) << 16);
                            } else if (gl == 3) {
                                *reinterpret_cast<uint2*>(grow + (g0 >> 3)) =
                                    make_uint2(key(m4[0]) | (key(m4[1]) << 16),
                                               key(m4[2]) | (key(m4[3]) << 16));
                            } else if (gl == 2) {
                                *reinterpret_cast<uint4*>(grow + (g0 >> 2)) =
                                    make_uint4(key(m8[0]) | (key(m8[1]) << 16),
                                               key(m8[2]) | (key(m8[3]) << 16),
                                               key(m8[4]) | (key(m8[5]) << 16),
                                               key(m8[6]) | (key(m8[7]) << 16));
                            }
                        }
                        if (gl == 5)
                            *reinterpret_cast<uint32_t*>(grow + (gh >> 5)) =
                                key(m32[0]) | (key(m32[1]) << 16);
                        else if (gl == 6)
                            grow[gh >> 6] = (uint16_t)key(fmaxf(m32[0], m32[1]));
                    }
                    if (PASS == 2) {
                        // append every eligible score >= theta: 8-score
                        // sub-batches that no row of the warp can reach are
                        // skipped after one warp vote
                        uint64_t vm = 0ull;              // eligible columns of the 64
                        if (gh + TC_COLS <= nb_row) vm = ~0ull;
                        else if (gh < nb_row) vm = (1ull << (uint32_t)(nb_row - gh)) - 1ull;
                        float m16[32], m8[16];
#pragma unroll
                        for (int j = 0; j < 32; ++j) m16[j] = fmaxf(va[2 * j], va[2 * j + 1]);
#pragma unroll
                        for (int j = 0; j < 16; ++j) m8[j] = fmaxf(m16[2 * j], m16[2 * j + 1]);
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            const float* v = va + 8 * q;
                            const uint32_t em = (uint32_t)(vm >> (8 * q)) & 0xFFu;
                            const bool act = em != 0u && fmaxf(m8[2 * q], m8[2 * q + 1]) >= theta;
                            if (__any_sync(FULL, act)) {
                                uint32_t bits = 0u;
                                if (act) {
#pragma unroll
                                    for (int e = 0; e < 8; ++e) bits |= (v[e] >= theta) ? (1u << e) : 0u;
                                    bits &= em;
                                }
                                while (bits) {
                                    const int e = __ffs(bits) - 1;
                                    bits &= bits - 1u;
                                    const int slot = atomicAdd(&rcnt[r], 1);
                                    if (slot < ws.lst_cap)
                                        ws.lst_g[lslot * ws.lst_cap + slot] = (int32_t)(gh + 8 * q + e);
                                    else
                                        lost = fmaxf(lost, pick8(v, e));
                                }
                            }
                        }
                    }
                }
                __syncwarp();
            }
            if (PASS == 2) {
                lostv[et] = lost;
                epi_sync();
                if (sl == 0) {
                    if (row_valid) {
                        // the row's four threads (one per column slice)
                        const float l2 = fmaxf(fmaxf(lost, lostv[et + 128]),
                                               fmaxf(lostv[et + 256], lostv[et + 384]));
                        ws.lst_n[lslot] = min(rcnt[r], ws.lst_cap);
                        ws.lst_tau[lslot] = (theta > -INFINITY) ? fmaxf(theta, l2) : l2;
                    }
                    rcnt[r] = 0;
                }
                epi_sync();      // the counters are clear before the next item appends
            }
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

constexpr int TH_REG = 64;   // group-maximum keys per lane held in registers (2048 per row)
constexpr int TH_WARPS = 8;

// The bin (0 .. 255) holding the want-th largest count-weighted entry of a
// warp's 256-bin histogram, bins counted from the top; *above receives the
// entries in higher bins.  Lane l reads bins 255-8l .. 248-8l.
__device__ __forceinline__ int th_bin(const unsigned* hist, int want, int* above)
{
    const int lane = threadIdx.x & 31;
    unsigned hb[8], tot = 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        hb[e] = hist[255 - 8 * lane - e];
        tot += hb[e];
    }
    unsigned incl = tot;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const unsigned y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    const unsigned excl = incl - tot;
    int bin = -1, abv = 0;
    if (excl < (unsigned)want && incl >= (unsigned)want) {
        unsigned cum = excl;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            if (bin < 0 && cum + hb[e] >= (unsigned)want) {
                bin = 255 - 8 * lane - e;
                abv = (int)cum;
            }
            cum += hb[e];
        }
    }
    const unsigned who = __ballot_sync(0xffffffffu, bin >= 0);
    if (!who) {                 // fewer than want entries (not reached: callers check)
        *above = 0;
        return -1;
    }
    const int src = __ffs(who) - 1;
    *above = __shfl_sync(0xffffffffu, abv, src);
    return __shfl_sync(0xffffffffu, bin, src);
}

// theta of every query row: a warp per row finds the m-th largest of the
// row's group maxima (16-bit keys) by a two-pass radix select, high byte then
// low byte, over keys held in registers.  A row with at most KCF eligible
// buckets gets -inf (its lists take every eligible bucket); a row with fewer
// than 2m groups uses half of them.
__global__ void __launch_bounds__(32 * TH_WARPS) score_theta_kernel(IndexView ix, int64_t n_blk,
                                                                    PosSrc pos, int64_t Nq,
                                                                    int W, SelectWs ws, TcSplit sp)
{
    __shared__ unsigned hist_s[TH_WARPS][256];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t row = (int64_t)blockIdx.x * TH_WARPS + warp;
    if (row >= ix.B * Nq) return;                 // warp-uniform; no CTA barrier here
    unsigned* hist = hist_s[warp];
    const int64_t b = row / Nq, i = row % Nq;
    const int64_t nb = tc_eligible(ix, n_blk, pos.at(b, Nq, i), W);
    if (nb <= KCF) {
        if (lane == 0) ws.theta[row] = -INFINITY;
        return;
    }
    const int64_t ng = (nb + (1 << sp.gw_log2) - 1) >> sp.gw_log2;
    const int m = (int)min((int64_t)sp.m, max((int64_t)1, ng / 2));
    const uint16_t* keys = ws.gmax + row * ws.n_grp;
    uint32_t th;
    if (ng <= 32 * TH_REG) {
        // keys in registers, 8 per 16-byte load (n_grp is a multiple of 8;
        // keys past ng count as 0, which no bin below 1 holds)
        uint32_t kw[TH_REG / 2];
        const uint4* k4 = reinterpret_cast<const uint4*>(keys);
        const int n_u = (int)((ng + 255) / 256);              // 16-byte chunks per lane in use
#pragma unroll
        for (int u = 0; u < TH_REG / 8; ++u) {
            const int64_t c = (int64_t)u * 32 + lane;        // 16-byte chunk
            uint4 w = make_uint4(0u, 0u, 0u, 0u);
            if (u < n_u && c * 8 < ng) w = k4[c];
            const uint32_t e[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                uint32_t x = e[q];
                const int64_t k0 = c * 8 + 2 * q;
                if (k0 >= ng) x = 0u;
                else if (k0 + 1 >= ng) x &= 0xFFFFu;
                kw[u * 4 + q] = x;
            }
        }
        // high byte
#pragma unroll
        for (int e = 0; e < 8; ++e) hist[8 * lane + e] = 0u;
        __syncwarp();
#pragma unroll
        for (int u = 0; u < TH_REG / 8; ++u) {
            if (u >= n_u) break;                              // warp-uniform
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const uint32_t k = (q & 1) ? (kw[4 * u + q / 2] >> 16) : (kw[4 * u + q / 2] & 0xFFFFu);
                if (k) atomicAdd(&hist[k >> 8], 1u);
            }
        }
        __syncwarp();
        int above;
        const int b1 = th_bin(hist, m, &above);
        const int m2 = m - above;
        // low byte among the keys of that high byte
        __syncwarp();
#pragma unroll
        for (int e = 0; e < 8; ++e) hist[8 * lane + e] = 0u;
        __syncwarp();
#pragma unroll
        for (int u = 0; u < TH_REG / 8; ++u) {
            if (u >= n_u) break;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const uint32_t k = (q & 1) ? (kw[4 * u + q / 2] >> 16) : (kw[4 * u + q / 2] & 0xFFFFu);
                if (k && (int)(k >> 8) == b1) atomicAdd(&hist[k & 255u], 1u);
            }
        }
        __syncwarp();
        int above2;
        const int b2 = (b1 >= 0) ? th_bin(hist, m2, &above2) : -1;
        th = (b1 >= 0 && b2 >= 0) ? (((uint32_t)b1 << 8) | (uint32_t)b2) : 0u;
    } else {
        uint32_t lo = 1u, hi = 0xFFFFu;               // count(key >= lo) >= m
        while (lo < hi) {
            const uint32_t mid = (lo + hi + 1u) >> 1;
            int cnt = 0;
            for (int64_t x = lane; x < ng; x += 32) cnt += keys[x] >= mid;
            cnt = __reduce_add_sync(0xffffffffu, cnt);
            if (cnt >= m) lo = mid;
            else hi = mid - 1u;
        }
        th = lo;
    }
    // key 0 marks no threshold found: every eligible bucket is listed
    if (lane == 0) ws.theta[row] = th ? tc_key_value(th) : -INFINITY;
}

// ---- host side ---------------------------------------------------------------
bool tc_scoring_available() { return true; }

// The widest group (2^gl buckets, gl = 2 .. 6) that still leaves a sequence of
// n buckets at least 4m groups.
static int tc_group_log2(int64_t n, int m)
{
    int gl = 6;
    while (gl > 2 && (n >> gl) < 4LL * m) --gl;
    return gl;
}

TcSplit tc_split_plan(const IndexView& ix, int64_t Nq, int64_t n_blk)
{
    TcSplit sp;
    sp.n_qt = (Nq + TC_M - 1) / TC_M;
    const int64_t n_ct = (ix.NBK + TC_N - 1) / TC_N;       // centroid tiles of a sequence
    const int64_t tiles = ix.B * sp.n_qt;
    // enough items for the persistent CTAs to end within one item of each other
    int ns = 1;
    while (ns < TC_MAX_SPLITS && tiles * ns < 4LL * sm_count() && ns < n_ct) ns *= 2;
    sp.tps = (int)((n_ct + ns - 1) / ns);
    sp.n_split = (int)((n_ct + sp.tps - 1) / sp.tps);
    if (sp.n_split < 1) sp.n_split = 1;
    sp.n_items = tiles * sp.n_split;
    // groups of 64 scores (one per epilogue thread and tile), narrower (down
    // to 4) while the sequence's buckets -- those of the blocks closed so far,
    // not the capacity -- make fewer than 4m groups: with g groups and the m-th
    // largest maximum as the threshold, scores without structure put about
    // -g ln(1 - m/g) ~ m (1 + m / 2g) of them above it
    sp.m = TC_TARGET;
    int64_t nb_now = (n_blk < 0 ? 0 : n_blk) * ix.k;
    if (nb_now > ix.NBK) nb_now = ix.NBK;
    sp.gw_log2 = tc_group_log2(nb_now, sp.m);
    // row stride: the capacity's groups at the capacity's width, and at least
    // 8m (a narrower width is picked only while the buckets make fewer than
    // 8m groups at it); rows of keys start on 16 bytes
    int64_t ng = (n_ct * TC_N) >> tc_group_log2(ix.NBK, sp.m);
    if (ng < 8LL * sp.m) ng = 8LL * sp.m;
    sp.n_grp = (ng + 7) / 8 * 8;
    return sp;
}

cudaError_t set_score_wait_polls(int64_t polls)
{
    const uint32_t v = (polls < 0 || polls > (int64_t)TC_WAIT) ? TC_WAIT : (uint32_t)polls;
    return cudaMemcpyToSymbol(g_tc_wait, &v, sizeof(v));
}

cudaError_t launch_score_lists_tc(const IndexView& ix, int64_t n_blk, const void* latent_Q,
                                  PosSrc pos, int64_t Nq, int W, const SelectWs& ws,
                                  cudaStream_t st)
{
    if (ix.dtype != LSA_BF16) return cudaErrorInvalidValue;
    const TcSplit sp = tc_split_plan(ix, Nq, n_blk);
    if (ws.n_lst != sp.n_split || ws.lst_cap != TC_LIST_CAP || !ws.gmax || !ws.theta ||
        ws.n_grp != sp.n_grp)
        return cudaErrorInvalidValue;
    CUtensorMap tmQ, tmC;
    if (!tmap_rows64_bf16(&tmQ, latent_Q, (uint64_t)ix.B * Nq, TC_M) ||
        !tmap_rows64_bf16(&tmC, ix.cent_rt, (uint64_t)ix.B * ix.NBK, TC_N))
        return cudaErrorInvalidValue;
    cudaError_t e = ensure_smem_attr((const void*)score_tc_kernel<1>, TC_SMEM);
    if (e == cudaSuccess) e = ensure_smem_attr((const void*)score_tc_kernel<2>, TC_SMEM);
    if (e != cudaSuccess) return e;
    const unsigned n_cta = (unsigned)(sp.n_items < sm_count() ? sp.n_items : sm_count());
    score_tc_kernel<1><<<n_cta, TC_THREADS, TC_SMEM, st>>>(tmQ, tmC, ix, n_blk, pos, Nq, W, ws, sp);
    note_launch();
    const int64_t rows = ix.B * Nq;
    score_theta_kernel<<<(unsigned)((rows + TH_WARPS - 1) / TH_WARPS), 32 * TH_WARPS, 0, st>>>(
        ix, n_blk, pos, Nq, W, ws, sp);
    note_launch();
    score_tc_kernel<2><<<n_cta, TC_THREADS, TC_SMEM, st>>>(tmQ, tmC, ix, n_blk, pos, Nq, W, ws, sp);
    note_launch();
    return cudaGetLastError();
}

}  // namespace lsa
