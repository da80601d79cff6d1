// k_perkey.cu -- the brute-force latent per-key indexer: every long-range key
// of a query is scored against it and the R best are read (the indexer that
// LSA's bucket retrieval replaces; tcgen05 MMA, TMEM accumulators, TMA tile
// loads; sm_100a).
//
// Method: "Prefrontal's Latent Sparse Attention speeds up one attention layer
// 72x at 10M tokens ...", section "What it changes": the baseline indexer
// scores every earlier key for every query, quadratic in the context, and is
// most of a layer's prefill time; "Latent Sparse Attention: un indice
// gerarchico per contesti lunghi", paragraph on the read budget (R long-range
// keys outside the W most recent, S sinks).  The exact result: per query at
// pos, the keys t in [S, pos - W] ranked by <q, latent_k[t]> (binary64 sum of
// the exact products in ascending dimension), descending, ties to the lower
// position; the R first are taken.  Emitted: sinks, the taken keys in
// ascending position, the recent window.
//
// No [queries][keys] matrix is written.  Scores S = Q K^T (bf16 in, fp32
// accumulated) come from the tensor cores twice:
//   pass 1   (perkey_tc_kernel<1>) per query row, the maximum score of every
//            strided group {t : t mod ng = c} of eligible keys, rounded to
//            the nearest fp16 (rounding is monotone, so the rounded maximum
//            is the maximum of the rounded scores; -inf: no eligible key).
//            Strided groups spread a run of similar neighbouring keys over
//            many groups, so the R-th largest group maximum sits close to the
//            R-th largest score;
//   theta    (perkey_theta_kernel, a CTA per row) h = the R-th largest group
//            maximum; each of R groups holds a key scoring >= theta = h less
//            half an fp16 ulp (bounded by |h| 2^-10 + 2^-24; 65504 when h is
//            +inf), so the R-th largest exact score is >= theta - eps, where
//            eps bounds |fp32 score - exact score| by
//            2^-12 sum_d |q_d| max_t |k_t,d|.  The row's threshold is
//            theta - 2 eps, rounded down;
//   pass 2   (perkey_tc_kernel<2>) recomputes the scores and appends every
//            eligible key scoring >= the threshold: every key of the exact
//            top R is among them (its approximate score is >= its exact
//            score - eps >= theta - 2 eps);
//   final    (perkey_final_kernel, a CTA per row) ranks the candidates by
//            exact binary64 scores (radix select of the R-th largest (score,
//            lower position) pair), sorts the R taken positions and emits the
//            row;
//   fallback (perkey_fallback_kernel) rows whose candidates overflowed the
//            list (scores tied over more than PK_CAP keys) rank every
//            eligible key exactly, recomputing the scores in each radix pass.
//
// Work items of the tensor-core passes: (sequence, group block of 256
// columns, 128-query tile), query tile fastest, so that the persistent CTAs
// (one per SM) running at the same time read the same key tiles from L2.  An
// item sweeps the key tiles t0 = 256 gb + i ng, i = 0, 1, ...  CTA = 18 warps:
// warp 0 TMA producer (query tile, key tiles into a 4-deep ring, 128-byte
// swizzle), warp 1 TMEM owner and MMA issuer (M = 128, N = 256, K = 16, four
// per tile, two accumulators), warps 2-17 epilogue (thread = query row and 64
// columns of every tile, read from TMEM in 32-column pieces).  Pass 2
// stages a row's appended keys in shared memory and reserves their place in
// the row's list with one global atomic per row and item.  Every mbarrier
// wait is bounded; a timeout records DEV_TIMEOUT in the status word and the
// CTA drains and exits as the bucket scorer does.
#include <cuda.h>

#include <cuda_fp16.h>
#include <math.h>

#include "lsa_internal.cuh"
#include "ptx.cuh"
#include "tc_common.cuh"
#include "tmap.cuh"

namespace lsa {

constexpr int PK_M = 128;
constexpr int PK_N = 256;                                 // keys per tile
constexpr int PK_ACC = 2;                                 // TMEM accumulators
constexpr int PK_TMEM_COLS = PK_ACC * PK_N;
constexpr int PK_STAGES = 4;
constexpr int PK_EPI_WARPS = 16;
constexpr int PK_COLS = PK_N / 4;                         // columns per epilogue thread
constexpr int PK_ST = 128;                                // staged appends per row and item
constexpr int PK_EPI_THREADS = 32 * PK_EPI_WARPS;
constexpr int PK_THREADS = 64 + PK_EPI_THREADS;
constexpr uint32_t PK_WAIT = 1u << 22;
constexpr uint32_t PK_IDESC = tc_idesc_bf16(PK_M, PK_N);

__device__ uint32_t g_pk_wait = PK_WAIT;

constexpr int PK_Q_BYTES = PK_M * DL * 2;
constexpr int PK_K_BYTES = PK_N * DL * 2;
constexpr int PK_OFF_K = 2 * PK_Q_BYTES;
constexpr int PK_OFF_ST = PK_OFF_K + PK_STAGES * PK_K_BYTES;     // [PK_M][PK_ST] staged keys
constexpr int PK_OFF_BAR = PK_OFF_ST + PK_M * PK_ST * 4;
constexpr int PK_NBAR = 2 + 2 + 2 * PK_STAGES + 2 * PK_ACC + 1;
constexpr int PK_OFF_MISC = PK_OFF_BAR + PK_NBAR * 8;
constexpr int PK_SMEM = PK_OFF_MISC + 64 + PK_M * 4 + 1024;      // + staged counts, alignment

// Position of query i of sequence b, or -1 when it lies outside [0, n_keys)
// (such a row reads nothing and the final kernel reports DEV_BAD_INDEX).
__device__ __forceinline__ int64_t pk_pos(const PerKeyArgs& a, int64_t b, int64_t i)
{
    const int64_t p = a.pos[b * a.Nq + i];
    return (p >= 0 && p < a.n_keys) ? p : -1;
}

// Ordered 16-bit key of the fp16 bits u (larger value, larger key); -inf
// (no eligible key in the group, or every score below -65520) maps to 0.
__device__ __forceinline__ uint32_t pk_half_key(uint32_t u)
{
    if (u == 0xFC00u) return 0u;
    return (u & 0x8000u) ? (~u & 0xFFFFu) : (u | 0x8000u);
}

__device__ __forceinline__ float pk_key_value(uint32_t k)
{
    const uint16_t u = (k & 0x8000u) ? (uint16_t)(k & 0x7FFFu) : (uint16_t)(~k & 0xFFFFu);
    return __half2float(__ushort_as_half(u));
}

// Ordered 64-bit key of a binary64 value.
__device__ __forceinline__ uint64_t pk_dkey(double x)
{
    const uint64_t u = (uint64_t)__double_as_longlong(x);
    return (u >> 63) ? ~u : (u | 0x8000000000000000ull);
}

// <q, latent_k> of one key: the exact products summed in binary64 in
// ascending dimension (qd holds q in binary64).
__device__ __forceinline__ double pk_exact(const double* qd, const __nv_bfloat16* krow)
{
    const uint4* k4 = reinterpret_cast<const uint4*>(krow);
    double s = 0.0;
#pragma unroll
    for (int c = 0; c < DL / 8; ++c) {
        const uint4 w = k4[c];
        const uint32_t e[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const double lo = (double)__uint_as_float(e[j] << 16);
            const double hi = (double)__uint_as_float(e[j] & 0xFFFF0000u);
            s = __dadd_rn(s, __dmul_rn(qd[8 * c + 2 * j], lo));
            s = __dadd_rn(s, __dmul_rn(qd[8 * c + 2 * j + 1], hi));
        }
    }
    return s;
}

// Two keys at once (both rows' loads in flight, the two sums interleaved);
// each sum is pk_exact's, in the same order.
__device__ __forceinline__ void pk_exact2(const double* qd, const __nv_bfloat16* ka,
                                          const __nv_bfloat16* kb, double* sa, double* sb)
{
    const uint4* a4 = reinterpret_cast<const uint4*>(ka);
    const uint4* b4 = reinterpret_cast<const uint4*>(kb);
    uint4 wa[DL / 8], wb[DL / 8];
#pragma unroll
    for (int c = 0; c < DL / 8; ++c) {
        wa[c] = a4[c];
        wb[c] = b4[c];
    }
    double x = 0.0, y = 0.0;
#pragma unroll
    for (int c = 0; c < DL / 8; ++c) {
        const uint32_t ea[4] = {wa[c].x, wa[c].y, wa[c].z, wa[c].w};
        const uint32_t eb[4] = {wb[c].x, wb[c].y, wb[c].z, wb[c].w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const double q0 = qd[8 * c + 2 * j], q1 = qd[8 * c + 2 * j + 1];
            x = __dadd_rn(x, __dmul_rn(q0, (double)__uint_as_float(ea[j] << 16)));
            y = __dadd_rn(y, __dmul_rn(q0, (double)__uint_as_float(eb[j] << 16)));
            x = __dadd_rn(x, __dmul_rn(q1, (double)__uint_as_float(ea[j] & 0xFFFF0000u)));
            y = __dadd_rn(y, __dmul_rn(q1, (double)__uint_as_float(eb[j] & 0xFFFF0000u)));
        }
    }
    *sa = x;
    *sb = y;
}

// ---------------------------------------------------------------------------
// max_t |latent_k[t][d]| over keys [0, n_keys) of every sequence, as fp32 bits
// (non-negative floats order like their bits); colmax is zero before.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) perkey_colmax_kernel(PerKeyArgs a, PerKeyWs ws)
{
    __shared__ float red[8][DL];
    const int64_t b = blockIdx.y;
    const int c = threadIdx.x & 7;            // 8 dimensions (16 bytes) of a row
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint4* lat = reinterpret_cast<const uint4*>(a.lat_k) + b * a.T_cap * (DL / 8);
    float m[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) m[j] = 0.f;
    for (int64_t t = (int64_t)blockIdx.x * 32 + (threadIdx.x >> 3); t < a.n_keys;
         t += (int64_t)gridDim.x * 32) {
        const uint4 w = lat[t * (DL / 8) + c];
        const uint32_t e[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            m[2 * j] = fmaxf(m[2 * j], fabsf(__uint_as_float(e[j] << 16)));
            m[2 * j + 1] = fmaxf(m[2 * j + 1], fabsf(__uint_as_float(e[j] & 0xFFFF0000u)));
        }
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        m[j] = fmaxf(m[j], __shfl_xor_sync(0xffffffffu, m[j], 8));
        m[j] = fmaxf(m[j], __shfl_xor_sync(0xffffffffu, m[j], 16));
    }
    if (lane < 8) {
#pragma unroll
        for (int j = 0; j < 8; ++j) red[warp][8 * lane + j] = m[j];
    }
    __syncthreads();
    if (threadIdx.x < DL) {
        float v = 0.f;
        for (int w = 0; w < 8; ++w) v = fmaxf(v, red[w][threadIdx.x]);
        atomicMax(&ws.colmax[b * DL + threadIdx.x], __float_as_uint(v));
    }
}

// ---------------------------------------------------------------------------
// The two tensor-core passes.
// ---------------------------------------------------------------------------
struct PkItem {
    int64_t b, q0;
    int64_t gb;      // group block: columns [256 gb, 256 gb + 256) of every row
    int n_t;         // key tiles t0 = 256 gb + i ng, i < n_t
};

// Every lane of the calling warp takes part (warp-collective).
__device__ __forceinline__ PkItem pk_item(int64_t it, const PerKeyArgs& a, int64_t ng,
                                          int64_t n_qt)
{
    PkItem r;
    const int64_t n_gb = ng / PK_N;
    const int64_t qt = it % n_qt;
    const int64_t rest = it / n_qt;
    r.gb = rest % n_gb;
    r.b = rest / n_gb;
    r.q0 = qt * PK_M;
    const int lane = threadIdx.x & 31;
    int hm = -1;                                   // largest eligible key of the tile's rows
#pragma unroll
    for (int u = 0; u < PK_M / 32; ++u) {
        const int64_t q = r.q0 + lane + 32 * u;
        if (q < a.Nq) {
            const int64_t p = pk_pos(a, r.b, q);
            if (p >= 0 && p - a.W >= a.S && (int)(p - a.W) > hm) hm = (int)(p - a.W);
        }
    }
    hm = __reduce_max_sync(0xffffffffu, hm);
    const int64_t c0 = r.gb * PK_N;
    r.n_t = (a.R > 0 && hm >= 0 && hm >= c0) ? (int)((hm - c0) / ng + 1) : 0;
    return r;
}

// Named barrier of the epilogue warps only.
__device__ __forceinline__ void pk_epi_sync()
{
    asm volatile("bar.sync 1, %0;" ::"n"(PK_EPI_THREADS) : "memory");
}

template <int PASS>
__global__ void __launch_bounds__(PK_THREADS, 1) perkey_tc_kernel(
    const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK, PerKeyArgs a,
    PerKeyWs ws, int64_t n_qt, int64_t n_items)
{
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem =
        (unsigned char*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);  // 1 KB aligned
    unsigned char* q_s = smem;                        // [2][PK_Q_BYTES]
    unsigned char* k_s = smem + PK_OFF_K;             // [PK_STAGES][PK_K_BYTES]
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + PK_OFF_BAR);
    uint64_t* q_full = bars;
    uint64_t* q_empty = bars + 2;
    uint64_t* full = bars + 4;
    uint64_t* empty = full + PK_STAGES;
    uint64_t* acc_full = empty + PK_STAGES;     // [PK_ACC]
    uint64_t* acc_empty = acc_full + PK_ACC;    // [PK_ACC]
    uint64_t* fin = acc_empty + PK_ACC;
    uint32_t* misc = reinterpret_cast<uint32_t*>(smem + PK_OFF_MISC);
    volatile uint32_t* tmem_slot = misc;
    volatile uint32_t* abort_flag = misc + 1;
    int32_t* st_buf = reinterpret_cast<int32_t*>(smem + PK_OFF_ST);        // [PK_M][PK_ST]
    int* st_cnt = reinterpret_cast<int*>(smem + PK_OFF_MISC + 64);          // [PK_M]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t ng = ws.ng;
    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(&q_full[i], 1);
            ptx::mbar_init(&q_empty[i], 1);
        }
        for (int i = 0; i < PK_ACC; ++i) {
            ptx::mbar_init(&acc_full[i], 1);
            ptx::mbar_init(&acc_empty[i], PK_EPI_WARPS);
        }
        for (int s = 0; s < PK_STAGES; ++s) {
            ptx::mbar_init(&full[s], 1);
            ptx::mbar_init(&empty[s], 1);
        }
        ptx::mbar_init(fin, 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (threadIdx.x < PK_M) st_cnt[threadIdx.x] = 0;
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         ptx::smem_addr((const void*)tmem_slot)), "n"(PK_TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t wl = g_pk_wait;

    auto waitw = [&](uint64_t* bar, uint32_t parity, uint32_t where) -> bool {
        bool ok = (*abort_flag == 0) && ptx::mbar_wait_bounded(bar, parity, wl);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok && lane == 0 && *abort_flag == 0) {
            *abort_flag = 1;
            dev_error(ws.status, DEV_TIMEOUT, where);
        }
        return ok;
    };

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        int64_t gt = 0, qi = 0;
        bool stop = false;
        for (int64_t it = blockIdx.x; it < n_items && !stop; it += gridDim.x) {
            const PkItem I = pk_item(it, a, ng, n_qt);
            if (I.n_t == 0) continue;
            const int qb = (int)(qi & 1);
            if (!waitw(&q_empty[qb], (uint32_t)(((qi >> 1) & 1) ^ 1), 5000u)) break;
            if (lane == 0) {
                ptx::mbar_arrive_expect_tx(&q_full[qb], PK_Q_BYTES);
                tma_load_2d(q_s + qb * PK_Q_BYTES, &tmQ, 0, (int)(I.b * a.Nq + I.q0), &q_full[qb]);
            }
            ++qi;
            for (int i = 0; i < I.n_t; ++i, ++gt) {
                const int s = (int)(gt % PK_STAGES);
                if (!waitw(&empty[s], (uint32_t)(((gt / PK_STAGES) & 1) ^ 1), 5100u)) {
                    stop = true;
                    break;
                }
                if (lane == 0) {
                    const int64_t t0 = I.gb * PK_N + (int64_t)i * ng;
                    ptx::mbar_arrive_expect_tx(&full[s], PK_K_BYTES);
                    tma_load_2d(k_s + s * PK_K_BYTES, &tmK, 0, (int)(I.b * a.T_cap + t0), &full[s]);
                }
            }
        }
        if (*abort_flag && lane == 0) {
            for (int64_t g = (gt > PK_STAGES ? gt - PK_STAGES : 0); g < gt; ++g)
                ptx::mbar_wait_bounded(&full[g % PK_STAGES], (uint32_t)((g / PK_STAGES) & 1),
                                       PK_WAIT);
            for (int64_t q = (qi > 2 ? qi - 2 : 0); q < qi; ++q)
                ptx::mbar_wait_bounded(&q_full[q & 1], (uint32_t)((q >> 1) & 1), PK_WAIT);
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        int64_t gt = 0, qi = 0;
        bool stop = false;
        for (int64_t it = blockIdx.x; it < n_items && !stop; it += gridDim.x) {
            const PkItem I = pk_item(it, a, ng, n_qt);
            if (I.n_t == 0) continue;
            const int qb = (int)(qi & 1);
            if (!waitw(&q_full[qb], (uint32_t)((qi >> 1) & 1), 6000u)) break;
            const uint64_t adesc = sw128_desc(q_s + qb * PK_Q_BYTES);
            ++qi;
            for (int i = 0; i < I.n_t; ++i, ++gt) {
                const int s = (int)(gt % PK_STAGES);
                const int buf = (int)(gt % PK_ACC);
                if (!waitw(&full[s], (uint32_t)((gt / PK_STAGES) & 1), 6100u) ||
                    !waitw(&acc_empty[buf], (uint32_t)(((gt / PK_ACC) & 1) ^ 1), 6200u)) {
                    stop = true;
                    break;
                }
                tc_fence_after();
                if (lane == 0) {
                    const uint64_t bdesc = sw128_desc(k_s + s * PK_K_BYTES);
                    const uint32_t d = tmem + (uint32_t)(buf * PK_N);
#pragma unroll
                    for (int kk = 0; kk < DL / 16; ++kk)
                        mma_bf16(d, adesc + 2ull * kk, bdesc + 2ull * kk, PK_IDESC, kk > 0 ? 1u : 0u);
                    mma_commit(&empty[s]);
                    mma_commit(&acc_full[buf]);
                }
                __syncwarp();
            }
            if (!stop && lane == 0) mma_commit(&q_empty[qb]);
            __syncwarp();
        }
        if (lane == 0) {
            mma_commit(fin);
            ptx::mbar_wait_bounded(fin, 0, PK_WAIT);
        }
        __syncwarp();
    } else {
        // ---------------- epilogue ----------------
        const int sl = (warp - 2) >> 2;                   // column slice of every tile
        const int r = 32 * (warp & 3) + lane;             // query row = TMEM lane
        const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
        const unsigned FULL = 0xffffffffu;
        uint32_t gt = 0;                                  // tiles so far (parities only)
        for (int64_t it = blockIdx.x; it < n_items; it += gridDim.x) {
            const PkItem I = pk_item(it, a, ng, n_qt);
            const bool row_valid = I.q0 + r < a.Nq;
            const int64_t row = I.b * a.Nq + I.q0 + r;
            int hi = -1;                                  // last eligible key of the row
            if (row_valid) {
                const int64_t p = pk_pos(a, I.b, I.q0 + r);
                if (p >= 0) hi = (int)(p - a.W);
            }
            const int lo = a.S;                           // keys (< 2^31) in 32 bits
            const float th = (PASS == 2 && row_valid) ? ws.theta[row] : INFINITY;
            __half2 m[PK_COLS / 2];                       // running maxima, two columns each
            if (PASS == 1) {
#pragma unroll
                for (int j = 0; j < PK_COLS / 2; ++j) m[j] = __half2half2(__ushort_as_half(0xFC00u));
            }
            const bool go = __all_sync(FULL, *abort_flag == 0);
            for (int i = 0; i < I.n_t; ++i, ++gt) {
                const int buf = (int)(gt % PK_ACC);
                const bool ok =
                    go && waitw(&acc_full[buf], (uint32_t)((gt / PK_ACC) & 1), 7000u);
                if (!ok) continue;
                tc_fence_after();
                const int c0 = (int)(I.gb * PK_N + (int64_t)i * ng) + sl * PK_COLS;   // first key here
                const uint32_t taddr = tmem + lane_base + (uint32_t)(buf * PK_N + sl * PK_COLS);
                if (PASS == 1) {
                    // running maxima of the eligible scores, column by column,
                    // 32 columns at a time
#pragma unroll
                    for (int h = 0; h < PK_COLS / 32; ++h) {
                        float v[32];
                        __syncwarp();
                        tmem_ld32(taddr + 32u * h, v);
                        if (h == PK_COLS / 32 - 1) {
                            // the accumulator is in registers: hand it back
                            tc_fence_before();
                            __syncwarp();
                            if (lane == 0) ptx::mbar_arrive(&acc_empty[buf]);
                        }
                        const int k0 = c0 + 32 * h;
                        if (k0 < lo || k0 + 31 > hi) {
#pragma unroll
                            for (int j = 0; j < 32; ++j)
                                if (k0 + j < lo || k0 + j > hi) v[j] = -INFINITY;
                        }
#pragma unroll
                        for (int j = 0; j < 16; ++j)
                            m[16 * h + j] = __hmax2(m[16 * h + j], __floats2half2_rn(v[2 * j], v[2 * j + 1]));
                    }
                } else {
                    float v[PK_COLS];
                    __syncwarp();
                    tmem_ld64(taddr, v);
                    // the accumulator is in registers: hand it back before the work
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(&acc_empty[buf]);
                    // append every eligible key scoring >= th; 8-score batches
                    // that no row of the warp reaches are skipped after a vote
                    uint64_t em = 0ull;                   // eligible columns of the 64
                    if (row_valid && hi >= lo) {
                        const int e0 = c0 < lo ? lo : c0;
                        const int e1 = (c0 + PK_COLS - 1 < hi) ? c0 + PK_COLS - 1 : hi;
                        if (e1 >= e0) {
                            const int n = e1 - e0 + 1, s0 = e0 - c0;
                            em = (n == 64 ? ~0ull : ((1ull << n) - 1ull)) << s0;
                        }
                    }
#pragma unroll
                    for (int q = 0; q < PK_COLS / 8; ++q) {
                        const float* w = v + 8 * q;
                        const float mx = fmaxf(fmaxf(fmaxf(w[0], w[1]), fmaxf(w[2], w[3])),
                                               fmaxf(fmaxf(w[4], w[5]), fmaxf(w[6], w[7])));
                        const uint32_t eb = (uint32_t)(em >> (8 * q)) & 0xFFu;
                        const bool act = eb != 0u && mx >= th;
                        if (__any_sync(FULL, act)) {
                            uint32_t bits = 0u;
                            if (act) {
#pragma unroll
                                for (int e = 0; e < 8; ++e) bits |= (w[e] >= th) ? (1u << e) : 0u;
                                bits &= eb;
                            }
                            if (bits) {
                                const int nb = __popc(bits);
                                int slot = atomicAdd(&st_cnt[r], nb);
                                // what finds the staging full goes straight to
                                // the row's list (one reservation per batch)
                                int g = 0;
                                if (slot + nb > PK_ST)
                                    g = atomicAdd(&ws.cnt[row], slot + nb - max(slot, PK_ST));
                                while (bits) {
                                    const int e = __ffs(bits) - 1;
                                    bits &= bits - 1u;
                                    const int32_t t = c0 + 8 * q + e;
                                    if (slot < PK_ST) {
                                        st_buf[r * PK_ST + slot] = t;
                                    } else {
                                        if (g < PK_CAP) ws.cand[row * PK_CAP + g] = t;
                                        ++g;
                                    }
                                    ++slot;
                                }
                            }
                        }
                    }
                }
                __syncwarp();
            }
            if (PASS == 2 && I.n_t > 0) {                 // block-uniform
                // the staged keys of each row go to its list: one reservation
                pk_epi_sync();
                if (sl == 0) {
                    const int n = min(st_cnt[r], PK_ST);
                    if (n > 0 && row_valid) {
                        const int base = atomicAdd(&ws.cnt[row], n);
                        for (int j = 0; j < n && base + j < PK_CAP; ++j)
                            ws.cand[row * PK_CAP + base + j] = st_buf[r * PK_ST + j];
                    }
                    st_cnt[r] = 0;
                }
                pk_epi_sync();
            }
            if (PASS == 1 && row_valid) {
                // the row's 64 group maxima of this block (fp16 bits)
                uint4* dst = reinterpret_cast<uint4*>(ws.gmax + row * ng + I.gb * PK_N + sl * PK_COLS);
#pragma unroll
                for (int c = 0; c < PK_COLS / 8; ++c) {
                    uint32_t w[4];
#pragma unroll
                    for (int j = 0; j < 4; ++j) w[j] = *reinterpret_cast<const uint32_t*>(&m[4 * c + j]);
                    dst[c] = make_uint4(w[0], w[1], w[2], w[3]);
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "n"(PK_TMEM_COLS)
                     : "memory");
    }
}

// ---------------------------------------------------------------------------
// Block-wide helpers (blockDim.x = NT, a multiple of 32, at most 1024).
// ---------------------------------------------------------------------------
// Exclusive prefix sum of one value per thread; *total receives the sum.
template <int NT>
__device__ __forceinline__ int pk_block_scan(int x, int* scratch, int* total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    __syncthreads();                        // scratch free from an earlier use
    if (lane == 31) scratch[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int w = (lane < NT / 32) ? scratch[lane] : 0;
        int wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += y;
        }
        if (lane < NT / 32) scratch[lane] = wi - w;
        if (lane == 31) scratch[32] = wi;
    }
    __syncthreads();
    *total = scratch[32];
    return scratch[warp] + incl - x;
}

// After a 256-bin histogram is complete: the bin holding the want-th largest
// entry (bins counted from the top), and the entries in higher bins.  Warp 0
// computes; every thread receives the answer.
template <int NT>
__device__ __forceinline__ void pk_hist_pick(const uint32_t* hist, uint32_t want, int* bin_out,
                                             uint32_t* above_out, uint32_t* bc)
{
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        uint32_t hb[8], tot = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            hb[e] = hist[255 - 8 * lane - e];
            tot += hb[e];
        }
        uint32_t incl = tot;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        const uint32_t excl = incl - tot;
        const uint32_t total = __shfl_sync(0xffffffffu, incl, 31);
        if (excl < want && incl >= want) {
            uint32_t cum = excl;
            int bin = -1;
            uint32_t abv = 0;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                if (bin < 0 && cum + hb[e] >= want) {
                    bin = 255 - 8 * lane - e;
                    abv = cum;
                }
                cum += hb[e];
            }
            bc[0] = (uint32_t)bin;
            bc[1] = abv;
        }
        if (lane == 0 && total < want) {
            bc[0] = 0xFFFFFFFFu;             // fewer than want entries
            bc[1] = 0u;
        }
    }
    __syncthreads();
    *bin_out = (int)bc[0];
    *above_out = bc[1];
    __syncthreads();
}

// ---------------------------------------------------------------------------
// theta: a CTA per row, the R-th largest strided-group maximum: the largest
// 16-bit key k with at least R keys >= k, by binary search over k with the
// row's keys held in registers (two per word, compared pairwise).
// ---------------------------------------------------------------------------
constexpr int PT_THREADS = 512;
constexpr int PT_WORDS = PK_NG_MAX / 2 / PT_THREADS;       // key pairs per thread (max)

__global__ void __launch_bounds__(PT_THREADS) perkey_theta_kernel(PerKeyArgs a, PerKeyWs ws)
{
    __shared__ int part[PT_THREADS / 32];
    const int64_t row = blockIdx.x;
    const int64_t b = row / a.Nq, i = row % a.Nq;
    const int64_t p = pk_pos(a, b, i);
    const int64_t n_valid = (p >= 0 && p - a.W >= a.S) ? p - a.W - a.S + 1 : 0;
    if (threadIdx.x == 0) ws.cnt[row] = 0;
    if (a.R == 0 || n_valid == 0) {
        if (threadIdx.x == 0) ws.theta[row] = INFINITY;          // no long-range key
        return;
    }
    if (n_valid <= a.R) {
        if (threadIdx.x == 0) ws.theta[row] = -INFINITY;         // every one of them
        return;
    }
    const int64_t ng = ws.ng;
    const int64_t n_c = ng / 8;                                  // 16-byte chunks of the row
    const uint4* k4 = reinterpret_cast<const uint4*>(ws.gmax + row * ng);
    uint32_t kw[PT_WORDS];
#pragma unroll
    for (int u = 0; u < PT_WORDS / 4; ++u) {
        const int64_t c = (int64_t)u * PT_THREADS + threadIdx.x;
        uint4 w = make_uint4(0u, 0u, 0u, 0u);
        if (c < n_c) w = k4[c];
        const uint32_t e[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int j = 0; j < 4; ++j)
            kw[4 * u + j] = (c < n_c) ? pk_half_key(e[j] & 0xFFFFu) | (pk_half_key(e[j] >> 16) << 16)
                                      : 0u;
    }
    const int warp = threadIdx.x >> 5;
    // largest k with count(key >= k) >= R; k = 0 (every key counts, ng >= R
    // here) always qualifies, so lo = 0 at the end means fewer than R groups
    // hold an eligible key
    uint32_t lo = 0u, hi = 0xFFFFu;
    while (lo < hi) {                            // block-uniform: every thread sums part[]
        const uint32_t mid = (lo + hi + 1u) >> 1;
        const uint32_t mid2 = mid | (mid << 16);
        int c = 0;
#pragma unroll
        for (int u = 0; u < PT_WORDS; ++u) c += __popc(__vcmpgeu2(kw[u], mid2));
        c = __reduce_add_sync(0xffffffffu, c) >> 4;
        __syncthreads();                         // part[] read by the previous step
        if ((threadIdx.x & 31) == 0) part[warp] = c;
        __syncthreads();
        int tot = 0;
#pragma unroll
        for (int w = 0; w < PT_THREADS / 32; ++w) tot += part[w];
        if (tot >= a.R) lo = mid;
        else hi = mid - 1u;
    }
    const bool found = lo > 0u;
    if (threadIdx.x == 0) {
        float th2 = -INFINITY;                   // fewer than R groups: every key
        if (found) {
            const float h = pk_key_value(lo);
            // at least R keys score >= theta (fp16 rounding of the maxima undone)
            const double theta = isinf(h) ? 65504.0
                                          : (double)h - (fabs((double)h) * 0x1p-10 + 0x1p-24);
            // eps >= |fp32 score - exact score| for every key of the sequence
            const __nv_bfloat16* q = reinterpret_cast<const __nv_bfloat16*>(a.lat_q) + row * DL;
            double l1 = 0.0;
            for (int d = 0; d < DL; ++d)
                l1 += fabs((double)__bfloat162float(q[d])) *
                      (double)__uint_as_float(ws.colmax[b * DL + d]);
            const double eps = ldexp(l1, -12) * (1.0 + 1e-12);
            th2 = __double2float_rd(theta - 2.0 * eps);
        }
        ws.theta[row] = th2;
    }
}

// ---------------------------------------------------------------------------
// final: a CTA per row.  The candidates' exact scores as ordered 64-bit keys;
// the R-th largest (score key, inverted position) pair by radix select -- the
// pairs are unique, so exactly R are at or above it, ties of the score going
// to the lower position; the four position passes are skipped when the cut's
// score is unique.  The R taken positions are compacted, sorted ascending
// (bitonic over R rounded up to a power of two) and emitted with the sinks
// and the window.
// ---------------------------------------------------------------------------
constexpr int PF_THREADS = 512;
constexpr int PF_PER = PK_CAP / PF_THREADS;                 // 16 candidates per thread
constexpr int PF_SMEM = PK_CAP * 4 + PK_CAP * 8 + DL * 8 + 256 * 4 + 40 * 4 + 16;

// Writes sinks [0, n_s) and the window [w0, p] around `taken` long-range
// entries already at out[n_s ..], pads with -1, and stores the count.
__device__ __forceinline__ void pk_emit_edges(const PerKeyArgs& a, int64_t row, int64_t p,
                                              int64_t taken)
{
    int32_t* out = a.indices + row * (int64_t)a.s_max;
    const int64_t n_s = p >= 0 ? (p + 1 < a.S ? p + 1 : a.S) : 0;
    const int64_t w0 = (p - a.W + 1 > n_s) ? p - a.W + 1 : n_s;
    const int64_t n_w = p >= 0 ? p - w0 + 1 : 0;
    for (int64_t x = threadIdx.x; x < n_s; x += blockDim.x) out[x] = (int32_t)x;
    for (int64_t x = threadIdx.x; x < n_w; x += blockDim.x) out[n_s + taken + x] = (int32_t)(w0 + x);
    for (int64_t x = n_s + taken + n_w + threadIdx.x; x < a.s_max; x += blockDim.x) out[x] = -1;
    if (threadIdx.x == 0) a.counts[row] = (int32_t)(n_s + taken + n_w);
}

// Bitonic sort of pos_s[0, P) ascending (P a power of two), whole CTA.
__device__ __forceinline__ void pk_bitonic(int32_t* pos_s, int P)
{
    for (int k = 2; k <= P; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            for (int x = threadIdx.x; x < P / 2; x += PF_THREADS) {
                const int lo = ((x & ~(j - 1)) << 1) | (x & (j - 1));   // j is a power of two
                const int hi = lo + j;
                const bool up = (lo & k) == 0;
                const int32_t u = pos_s[lo], v = pos_s[hi];
                if ((u > v) == up) {
                    pos_s[lo] = v;
                    pos_s[hi] = u;
                }
            }
            __syncthreads();
        }
    }
}

__global__ void __launch_bounds__(PF_THREADS) perkey_final_kernel(PerKeyArgs a, PerKeyWs ws)
{
    extern __shared__ unsigned char fsm[];
    uint64_t* key_s = reinterpret_cast<uint64_t*>(fsm);                      // [PK_CAP]
    int32_t* pos_s = reinterpret_cast<int32_t*>(fsm + PK_CAP * 8);           // [PK_CAP]
    double* q_s = reinterpret_cast<double*>(fsm + PK_CAP * 12);              // [DL]
    uint32_t* hist = reinterpret_cast<uint32_t*>(fsm + PK_CAP * 12 + DL * 8); // [256]
    int* scan = reinterpret_cast<int*>(hist + 256);                           // [40]
    uint32_t* bc = reinterpret_cast<uint32_t*>(scan + 40);                    // [2]
    const int64_t row = blockIdx.x;
    const int64_t b = row / a.Nq, i = row % a.Nq;
    const int64_t p = pk_pos(a, b, i);
    if (p < 0 && threadIdx.x == 0) dev_error(ws.status, DEV_BAD_INDEX, (uint32_t)a.pos[row]);
    const bool longr = a.R > 0 && p >= 0 && p - a.W >= a.S;
    const int n = longr ? ws.cnt[row] : 0;
    if (n > PK_CAP) {
        // list overflow: the fallback ranks every eligible key of the row
        if (threadIdx.x == 0) {
            const uint32_t slot = atomicAdd(&ws.status[3], 1u);
            ws.over[slot] = (int32_t)row;
            atomicAdd(&ws.status[1], 1u);
        }
        return;
    }
    const int32_t* cand = ws.cand + row * PK_CAP;
    for (int x = threadIdx.x; x < n; x += PF_THREADS) pos_s[x] = cand[x];
    if (threadIdx.x < DL)
        q_s[threadIdx.x] = (double)__bfloat162float(
            reinterpret_cast<const __nv_bfloat16*>(a.lat_q)[row * DL + threadIdx.x]);
    __syncthreads();
    int taken = n;
    if (n > a.R) {
        // exact scores as ordered keys, two rows in flight per thread
        const __nv_bfloat16* lat =
            reinterpret_cast<const __nv_bfloat16*>(a.lat_k) + b * a.T_cap * DL;
        for (int x = threadIdx.x; x < n; x += 2 * PF_THREADS) {
            const int y = x + PF_THREADS;
            double sx, sy;
            pk_exact2(q_s, lat + (int64_t)pos_s[x] * DL, lat + (int64_t)pos_s[y < n ? y : x] * DL,
                      &sx, &sy);
            key_s[x] = pk_dkey(sx);
            if (y < n) key_s[y] = pk_dkey(sy);
        }
        __syncthreads();
        // the R-th largest (key, ~position) pair: 8 passes over the key bytes,
        // then, unless the cut's key is unique among the rest, 4 over the
        // inverted position's bytes
        uint64_t kp = 0ull, km = 0ull;
        uint32_t ip = 0u, im = 0u;
        uint32_t want = (uint32_t)a.R;
        for (int pass = 0; pass < 12; ++pass) {
            const bool on_key = pass < 8;
            const int sh = on_key ? 56 - 8 * pass : 24 - 8 * (pass - 8);
            for (int x = threadIdx.x; x < 256; x += PF_THREADS) hist[x] = 0u;
            __syncthreads();
            for (int x = threadIdx.x; x < n; x += PF_THREADS) {
                const uint64_t k = key_s[x];
                if (on_key) {
                    if ((k & km) == kp) atomicAdd(&hist[(k >> sh) & 255u], 1u);
                } else if (k == kp) {
                    const uint32_t v = 0xFFFFFFFFu - (uint32_t)pos_s[x];
                    if ((v & im) == ip) atomicAdd(&hist[(v >> sh) & 255u], 1u);
                }
            }
            __syncthreads();
            int bin;
            uint32_t above;
            pk_hist_pick<PF_THREADS>(hist, want, &bin, &above, bc);
            const uint32_t in_bin = hist[bin];
            want -= above;
            if (on_key) {
                kp |= (uint64_t)(uint32_t)bin << sh;
                km |= 255ull << sh;
            } else {
                ip |= (uint32_t)bin << sh;
                im |= 255u << sh;
            }
            __syncthreads();                   // hist read before the next pass clears it
            if (pass == 7 && in_bin == want) break;    // every pair with the cut's key is taken
        }
        // compaction of the taken positions (pairs at or above the cut)
        int32_t mine[PF_PER];
        uint32_t fl = 0u;
        int nt = 0;
        const int x0 = threadIdx.x * PF_PER;
#pragma unroll
        for (int e = 0; e < PF_PER; ++e) {
            const int x = x0 + e;
            mine[e] = 0;
            if (x < n) {
                const uint64_t k = key_s[x];
                const int32_t t = pos_s[x];
                const bool take = k > kp || (k == kp && (0xFFFFFFFFu - (uint32_t)t) >= ip);
                mine[e] = t;
                if (take) {
                    fl |= 1u << e;
                    ++nt;
                }
            }
        }
        int o = pk_block_scan<PF_THREADS>(nt, scan, &taken);   // syncs before pos_s is rewritten
#pragma unroll
        for (int e = 0; e < PF_PER; ++e)
            if (fl & (1u << e)) pos_s[o++] = mine[e];
        __syncthreads();
    }
    // the taken positions ascending, then the row
    int P = 1;
    while (P < taken) P <<= 1;
    for (int x = taken + threadIdx.x; x < P; x += PF_THREADS) pos_s[x] = 0x7FFFFFFF;
    __syncthreads();
    pk_bitonic(pos_s, P);
    const int n_s = (int)(p >= 0 ? (p + 1 < a.S ? p + 1 : a.S) : 0);
    int32_t* out = a.indices + row * (int64_t)a.s_max + n_s;
    for (int x = threadIdx.x; x < taken; x += PF_THREADS) out[x] = pos_s[x];
    pk_emit_edges(a, row, p, taken);
}

// ---------------------------------------------------------------------------
// fallback: rows whose candidate list overflowed.  Every eligible key is
// ranked exactly; each radix pass recomputes the binary64 scores.
// ---------------------------------------------------------------------------
constexpr int PB_THREADS = 256;

__global__ void __launch_bounds__(PB_THREADS) perkey_fallback_kernel(PerKeyArgs a, PerKeyWs ws)
{
    __shared__ double q_s[DL];
    __shared__ uint32_t hist[256];
    __shared__ int scan[40];
    __shared__ uint32_t bc[2];
    const uint32_t n_over = ws.status[3];
    for (uint32_t oi = blockIdx.x; oi < n_over; oi += gridDim.x) {
        const int64_t row = ws.over[oi];
        const int64_t b = row / a.Nq, i = row % a.Nq;
        const int64_t p = pk_pos(a, b, i);
        const int64_t lo = a.S, hi = p - a.W;             // n_valid > PK_CAP >= R here
        const __nv_bfloat16* lat = reinterpret_cast<const __nv_bfloat16*>(a.lat_k) + b * a.T_cap * DL;
        __syncthreads();                                   // q_s free from the previous row
        if (threadIdx.x < DL)
            q_s[threadIdx.x] = (double)__bfloat162float(
                reinterpret_cast<const __nv_bfloat16*>(a.lat_q)[row * DL + threadIdx.x]);
        __syncthreads();
        uint64_t prefix = 0ull, mask = 0ull;
        uint32_t want = (uint32_t)a.R;
        for (int pass = 0; pass < 8; ++pass) {
            const int sh = 56 - 8 * pass;
            for (int x = threadIdx.x; x < 256; x += PB_THREADS) hist[x] = 0u;
            __syncthreads();
            for (int64_t t = lo + threadIdx.x; t <= hi; t += PB_THREADS) {
                const uint64_t k = pk_dkey(pk_exact(q_s, lat + t * DL));
                if ((k & mask) == prefix) atomicAdd(&hist[(k >> sh) & 255u], 1u);
            }
            __syncthreads();
            int bin;
            uint32_t above;
            pk_hist_pick<PB_THREADS>(hist, want, &bin, &above, bc);
            prefix |= (uint64_t)(uint32_t)bin << sh;
            mask |= 255ull << sh;
            want -= above;
        }
        const uint64_t cut = prefix;
        const uint32_t need = want;
        const int n_s = (int)(p + 1 < a.S ? p + 1 : a.S);
        int32_t* out = a.indices + row * (int64_t)a.s_max + n_s;
        int64_t taken = 0, eq_seen = 0;
        for (int64_t t0 = lo; t0 <= hi; t0 += PB_THREADS) {
            const int64_t t = t0 + threadIdx.x;
            uint64_t k = 0ull;
            if (t <= hi) k = pk_dkey(pk_exact(q_s, lat + t * DL));
            const int is_eq = (t <= hi && k == cut) ? 1 : 0;
            int n_eq;
            const int eq_rank = pk_block_scan<PB_THREADS>(is_eq, scan, &n_eq);
            const bool take = t <= hi && (k > cut || (is_eq && eq_seen + eq_rank < (int64_t)need));
            int n_take;
            const int o = pk_block_scan<PB_THREADS>(take ? 1 : 0, scan, &n_take);
            if (take) out[taken + o] = (int32_t)t;
            taken += n_take;
            eq_seen += n_eq;
        }
        pk_emit_edges(a, row, p, taken);
    }
}

// ---- host side ---------------------------------------------------------------
int64_t per_key_groups(int64_t T_cap)
{
    int64_t ng = PK_N;
    while (ng < T_cap && ng < PK_NG_MAX) ng <<= 1;
    return ng;
}

cudaError_t set_per_key_wait_polls(int64_t polls)
{
    const uint32_t v = (polls < 0 || polls > (int64_t)PK_WAIT) ? PK_WAIT : (uint32_t)polls;
    return cudaMemcpyToSymbol(g_pk_wait, &v, sizeof(v));
}

cudaError_t launch_per_key(const PerKeyArgs& a, const PerKeyWs& ws, cudaStream_t st)
{
    const int64_t rows = a.B * a.Nq;
    if (rows <= 0) return cudaSuccess;
    if (ws.ng != per_key_groups(a.T_cap)) return cudaErrorInvalidValue;
    if (a.R > 0) {
        CUtensorMap tmQ, tmK;
        if (!tmap_rows64_bf16(&tmQ, a.lat_q, (uint64_t)rows, PK_M) ||
            !tmap_rows64_bf16(&tmK, a.lat_k, (uint64_t)(a.B * a.T_cap), PK_N))
            return cudaErrorInvalidValue;
        cudaError_t e = ensure_smem_attr((const void*)perkey_tc_kernel<1>, PK_SMEM);
        if (e == cudaSuccess) e = ensure_smem_attr((const void*)perkey_tc_kernel<2>, PK_SMEM);
        if (e != cudaSuccess) return e;
        const int64_t per_seq = (a.n_keys + 31) / 32;
        const unsigned gx = (unsigned)(per_seq < 4LL * sm_count() ? per_seq : 4LL * sm_count());
        if (gx > 0) {
            perkey_colmax_kernel<<<dim3(gx, (unsigned)a.B), 256, 0, st>>>(a, ws);
            note_launch();
        }
        const int64_t n_qt = (a.Nq + PK_M - 1) / PK_M;
        const int64_t n_items = a.B * (ws.ng / PK_N) * n_qt;
        const unsigned n_cta = (unsigned)(n_items < sm_count() ? n_items : sm_count());
        perkey_tc_kernel<1><<<n_cta, PK_THREADS, PK_SMEM, st>>>(tmQ, tmK, a, ws, n_qt, n_items);
        note_launch();
        perkey_theta_kernel<<<(unsigned)rows, PT_THREADS, 0, st>>>(a, ws);
        note_launch();
        perkey_tc_kernel<2><<<n_cta, PK_THREADS, PK_SMEM, st>>>(tmQ, tmK, a, ws, n_qt, n_items);
        note_launch();
    }
    cudaError_t e = ensure_smem_attr((const void*)perkey_final_kernel, PF_SMEM);
    if (e != cudaSuccess) return e;
    perkey_final_kernel<<<(unsigned)rows, PF_THREADS, PF_SMEM, st>>>(a, ws);
    note_launch();
    const unsigned nb = (unsigned)(rows < 2LL * sm_count() ? rows : 2LL * sm_count());
    perkey_fallback_kernel<<<nb, PB_THREADS, 0, st>>>(a, ws);
    note_launch();
    return cudaGetLastError();
}

}  // namespace lsa
