// k_select.cu -- per-query bucket retrieval: candidate nomination, exact
// ranking, greedy budget fill, sinks + window, exact fallback.
//
// Method: "Latent Sparse Attention: un indice gerarchico per contesti
// lunghi", paragraph on retrieval (the query is compared with the centroids
// to choose the buckets whose keys are read) and paragraph on the read budget
// (a fixed number of long-range keys outside the recent window, the most
// recent keys, and sink keys at the start of the sequence).
//
// Exactness.  The ranking that decides the selection uses exact binary64
// scores (exact products of the binary32/bf16 inputs summed in ascending
// dimension), identical bit for bit to a sequential evaluation.  A cheaper
// binary32 (or tensor-core) pass only nominates KC candidate buckets per
// query together with tau, an upper bound of the approximate score of every
// bucket it did not nominate.  With |approx - exact| <= eps for every bucket,
// the candidates' exact ranking is the true ranking up to the bucket c at
// which the fill stops whenever exact(c) > tau + eps; otherwise (or when the
// candidates run out while more keys are available) the query is sent to an
// exact fallback that ranks every bucket.
#include <float.h>

#include "lsa_internal.cuh"

namespace lsa {

// Buckets of the closed blocks whose first key lies at or below pos - W (the
// only ones that can hold an available key).
__device__ __forceinline__ int64_t eligible_buckets(const IndexView& ix, int64_t n_blk, int64_t pos,
                                                    int W)
{
    const int64_t hi = pos - W;
    if (hi < 0) return 0;
    const int64_t span = (int64_t)ix.p * ix.G;
    int64_t nb = hi / span + 1;
    if (nb > n_blk) nb = n_blk;
    return nb * ix.k;
}

// Keys of pooled group j inside [S, hi].
__device__ __forceinline__ int group_avail(int64_t j, int p, int64_t S, int64_t hi)
{
    int64_t lo = j * p, up = lo + p - 1;
    if (lo < S) lo = S;
    if (up > hi) up = hi;
    return (up >= lo) ? (int)(up - lo + 1) : 0;
}

__device__ __forceinline__ float rt_load(const IndexView& ix, int64_t bseq, int64_t g, int i)
{
    const int64_t x = (bseq * ix.NBK + g) * DL + i;
    if (ix.dtype == LSA_BF16) return __bfloat162float(((const __nv_bfloat16*)ix.cent_rt)[x]);
    return ((const float*)ix.cent_rt)[x];
}

__device__ __forceinline__ bool rank_before(double s, int g, double s2, int g2)
{
    return s > s2 || (s == s2 && g < g2);  // score descending, then lowest bucket id
}

__device__ __forceinline__ uint32_t ord_key(float f)
{
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float key_to_float(uint32_t k)
{
    const uint32_t u = (k & 0x80000000u) ? (k & 0x7fffffffu) : ~k;
    return __uint_as_float(u);
}

template <typename T>
__device__ __forceinline__ void load_query(float* q_s, const T* lq, int64_t row)
{
    if (threadIdx.x < DL) q_s[threadIdx.x] = load_elt(lq + row * DL + threadIdx.x);
}

// ---------------------------------------------------------------------------
// Helpers of the SIMT nominator (fp32 indices, decode, small chunks) and of
// the D-LSA Tree walk: approximate scores, exact scores, radix top-KC.
// ---------------------------------------------------------------------------
constexpr int SIMT_THREADS = 256;
constexpr int64_t SIMT_SMEM_MAX = 220 * 1024;

// Approximate (binary32) scores of buckets [0, nb) into sc.  Each lane reads
// 16 bytes of a centroid row, so a warp covers several rows per load
// (128-byte bf16 rows: 8 lanes per row; 256-byte fp32 rows: 16 lanes per
// row) and the partial sums are reduced across the row's lanes.  The order of
// the fp32 sum is irrelevant here: these scores only nominate candidates.
__device__ void approx_scores(const IndexView& ix, const float* q_s, int64_t bseq, int64_t nb,
                              float* sc)
{
    // Each warp handles a contiguous range of rows; the loads of UNR
    // iterations are issued before any of them is consumed, so a warp keeps
    // UNR * 512 bytes in flight instead of waiting on one load at a time.
    constexpr int UNR = 8;
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
    if (ix.dtype == LSA_BF16) {
        constexpr int LPR = 8, RPI = 32 / LPR;  // lanes per row, rows per iteration
        const int sub = lane % LPR, rsel = lane / LPR;
        float q[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) q[e] = q_s[sub * 8 + e];
        const uint4* base = reinterpret_cast<const uint4*>(
            (const __nv_bfloat16*)ix.cent_rt + bseq * ix.NBK * DL);
        for (int64_t g0 = (int64_t)warp * RPI * UNR; g0 < nb; g0 += (int64_t)nwarps * RPI * UNR) {
            uint4 raw[UNR];
#pragma unroll
            for (int u = 0; u < UNR; ++u) {
                const int64_t g = g0 + u * RPI + rsel;
                raw[u] = (g < nb) ? __ldg(base + g * (DL / 8) + sub) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int u = 0; u < UNR; ++u) {
                const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw[u]);
                float acc = 0.f;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 f = __bfloat1622float2(h[e]);
                    acc = fmaf(q[2 * e], f.x, acc);
                    acc = fmaf(q[2 * e + 1], f.y, acc);
                }
#pragma unroll
                for (int o = LPR / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
                const int64_t g = g0 + u * RPI + rsel;
                if (sub == 0 && g < nb) sc[g] = acc;
            }
        }
    } else {
        constexpr int LPR = 16, RPI = 32 / LPR;
        const int sub = lane % LPR, rsel = lane / LPR;
        float q[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) q[e] = q_s[sub * 4 + e];
        const float4* base =
            reinterpret_cast<const float4*>((const float*)ix.cent_rt + bseq * ix.NBK * DL);
        for (int64_t g0 = (int64_t)warp * RPI * UNR; g0 < nb; g0 += (int64_t)nwarps * RPI * UNR) {
            float4 f[UNR];
#pragma unroll
            for (int u = 0; u < UNR; ++u) {
                const int64_t g = g0 + u * RPI + rsel;
                f[u] = (g < nb) ? __ldg(base + g * (DL / 4) + sub) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int u = 0; u < UNR; ++u) {
                float acc = fmaf(q[0], f[u].x, 0.f);
                acc = fmaf(q[1], f[u].y, acc);
                acc = fmaf(q[2], f[u].z, acc);
                acc = fmaf(q[3], f[u].w, acc);
#pragma unroll
                for (int o = LPR / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
                const int64_t g = g0 + u * RPI + rsel;
                if (sub == 0 && g < nb) sc[g] = acc;
            }
        }
    }
    __syncthreads();
}

// Exact score of one bucket: the retrieval centroid's row is read with 16-byte
// loads (all in flight together), then summed in ascending dimension as exact
// binary64 products.
__device__ __forceinline__ double exact_score(const IndexView& ix, int64_t bseq, int64_t g,
                                              const float* q_s)
{
    double s = 0.0;
    if (ix.dtype == LSA_BF16) {
        const uint4* row = reinterpret_cast<const uint4*>((const __nv_bfloat16*)ix.cent_rt +
                                                          (bseq * ix.NBK + g) * DL);
        uint4 raw[DL / 8];
#pragma unroll
        for (int x = 0; x < DL / 8; ++x) raw[x] = __ldg(row + x);
#pragma unroll
        for (int x = 0; x < DL / 8; ++x) {
            const __nv_bfloat16* h = reinterpret_cast<const __nv_bfloat16*>(&raw[x]);
#pragma unroll
            for (int e = 0; e < 8; ++e)
                s = __fma_rn((double)q_s[x * 8 + e], (double)__bfloat162float(h[e]), s);
        }
    } else {
        const float4* row =
            reinterpret_cast<const float4*>((const float*)ix.cent_rt + (bseq * ix.NBK + g) * DL);
        float4 f[DL / 4];
#pragma unroll
        for (int x = 0; x < DL / 4; ++x) f[x] = __ldg(row + x);
#pragma unroll
        for (int x = 0; x < DL / 4; ++x) {
            s = __fma_rn((double)q_s[4 * x + 0], (double)f[x].x, s);
            s = __fma_rn((double)q_s[4 * x + 1], (double)f[x].y, s);
            s = __fma_rn((double)q_s[4 * x + 2], (double)f[x].z, s);
            s = __fma_rn((double)q_s[4 * x + 3], (double)f[x].w, s);
        }
    }
    return s;
}

// The KC largest of the nb > KC approximate scores sc[0 .. nb) (shared
// memory), by an MSB-first radix select of the KC-th largest (4 passes of 8
// bits over ordered keys): every bucket above that score plus enough of those
// equal to it, written to cand[0 .. KC) (any memory).  Returns tau = that
// score, which bounds every bucket left out.  Called by every thread of the
// CTA.
__device__ float radix_top_kc(const float* sc, int64_t nb, int32_t* cand)
{
    __shared__ unsigned hist[256];
    __shared__ uint32_t sh_prefix, sh_want;
    __shared__ int sh_gt, sh_eq;
    if (threadIdx.x == 0) {
        sh_prefix = 0;
        sh_want = KC;
        sh_gt = 0;
        sh_eq = 0;
    }
    __syncthreads();
    uint32_t mask = 0;
    for (int pass = 3; pass >= 0; --pass) {
        const int sh = 8 * pass;
        for (int x = threadIdx.x; x < 256; x += blockDim.x) hist[x] = 0;
        __syncthreads();
        const uint32_t prefix = sh_prefix;
        // warp-aggregated counts: scores share their leading bytes, so one
        // atomic per distinct bin of a warp instead of one per score
        const int64_t nb_up = (nb + 31) & ~(int64_t)31;
        for (int64_t g = threadIdx.x; g < nb_up; g += blockDim.x) {
            uint32_t bin = 0xFFFFFFFFu;
            if (g < nb) {
                const uint32_t kk = ord_key(sc[g]);
                if ((kk & mask) == prefix) bin = (kk >> sh) & 255u;
            }
            const unsigned same = __match_any_sync(0xffffffffu, bin);
            if (bin != 0xFFFFFFFFu && (threadIdx.x & 31) == __ffs(same) - 1)
                atomicAdd(&hist[bin], (unsigned)__popc(same));
        }
        __syncthreads();
        if (threadIdx.x < 32) {
            // warp 0 finds the bin holding the want-th largest key: lane l owns
            // bins 255-8l .. 248-8l (high to low); an exclusive scan of the lane
            // totals gives each lane the count above its bins.
            const int l = threadIdx.x;
            uint32_t hb[8], tot = 0;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                hb[e] = hist[255 - 8 * l - e];
                tot += hb[e];
            }
            uint32_t incl = tot;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
                if (l >= o) incl += y;
            }
            const uint32_t want = sh_want;
            uint32_t cum = incl - tot;
            const bool mine = cum < want && incl >= want;
            if (mine) {
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    if (cum + hb[e] >= want) {
                        sh_prefix = prefix | ((uint32_t)(255 - 8 * l - e) << sh);
                        sh_want = want - cum;
                        break;
                    }
                    cum += hb[e];
                }
            }
        }
        mask |= 255u << sh;
        __syncthreads();
    }
    const uint32_t thr = sh_prefix;      // key of the KC-th largest score
    const int need_eq = (int)sh_want;    // how many of the ties at thr to take
    for (int64_t g = threadIdx.x; g < nb; g += blockDim.x) {
        const uint32_t kk = ord_key(sc[g]);
        if (kk > thr) {
            const int s = atomicAdd(&sh_gt, 1);
            cand[s] = (int32_t)g;
        } else if (kk == thr) {
            const int s = atomicAdd(&sh_eq, 1);
            if (s < need_eq) cand[KC - need_eq + s] = (int32_t)g;
        }
    }
    __syncthreads();
    return key_to_float(thr);
}

// Body of the SIMT nominator for query `row` at position pq; q_s holds the
// latent query (every thread of the CTA calls it; sc holds n_blk*k floats).
__device__ void simt_nominate(const IndexView& ix, int64_t n_blk, const float* q_s, int64_t bseq,
                              int64_t row, int64_t pq, int W, const SelectWs& ws, float* sc)
{
    const int64_t nb = eligible_buckets(ix, n_blk, pq, W);
    int32_t* cand = ws.lst_g + row * KC;      // one list of KC per row
    if (nb <= KC) {
        for (int x = threadIdx.x; x < KC; x += blockDim.x) cand[x] = (x < nb) ? x : -1;
        if (threadIdx.x == 0) {
            ws.lst_n[row] = (int32_t)nb;
            ws.lst_tau[row] = -INFINITY;
        }
        return;
    }
    approx_scores(ix, q_s, bseq, nb, sc);
    __syncthreads();
    const float tau = radix_top_kc(sc, nb, cand);
    if (threadIdx.x == 0) {
        ws.lst_n[row] = KC;
        ws.lst_tau[row] = tau;
    }
}

// ---------------------------------------------------------------------------
// Candidate nomination, SIMT: one CTA per query.  Binary32 FMA scores of the
// eligible buckets into shared memory, then an MSB-first radix select of the
// KC-th largest score (4 passes of 8 bits).  Candidates: every bucket above
// that score plus enough of those equal to it.  tau = that score.
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(SIMT_THREADS) score_topk_simt_kernel(IndexView ix, int64_t n_blk,
                                                                       const T* lq, PosSrc pos,
                                                                       int64_t Nq, int W,
                                                                       SelectWs ws)
{
    extern __shared__ float sc[];
    __shared__ float q_s[DL];
    const int64_t b = blockIdx.y, i = blockIdx.x;
    const int64_t row = b * Nq + i;
    if (row == 0 && threadIdx.x == 0) *ws.fb_count = 0;
    for (int64_t x = row * blockDim.x + threadIdx.x; x < ws.plan.n_zero;
         x += (int64_t)Nq * gridDim.y * blockDim.x)
        ws.plan.zero[x] = 0;
    load_query(q_s, lq, row);
    __syncthreads();
    simt_nominate(ix, n_blk, q_s, b, row, pos.at(b, Nq, i), W, ws, sc);
}

// ---------------------------------------------------------------------------
// Availability and emission helpers (closed CSR members, then open members).
// ---------------------------------------------------------------------------
struct FillCtx {
    IndexView ix;
    int64_t bseq;
    int64_t n_blk;
    int64_t pos;
    int64_t hi;     // pos - W
    int64_t S;
    bool open_live; // the open block has keys at or below hi
    // the open block's assigned groups in ascending order (shared memory):
    // slot ol_o[x] of the open block belongs to bucket ol_g[x]
    const int32_t* ol_o;
    const int32_t* ol_g;
    int ol_n;
};

// Compacts sequence bseq's open list into (slot, bucket) pairs in ascending
// slot order; returns the count.  Called by every thread of the CTA (blockDim
// a multiple of 32, at most 1024); cnt_s holds one int per warp.
__device__ int build_open_list(const IndexView& ix, int64_t bseq, int32_t* ol_o, int32_t* ol_g,
                               int* cnt_s)
{
    const int32_t* open = ix.open_bucket + bseq * ix.G;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    constexpr int U = 8;   // loads in flight per thread
    int base = 0;
    for (int x00 = 0; x00 < ix.G; x00 += U * (int)blockDim.x) {
        int32_t gv[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int x = x00 + u * (int)blockDim.x + (int)threadIdx.x;
            gv[u] = (x < ix.G) ? open[x] : -1;
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            if (x00 + u * (int)blockDim.x >= ix.G) break;   // uniform over the CTA
            const int x = x00 + u * (int)blockDim.x + (int)threadIdx.x;
            const int32_t g = gv[u];
            const unsigned bal = __ballot_sync(0xffffffffu, g >= 0);
            if (lane == 0) cnt_s[warp] = __popc(bal);
            __syncthreads();
            int before = base;
            for (int w = 0; w < warp; ++w) before += cnt_s[w];
            if (g >= 0) {
                const int at = before + __popc(bal & ((1u << lane) - 1u));
                ol_o[at] = x;
                ol_g[at] = g;
            }
            for (int w = 0; w < nw; ++w) base += cnt_s[w];
            __syncthreads();
        }
    }
    return base;
}

// True when bucket g has a member in the open block.
__device__ __forceinline__ bool has_open(const FillCtx& f, int64_t g)
{
    for (int x = 0; x < f.ol_n; ++x)
        if (f.ol_g[x] == g) return true;
    return false;
}

// Warp-cooperative count of available keys of bucket g (closed members plus
// open-block members); *closed_out, when given, receives the closed part.
__device__ int64_t warp_avail(const FillCtx& f, int64_t g, int64_t* closed_out = nullptr)
{
    const int lane = threadIdx.x & 31;
    const IndexView& ix = f.ix;
    const int32_t* off = ix.offsets + f.bseq * (ix.NBK + 1);
    const int32_t* mem = ix.members + f.bseq * ix.NP;
    const int p = ix.p;
    const int64_t span = (int64_t)p * ix.G;
    const int64_t blk = g / ix.k;
    const int64_t bstart = blk * span, bend = bstart + span;
    const int32_t o0 = off[g], o1 = off[g + 1];
    int64_t a = 0;
    if (bstart >= f.S && bend - 1 <= f.hi) {
        a = (int64_t)(o1 - o0) * p;
    } else if (bstart <= f.hi) {
        int64_t c = 0;
        for (int32_t x = o0 + lane; x < o1; x += 32) c += group_avail(mem[x], p, f.S, f.hi);
        for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
        a = c;
    }
    if (closed_out) *closed_out = a;
    if (f.open_live) {
        const int64_t j0 = f.n_blk * ix.G;
        int64_t c = 0;
        for (int x = lane; x < f.ol_n; x += 32)
            if (f.ol_g[x] == g) c += group_avail(j0 + f.ol_o[x], p, f.S, f.hi);
        for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
        a += c;
    }
    return a;
}

// Closed keys of bucket g below the first sink-free position S: they open the
// bucket's ascending key list (only block 0 can hold any).
__device__ int64_t keys_below_sinks(const FillCtx& f, int64_t g)
{
    const IndexView& ix = f.ix;
    const int p = ix.p;
    const int64_t span = (int64_t)p * ix.G;
    if ((g / ix.k) * span >= f.S) return 0;
    const int32_t* off = ix.offsets + f.bseq * (ix.NBK + 1);
    const int32_t* mem = ix.members + f.bseq * ix.NP;
    int64_t n = 0;
    for (int32_t x = off[g]; x < off[g + 1]; ++x) {
        const int64_t lo = (int64_t)mem[x] * p;
        if (lo >= f.S) break;
        n += (f.S - lo < p) ? f.S - lo : p;
    }
    return n;
}

// Lists a row for bucket-major attention: reserves nt + 1 partial slots and
// records every taken bucket as the range [lo, hi) of its closed key list
// plus the count of open-block keys taken after it.  Rows that find no room
// become gather rows.  Called by every thread of the fill CTA.
__device__ void plan_list_row(const BucketPlan& P, int64_t row, int64_t bseq, int64_t NBK, int nt,
                              const int* take_g, const int64_t* take_n, const int64_t* take_lo,
                              const int64_t* take_closed, int* sh_base)
{
    if (threadIdx.x == 0) {
        int base = atomicAdd(P.ctr + CTR_RESERVED, nt + 1);
        if ((int64_t)base + nt + 1 > P.ent_cap) {
            base = -1;
            P.gather_rows[atomicAdd(P.ctr + CTR_GATHER, 1)] = (int32_t)row;
        } else {
            atomicMax(P.ctr + CTR_VALID_END, base + nt + 1);
            P.ent[base + nt] = make_int4((int)row, -1, 0, 0);   // sinks + window slot
        }
        P.row_n[row] = (base < 0) ? -1 : nt;
        P.row_base[row] = base;
        *sh_base = base;
    }
    __syncthreads();
    const int base = *sh_base;
    if (base < 0) return;
    for (int t = threadIdx.x; t < nt; t += blockDim.x) {
        const int64_t gg = bseq * NBK + take_g[t];
        const int64_t closed = (take_n[t] < take_closed[t]) ? take_n[t] : take_closed[t];
        const int rank = atomicAdd(P.bucket_cnt + gg, 1);
        P.ent[base + t] = make_int4((int)row, (int)gg, (int)take_lo[t], (int)(take_lo[t] + closed));
        P.ent2[base + t] = make_int2(rank, (int)(take_n[t] - closed));
    }
}

__device__ void warp_emit_partial(const FillCtx& f, int64_t g, int64_t take, int32_t* out);

// True when every key of bucket g's closed members is available and it has no
// available open member: the bucket's available keys are then its closed
// members expanded.
__device__ __forceinline__ bool bucket_full(const FillCtx& f, int64_t g)
{
    const int64_t span = (int64_t)f.ix.p * f.ix.G;
    const int64_t bstart = (g / f.ix.k) * span;
    return bstart >= f.S && bstart + span - 1 <= f.hi && !(f.open_live && has_open(f, g));
}

// Writes the first `take` available keys of bucket g (ascending) to out.
// Called by every thread of the CTA; uses warp 0 for partial buckets.
__device__ void cta_emit(const FillCtx& f, int64_t g, int64_t take, int32_t* out)
{
    const IndexView& ix = f.ix;
    const int32_t* off = ix.offsets + f.bseq * (ix.NBK + 1);
    const int32_t* mem = ix.members + f.bseq * ix.NP;
    const int p = ix.p;
    const int64_t span = (int64_t)p * ix.G;
    const int64_t blk = g / ix.k;
    const int64_t bstart = blk * span, bend = bstart + span;
    const int32_t o0 = off[g];
    const bool full = (bstart >= f.S && bend - 1 <= f.hi) && !(f.open_live && has_open(f, g));
    if (full) {
        for (int64_t x = threadIdx.x; x < take; x += blockDim.x)
            out[x] = mem[o0 + x / p] * p + (int32_t)(x % p);
        return;
    }
    if (threadIdx.x >= 32) return;
    warp_emit_partial(f, g, take, out);
}

// Warp-cooperative emission of the first `take` available keys of bucket g
// (closed members, then open-block members), in ascending position.
__device__ void warp_emit_partial(const FillCtx& f, int64_t g, int64_t take, int32_t* out)
{
    const IndexView& ix = f.ix;
    const int32_t* off = ix.offsets + f.bseq * (ix.NBK + 1);
    const int32_t* mem = ix.members + f.bseq * ix.NP;
    const int p = ix.p;
    const int32_t o0 = off[g], o1 = off[g + 1];
    const int lane = threadIdx.x & 31;
    int64_t cur = 0;
    const int64_t nkeys = (int64_t)(o1 - o0) * p;
    for (int64_t x0 = 0; x0 < nkeys && cur < take; x0 += 32) {
        const int64_t x = x0 + lane;
        int64_t t = -1;
        if (x < nkeys) t = (int64_t)mem[o0 + x / p] * p + x % p;
        const bool ok = (t >= f.S) && (t <= f.hi);
        const unsigned bal = __ballot_sync(0xffffffffu, ok);
        const int64_t at = cur + __popc(bal & ((1u << lane) - 1u));
        if (ok && at < take) out[at] = (int32_t)t;
        cur += __popc(bal);
    }
    if (f.open_live) {
        // the bucket's open groups in ascending order; each contributes the
        // contiguous run of its keys inside [S, hi]
        const int64_t j0 = f.n_blk * ix.G;
        for (int x0 = 0; x0 < f.ol_n && cur < take; x0 += 32) {
            const int x = x0 + lane;
            int na = 0;
            int64_t lo = 0;
            if (x < f.ol_n && f.ol_g[x] == g) {
                const int64_t jj = j0 + f.ol_o[x];
                na = group_avail(jj, p, f.S, f.hi);
                lo = (jj * p > f.S) ? jj * p : f.S;
            }
            int incl = na;
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            const int64_t at0 = cur + incl - na;
            for (int r = 0; r < na; ++r)
                if (at0 + r < take) out[at0 + r] = (int32_t)(lo + r);
            cur += __shfl_sync(0xffffffffu, incl, 31);
        }
    }
}

__device__ void cta_emit_tail(int64_t pq, int W, int64_t n_s, int64_t off, int s_max, int32_t* out,
                              int32_t* count)
{
    int64_t w0 = pq - W + 1;
    if (w0 < n_s) w0 = n_s;
    const int64_t n_w = pq + 1 - w0;
    for (int64_t x = threadIdx.x; x < n_w; x += blockDim.x) out[off + x] = (int32_t)(w0 + x);
    for (int64_t x = off + n_w + threadIdx.x; x < s_max; x += blockDim.x) out[x] = -1;
    if (threadIdx.x == 0) *count = (int32_t)(off + n_w);
}

constexpr int FILL_THREADS = 128;
static_assert(FILL_THREADS == KCF, "one candidate per fill thread");

// ---------------------------------------------------------------------------
// Exact ranking + greedy fill + emission.  One CTA (128 threads) per query.
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(FILL_THREADS) select_fill_kernel(IndexView ix, int64_t n_blk,
                                                                   const T* lq, PosSrc pos,
                                                                   int64_t Nq, int R, int W, int S,
                                                                   int s_max, int32_t* indices,
                                                                   int32_t* counts, SelectWs ws)
{
    extern __shared__ int32_t open_sm[];   // [2][G] when the open block exists
    __shared__ float q_s[DL];
    __shared__ int cg[KCF];
    __shared__ double es[KCF];
    __shared__ int order[KCF];
    __shared__ int64_t av[KCF];
    __shared__ int64_t avc[KCF];          // closed part of av
    __shared__ int take_g[KCF];
    __shared__ int64_t take_n[KCF];
    __shared__ int64_t take_closed[KCF];  // its available closed keys
    __shared__ int64_t take_lo[KCF];      // its closed keys below the sinks bound
    __shared__ int64_t take_off[KCF];     // output offset of each taken bucket
    __shared__ int32_t take_o0[KCF];      // its first CSR position
    __shared__ int take_full[KCF];
    __shared__ int sh_ntake, sh_exact, sh_nc, sh_complete;
    __shared__ float sh_l1, sh_tau;
    __shared__ int lst_off[FILL_THREADS + 1];
    __shared__ float lst_tau_s[FILL_THREADS];
    const int64_t b = blockIdx.y, i = blockIdx.x;
    const int64_t row = b * Nq + i;
    const int64_t pq = pos.at(b, Nq, i);
    if (ws.app_n > 0 && i == 0 && threadIdx.x < 32) {
        // decode: the best of the sliced nearest-centroid searches (highest
        // exact score, lowest bucket on ties) joins the open block.  The group
        // lies inside this query's window, so the selection below never reads
        // it; the barriers before any open-list read order it anyway.
        const int o = ws.app_slot[b];
        if (o >= 0) {
            double bs = -INFINITY;
            int bg = 0x7fffffff;
            for (int x = threadIdx.x; x < ws.app_n; x += 32) {
                const double sx = ws.app_score[b * ws.app_n + x];
                const int gx = ws.app_g[b * ws.app_n + x];
                if (sx > bs || (sx == bs && gx < bg)) {
                    bs = sx;
                    bg = gx;
                }
            }
            for (int off = 16; off > 0; off >>= 1) {
                const double os = __shfl_xor_sync(0xffffffffu, bs, off);
                const int og = __shfl_xor_sync(0xffffffffu, bg, off);
                if (os > bs || (os == bs && og < bg)) {
                    bs = os;
                    bg = og;
                }
            }
            if (threadIdx.x == 0 && bg != 0x7fffffff) ix.open_bucket[b * ix.G + o] = bg;
        }
    }
    load_query(q_s, lq, row);
    // The row's candidate lists (n_lst <= FILL_THREADS): counts and bounds in
    // parallel, their offsets by one thread, then the bucket ids.  tau bounds
    // every eligible bucket left out of the lists; with every list complete
    // there is none.
    {
        const int nl = ws.n_lst;
        if ((int)threadIdx.x < nl) {
            lst_off[threadIdx.x + 1] = ws.lst_n[row * nl + threadIdx.x];
            lst_tau_s[threadIdx.x] = ws.lst_tau[row * nl + threadIdx.x];
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            int tot = 0, comp = 1;
            float tmax = -INFINITY;
            lst_off[0] = 0;
            for (int l = 0; l < nl; ++l) {
                tot += lst_off[l + 1];
                lst_off[l + 1] = tot;
                const float t = lst_tau_s[l];
                if (t > -INFINITY) comp = 0;
                tmax = fmaxf(tmax, t);
            }
            sh_nc = tot;
            sh_tau = tmax;
            sh_complete = comp;
        }
        __syncthreads();
        const int tot = sh_nc;
        if (tot > KCF) {
            // more candidates than the fill ranks: the exact fallback takes the row
            if (threadIdx.x == 0) {
                const int slot = atomicAdd(ws.fb_count, 1);
                ws.fb_list[slot] = (int32_t)row;
                atomicAdd(ix.status + 1, 1u);
                if (ws.plan.row_n) {
                    ws.plan.row_n[row] = -1;
                    ws.plan.row_base[row] = -1;
                    ws.plan.gather_rows[atomicAdd(ws.plan.ctr + CTR_GATHER, 1)] = (int32_t)row;
                }
            }
            return;
        }
        if ((int)threadIdx.x < tot) {
            int l = 0;
            while (lst_off[l + 1] <= (int)threadIdx.x) ++l;
            cg[threadIdx.x] =
                ws.lst_g[(row * nl + l) * ws.lst_cap + ((int)threadIdx.x - lst_off[l])];
        }
    }
    const int nc = sh_nc;
    const float tau = sh_tau;
    __syncthreads();
    if (threadIdx.x == 0) {
        float l1 = 0.f;
        for (int d = 0; d < DL; ++d) l1 += fabsf(q_s[d]);
        sh_l1 = l1;
    }
    if ((int)threadIdx.x < nc) es[threadIdx.x] = exact_score(ix, b, cg[threadIdx.x], q_s);
    __syncthreads();
    if ((int)threadIdx.x < nc) {
        const int c = threadIdx.x;
        int r = 0;
        for (int c2 = 0; c2 < nc; ++c2) r += rank_before(es[c2], cg[c2], es[c], cg[c]);
        order[r] = c;
    }
    FillCtx f;
    f.ix = ix;
    f.bseq = b;
    f.n_blk = n_blk;
    f.pos = pq;
    f.hi = pq - W;
    f.S = S;
    f.open_live = (n_blk * ix.G < ix.NP) && (n_blk > 0) && (n_blk * (int64_t)ix.p * ix.G <= f.hi);
    f.ol_n = 0;
    f.ol_o = open_sm;
    f.ol_g = open_sm + ix.G;
    if (f.open_live) {
        __shared__ int cnt_w[FILL_THREADS / 32];
        f.ol_n = build_open_list(ix, b, open_sm, open_sm + ix.G, cnt_w);
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __shared__ int slow[KCF];
    __shared__ int n_slow;
    if (threadIdx.x == 0) n_slow = 0;
    __syncthreads();
    if ((int)threadIdx.x < nc) {
        // buckets whose keys are all available: count = p * members, one
        // round trip for every candidate at once
        const int c = threadIdx.x;
        const int g = cg[c];
        if (bucket_full(f, g)) {
            const int32_t* off = ix.offsets + b * (ix.NBK + 1);
            av[c] = (int64_t)(off[g + 1] - off[g]) * ix.p;
            avc[c] = av[c];
        } else {
            slow[atomicAdd(&n_slow, 1)] = c;
        }
    }
    __syncthreads();
    for (int e = warp; e < n_slow; e += FILL_THREADS / 32) {
        const int c = slow[e];
        int64_t closed;
        const int64_t a = warp_avail(f, cg[c], &closed);
        if (lane == 0) {
            av[c] = a;
            avc[c] = closed;
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int64_t rem = R;
        int nt = 0, cut = -1;
        for (int r = 0; r < nc && rem > 0; ++r) {
            const int c = order[r];
            const int64_t a = av[c];
            if (a == 0) continue;
            const int64_t t = (a <= rem) ? a : rem;
            take_g[nt] = cg[c];
            take_n[nt] = t;
            take_closed[nt] = avc[c];
            take_off[nt] = (int64_t)R - rem;
            ++nt;
            rem -= t;
            if (rem == 0) cut = c;
        }
        int exact = 1;
        if (!sh_complete) {
            const double eps = ldexp((double)sh_l1, -12);
            if (rem > 0) {
                int64_t total = f.hi - S + 1;  // keys in [S, pos - W]
                if (total < 0) total = 0;
                exact = ((int64_t)R - rem) >= total;
            } else if (cut >= 0) {
                exact = es[cut] > (double)tau + eps;
            }
        }
        sh_ntake = nt;
        sh_exact = exact;
    }
    __syncthreads();
    if (!sh_exact) {
        if (threadIdx.x == 0) {
            const int slot = atomicAdd(ws.fb_count, 1);
            ws.fb_list[slot] = (int32_t)row;
            atomicAdd(ix.status + 1, 1u);
            if (ws.plan.row_n) {   // the fallback's selection is attended key by key
                ws.plan.row_n[row] = -1;
                ws.plan.row_base[row] = -1;
                ws.plan.gather_rows[atomicAdd(ws.plan.ctr + CTR_GATHER, 1)] = (int32_t)row;
            }
        }
        return;
    }
    int32_t* out = indices + row * (int64_t)s_max;
    const int64_t n_s = (S < pq + 1) ? S : pq + 1;
    for (int64_t x = threadIdx.x; x < n_s; x += FILL_THREADS) out[x] = (int32_t)x;
    const int nt = sh_ntake;
    const int32_t* offs = ix.offsets + b * (ix.NBK + 1);
    const int32_t* mem = ix.members + b * ix.NP;
    for (int t = threadIdx.x; t < nt; t += FILL_THREADS) {
        take_full[t] = bucket_full(f, take_g[t]) ? 1 : 0;
        take_o0[t] = offs[take_g[t]];
        take_lo[t] = take_full[t] ? 0 : keys_below_sinks(f, take_g[t]);
    }
    __syncthreads();
    if (ws.plan.row_n) {
        __shared__ int sh_base;
        plan_list_row(ws.plan, row, b, ix.NBK, nt, take_g, take_n, take_lo, take_closed, &sh_base);
    }
    const int64_t n_lr = nt ? take_off[nt - 1] + take_n[nt - 1] : 0;
    // Whole-member buckets: every long-range slot independently (a binary
    // search finds its bucket), so all member reads are in flight at once.
    const int p = ix.p;
    constexpr int EU = 8;   // slots per thread per batch: EU member loads in flight
    for (int64_t x0 = threadIdx.x; x0 < n_lr; x0 += (int64_t)FILL_THREADS * EU) {
        int64_t src[EU];
        int rem_[EU];
#pragma unroll
        for (int u = 0; u < EU; ++u) {
            const int64_t x = x0 + (int64_t)u * FILL_THREADS;
            src[u] = -1;
            rem_[u] = 0;
            if (x < n_lr) {
                int lo = 0, hi = nt - 1;
                while (lo < hi) {
                    const int mid = (lo + hi + 1) >> 1;
                    if (take_off[mid] <= x) lo = mid;
                    else hi = mid - 1;
                }
                if (take_full[lo]) {
                    const int64_t rel = x - take_off[lo];
                    src[u] = take_o0[lo] + rel / p;
                    rem_[u] = (int)(rel % p);
                }
            }
        }
        int32_t m[EU];
#pragma unroll
        for (int u = 0; u < EU; ++u) m[u] = (src[u] >= 0) ? __ldg(mem + src[u]) : 0;
#pragma unroll
        for (int u = 0; u < EU; ++u)
            if (src[u] >= 0) out[n_s + x0 + (int64_t)u * FILL_THREADS] = m[u] * p + rem_[u];
    }
    // Buckets cut by the window or the sinks, or with open members: one warp each.
    for (int t = warp; t < nt; t += FILL_THREADS / 32)
        if (!take_full[t]) warp_emit_partial(f, take_g[t], take_n[t], out + n_s + take_off[t]);
    __syncthreads();
    cta_emit_tail(pq, W, n_s, n_s + n_lr, s_max, out, counts + row);
}

// ---------------------------------------------------------------------------
// Exact ranking + greedy fill + emission, one warp per query row: the same
// steps and results as select_fill_kernel, for launches with many rows (a
// prefill chunk).  Each warp works alone -- no barrier spans the CTA -- so an
// SM keeps several times more rows in flight, and every serial step of the
// CTA kernel becomes a warp-wide scan: the greedy fill is a prefix sum of the
// ranked candidates' available keys, and whole buckets are emitted member by
// member (p keys per member load).
// ---------------------------------------------------------------------------
constexpr int FW_WARPS = 4;            // query rows per CTA
constexpr int64_t FW_MIN_ROWS = 64;    // fewer rows: a CTA per row (shorter latency per row)
constexpr int FW_DSMEM_MAX = 192 * 1024;   // dynamic shared memory (open lists) it may use
constexpr int FW_LISTS = 32;           // candidate lists per row this kernel takes
constexpr int FW_PL = KCF / 32;        // candidates per lane

struct FwRow {
    float q[DL];
    double es[KCF];
    int cg[KCF];
    int av[KCF];          // available keys of candidate c
    int avc[KCF];         // its closed part
    int order[KCF];       // candidate at rank r
    int t_g[KCF];         // taken bucket t: id
    int t_n[KCF];         //   keys taken
    int t_off[KCF];       //   first long-range slot
    int t_o0[KCF];        //   first CSR position
    int t_closed[KCF];    //   available closed keys
    int t_lo[KCF];        //   closed keys below the sinks bound
    int t_full[KCF];      //   every closed key available, no open member
    int t_mc[KCF + 1];    //   members of the whole buckets before it (prefix)
    int lst_off[FW_LISTS];
};

template <typename T>
__global__ void __launch_bounds__(32 * FW_WARPS) select_fill_warp_kernel(
    IndexView ix, int64_t n_blk, const T* lq, PosSrc pos, int64_t Nq, int R, int W, int S,
    int s_max, int32_t* indices, int32_t* counts, SelectWs ws)
{
    extern __shared__ int32_t fw_open[];   // [FW_WARPS][2][G] when the open block may hold keys
    __shared__ FwRow fw[FW_WARPS];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * FW_WARPS + warp;
    if (row >= ix.B * Nq) return;          // warp-uniform; no barrier spans the CTA
    const unsigned FULL = 0xffffffffu;
    FwRow& F = fw[warp];
    const int64_t b = row / Nq, i = row % Nq;
    const int64_t pq = pos.at(b, Nq, i);
    F.q[lane] = load_elt(lq + row * DL + lane);
    F.q[lane + 32] = load_elt(lq + row * DL + lane + 32);

    // ---- the row's candidate lists ----
    const int nl = ws.n_lst;               // <= FW_LISTS (checked at launch)
    int ln = 0;
    float lt = -INFINITY;
    if (lane < nl) {
        ln = ws.lst_n[row * nl + lane];
        lt = ws.lst_tau[row * nl + lane];
    }
    int incl = ln;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(FULL, incl, o);
        if (lane >= o) incl += y;
    }
    const int tot = __shfl_sync(FULL, incl, 31);
    if (lane < nl) F.lst_off[lane] = incl - ln;
    float tau = lt;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) tau = fmaxf(tau, __shfl_xor_sync(FULL, tau, o));
    const bool complete = !(tau > -INFINITY);   // every list holds all of its range
    auto to_fallback = [&]() {
        if (lane == 0) {
            const int slot = atomicAdd(ws.fb_count, 1);
            ws.fb_list[slot] = (int32_t)row;
            atomicAdd(ix.status + 1, 1u);
            if (ws.plan.row_n) {   // the fallback's selection is attended key by key
                ws.plan.row_n[row] = -1;
                ws.plan.row_base[row] = -1;
                ws.plan.gather_rows[atomicAdd(ws.plan.ctr + CTR_GATHER, 1)] = (int32_t)row;
            }
        }
    };
    if (tot > KCF) {                       // more candidates than the fill ranks
        to_fallback();
        return;
    }
    __syncwarp();
#pragma unroll
    for (int u = 0; u < FW_PL; ++u) {
        const int c = lane + 32 * u;
        if (c < tot) {
            int l = 0;
            while (l + 1 < nl && F.lst_off[l + 1] <= c) ++l;
            F.cg[c] = ws.lst_g[(row * nl + l) * ws.lst_cap + (c - F.lst_off[l])];
        }
    }
    __syncwarp();

    // ---- exact scores and ranking ----
    float l1 = fabsf(F.q[lane]) + fabsf(F.q[lane + 32]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) l1 += __shfl_xor_sync(FULL, l1, o);
#pragma unroll
    for (int u = 0; u < FW_PL; ++u) {
        const int c = lane + 32 * u;
        if (c < tot) F.es[c] = exact_score(ix, b, F.cg[c], F.q);
    }
    __syncwarp();
#pragma unroll
    for (int u = 0; u < FW_PL; ++u) {
        const int c = lane + 32 * u;
        if (c < tot) {
            const double e = F.es[c];
            const int g = F.cg[c];
            int r = 0;
            for (int c2 = 0; c2 < tot; ++c2) r += rank_before(F.es[c2], F.cg[c2], e, g);
            F.order[r] = c;
        }
    }

    // ---- availability of every candidate ----
    FillCtx f;
    f.ix = ix;
    f.bseq = b;
    f.n_blk = n_blk;
    f.pos = pq;
    f.hi = pq - W;
    f.S = S;
    f.open_live = (n_blk * ix.G < ix.NP) && (n_blk > 0) && (n_blk * (int64_t)ix.p * ix.G <= f.hi);
    f.ol_n = 0;
    int32_t* ol_o = fw_open + (size_t)warp * 2 * ix.G;
    int32_t* ol_g = ol_o + ix.G;
    f.ol_o = ol_o;
    f.ol_g = ol_g;
    if (f.open_live) {
        // the open block's assigned groups in ascending slot order
        const int32_t* open = ix.open_bucket + b * ix.G;
        int n = 0;
        for (int x0 = 0; x0 < ix.G; x0 += 32) {
            const int x = x0 + lane;
            const int32_t g = (x < ix.G) ? open[x] : -1;
            const unsigned bal = __ballot_sync(FULL, g >= 0);
            if (g >= 0) {
                const int at = n + __popc(bal & ((1u << lane) - 1u));
                ol_o[at] = x;
                ol_g[at] = g;
            }
            n += __popc(bal);
        }
        f.ol_n = n;
    }
    __syncwarp();
    const int32_t* offs = ix.offsets + b * (ix.NBK + 1);
    const int32_t* mem = ix.members + b * ix.NP;
    const int p = ix.p;
    unsigned slow_u = 0;                   // bit u: candidate lane + 32u needs a member scan
#pragma unroll
    for (int u = 0; u < FW_PL; ++u) {
        const int c = lane + 32 * u;
        if (c < tot) {
            const int g = F.cg[c];
            if (bucket_full(f, g)) {
                F.av[c] = (offs[g + 1] - offs[g]) * p;
                F.avc[c] = F.av[c];
            } else {
                slow_u |= 1u << u;
            }
        }
    }
    for (int u = 0; u < FW_PL; ++u) {
        unsigned bal = __ballot_sync(FULL, (slow_u >> u) & 1u);
        while (bal) {
            const int src = __ffs(bal) - 1;
            bal &= bal - 1u;
            const int c = src + 32 * u;
            int64_t closed;
            const int64_t a = warp_avail(f, F.cg[c], &closed);
            if (lane == 0) {
                F.av[c] = (int)a;
                F.avc[c] = (int)closed;
            }
        }
    }
    __syncwarp();

    // ---- greedy fill: a prefix sum over the ranked candidates ----
    // lane holds ranks FW_PL*lane .. FW_PL*lane + FW_PL - 1
    int rc[FW_PL], ra[FW_PL], pre[FW_PL];
    int lsum = 0;
#pragma unroll
    for (int u = 0; u < FW_PL; ++u) {
        const int r = FW_PL * lane + u;
        rc[u] = (r < tot) ? F.order[r] : -1;
        ra[u] = (rc[u] >= 0) ? F.av[rc[u]] : 0;
        pre[u] = lsum;
        lsum += ra[u];
    }
    int sc = lsum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(FULL, sc, o);
        if (lane >= o) sc += y;
    }
    const int total_av = __shfl_sync(FULL, sc, 31);
    const int lbase = sc - lsum;           // keys available before this lane's ranks
    // taken: available keys and fewer than R keys before it
    int n_take = 0;
    int cut_c = -1;
#pragma unroll
    for (int u = 0; u < FW_PL; ++u) {
        const int A = lbase + pre[u];
        if (ra[u] > 0 && A < R) {
            ++n_take;
            if (A + ra[u] >= R) cut_c = rc[u];
        }
    }
    int tinc = n_take;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(FULL, tinc, o);
        if (lane >= o) tinc += y;
    }
    const int nt = __shfl_sync(FULL, tinc, 31);
    int t = tinc - n_take;
#pragma unroll
    for (int u = 0; u < FW_PL; ++u) {
        const int A = lbase + pre[u];
        if (ra[u] > 0 && A < R) {
            const int c = rc[u];
            const int g = F.cg[c];
            const int full = bucket_full(f, g) ? 1 : 0;
            F.t_g[t] = g;
            F.t_n[t] = min(ra[u], R - A);
            F.t_off[t] = A;
            F.t_o0[t] = offs[g];
            F.t_closed[t] = F.avc[c];
            F.t_full[t] = full;
            F.t_lo[t] = full ? 0 : (int)keys_below_sinks(f, g);
            ++t;
        }
    }
    // the cut candidate (rank at which the budget is met), if any
    const unsigned cb = __ballot_sync(FULL, cut_c >= 0);
    cut_c = cb ? __shfl_sync(FULL, cut_c, __ffs(cb) - 1) : -1;
    bool exact = true;
    if (!complete) {
        const double eps = ldexp((double)l1, -12);
        if (total_av < R) {
            int64_t total = f.hi - S + 1;      // keys in [S, pos - W]
            if (total < 0) total = 0;
            exact = (int64_t)total_av >= total;
        } else if (cut_c >= 0) {
            exact = F.es[cut_c] > (double)tau + eps;
        }
    }
    if (!exact) {
        to_fallback();
        return;
    }
    __syncwarp();

    int32_t* out = indices + row * (int64_t)s_max;
    const int64_t n_s = (S < pq + 1) ? S : pq + 1;
    for (int64_t x = lane; x < n_s; x += 32) out[x] = (int32_t)x;
    // bucket-major attention lists of the row
    if (ws.plan.row_n) {
        const BucketPlan& P = ws.plan;
        int base = 0;
        if (lane == 0) {
            base = atomicAdd(P.ctr + CTR_RESERVED, nt + 1);
            if ((int64_t)base + nt + 1 > P.ent_cap) {
                base = -1;
                P.gather_rows[atomicAdd(P.ctr + CTR_GATHER, 1)] = (int32_t)row;
            } else {
                atomicMax(P.ctr + CTR_VALID_END, base + nt + 1);
                P.ent[base + nt] = make_int4((int)row, -1, 0, 0);   // sinks + window slot
            }
            P.row_n[row] = (base < 0) ? -1 : nt;
            P.row_base[row] = base;
        }
        base = __shfl_sync(FULL, base, 0);
        if (base >= 0) {
            for (int tt = lane; tt < nt; tt += 32) {
                const int64_t gg = b * ix.NBK + F.t_g[tt];
                const int closed = min(F.t_n[tt], F.t_closed[tt]);
                const int rank = atomicAdd(P.bucket_cnt + gg, 1);
                P.ent[base + tt] =
                    make_int4((int)row, (int)gg, F.t_lo[tt], F.t_lo[tt] + closed);
                P.ent2[base + tt] = make_int2(rank, F.t_n[tt] - closed);
            }
        }
    }
    // whole buckets, member by member: prefix of their member counts
    if (lane == 0) {
        int acc = 0;
        for (int tt = 0; tt < nt; ++tt) {
            F.t_mc[tt] = acc;
            if (F.t_full[tt]) acc += (F.t_n[tt] + p - 1) / p;
        }
        F.t_mc[nt] = acc;
    }
    __syncwarp();
    const int n_mem = F.t_mc[nt];
    int32_t* lr = out + n_s;
    constexpr int EU = 4;                  // member loads in flight per lane
    for (int m0 = lane; m0 < n_mem; m0 += 32 * EU) {
        int tk[EU], mi[EU];
        int32_t mv[EU];
#pragma unroll
        for (int e = 0; e < EU; ++e) {
            const int m = m0 + 32 * e;
            tk[e] = -1;
            if (m < n_mem) {
                int lo = 0, hi = nt - 1;   // last bucket with t_mc <= m among whole ones
                while (lo < hi) {
                    const int mid = (lo + hi + 1) >> 1;
                    if (F.t_mc[mid] <= m) lo = mid;
                    else hi = mid - 1;
                }
                while (lo + 1 < nt && (!F.t_full[lo] || F.t_mc[lo + 1] <= m)) ++lo;
                tk[e] = lo;
                mi[e] = m - F.t_mc[lo];
            }
        }
#pragma unroll
        for (int e = 0; e < EU; ++e) mv[e] = (tk[e] >= 0) ? __ldg(mem + F.t_o0[tk[e]] + mi[e]) : 0;
#pragma unroll
        for (int e = 0; e < EU; ++e) {
            if (tk[e] < 0) continue;
            const int tt = tk[e];
            const int k0 = mi[e] * p;
            int32_t* dst = lr + F.t_off[tt];
            const int nk = min(p, F.t_n[tt] - k0);
            for (int q = 0; q < nk; ++q) dst[k0 + q] = mv[e] * p + q;
        }
    }
    // buckets cut by the window or the sinks, or with open members
    for (int tt = 0; tt < nt; ++tt)
        if (!F.t_full[tt]) warp_emit_partial(f, F.t_g[tt], F.t_n[tt], lr + F.t_off[tt]);
    // recent window, padding, count
    const int64_t n_lr = nt ? (int64_t)F.t_off[nt - 1] + F.t_n[nt - 1] : 0;
    const int64_t off = n_s + n_lr;
    int64_t w0 = pq - W + 1;
    if (w0 < n_s) w0 = n_s;
    const int64_t n_w = pq + 1 - w0;
    for (int64_t x = lane; x < n_w; x += 32) out[off + x] = (int32_t)(w0 + x);
    for (int64_t x = off + n_w + lane; x < s_max; x += 32) out[x] = -1;
    if (lane == 0) counts[row] = (int32_t)(off + n_w);
}

// ---------------------------------------------------------------------------
// Decode selection, one CTA of DF_THREADS per sequence (latency matters: a
// decode step has one query per sequence).  Candidates: the KC best of the
// union of the slices' sorted lists (rank by counting); tau = the larger of
// the union's next score and every slice's next unlisted score, which bounds
// every bucket left out.  Then the steps of select_fill_kernel: exact
// binary64 rescoring, ranking, availability, a prefix-sum greedy fill (one
// warp), emission of whole buckets member by member over the CTA, partial
// buckets by warps, recent window.
// ---------------------------------------------------------------------------
constexpr int DF_THREADS = 512;
constexpr int DF_UNION = DEC_MAX_SLICES * DEC_M;

template <typename T>
__global__ void __launch_bounds__(DF_THREADS) decode_fill_kernel(IndexView ix, int64_t n_blk,
                                                                 const T* lq, const int32_t* pos,
                                                                 int R, int W, int S, int s_max,
                                                                 int32_t* indices,
                                                                 int32_t* counts, SelectWs ws)
{
    extern __shared__ int32_t open_sm[];   // [2][G] when the open block exists
    __shared__ float q_s[DL];
    __shared__ float us[DF_UNION];
    __shared__ int ug[DF_UNION];
    __shared__ int cg[KC];
    __shared__ double es[KC];
    __shared__ int order[KC];
    __shared__ int av[KC], avc[KC];
    __shared__ int t_g[KC], t_n[KC], t_off[KC], t_o0[KC], t_full[KC], t_mc[KC + 1];
    __shared__ int c_o0[KC], c_full[KC];    // per candidate: first CSR position, all keys available
    __shared__ int sh_nc, sh_nt, sh_exact, sh_cmpl, sh_tot;
    __shared__ float sh_tau;
    __shared__ unsigned sh_slow;
    const unsigned FULL = 0xffffffffu;
    const int64_t b = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t pq = pos[b];
    if (pq < 0 || pq >= ix.T_cap) return;       // recorded by the prep pass
    // the best of the sliced nearest-centroid searches joins the open block
    if (ws.app_n > 0 && warp == 0) {
        const int o = ws.app_slot[b];
        if (o >= 0) {
            double bs = -INFINITY;
            int bg = 0x7fffffff;
            for (int x = lane; x < ws.app_n; x += 32) {
                const double sx = ws.app_score[b * ws.app_n + x];
                const int gx = ws.app_g[b * ws.app_n + x];
                if (sx > bs || (sx == bs && gx < bg)) {
                    bs = sx;
                    bg = gx;
                }
            }
            for (int off = 16; off > 0; off >>= 1) {
                const double os = __shfl_xor_sync(FULL, bs, off);
                const int og = __shfl_xor_sync(FULL, bg, off);
                if (os > bs || (os == bs && og < bg)) {
                    bs = os;
                    bg = og;
                }
            }
            if (lane == 0 && bg != 0x7fffffff) ix.open_bucket[b * ix.G + o] = bg;
        }
    }
    load_query(q_s, lq, b);
    // ---- the union of the slices' lists ----
    const int nsl = ws.n_slice;
    const int nu = nsl * DEC_M;
    for (int e = threadIdx.x; e < nu; e += DF_THREADS) {
        const int sl = e / DEC_M, r = e % DEC_M;
        const int64_t ls = b * nsl + sl;
        const bool ok = r < ws.dl_n[ls];
        us[e] = ok ? ws.dl_s[ls * DEC_M + r] : -INFINITY;
        ug[e] = ok ? ws.dl_g[ls * DEC_M + r] : -1;
    }
    if (warp == 0) {
        float tm = -INFINITY;
        int tot = 0;
        for (int sl = lane; sl < nsl; sl += 32) {
            tm = fmaxf(tm, ws.dl_tau[b * nsl + sl]);
            tot += ws.dl_n[b * nsl + sl];
        }
        for (int off = 16; off > 0; off >>= 1) {
            tm = fmaxf(tm, __shfl_xor_sync(FULL, tm, off));
            tot += __shfl_xor_sync(FULL, tot, off);
        }
        if (lane == 0) {
            sh_tau = tm;                 // every slice's next unlisted score
            sh_tot = tot;
            sh_nc = min(tot, KC);
            sh_cmpl = (tm == -INFINITY) && tot <= KC;
        }
    }
    __shared__ float sh_next;                 // the union's score after its KC best
    if (threadIdx.x == 0) sh_next = -INFINITY;
    __syncthreads();
    for (int e = threadIdx.x; e < nu; e += DF_THREADS) {
        const int g = ug[e];
        if (g < 0) continue;
        const float x = us[e];
        // every slice's list is sorted (score desc, bucket asc; unlisted
        // entries at the end): the entries ranking before (x, g) are a prefix,
        // found by binary search
        int rank = 0;
        for (int sl = 0; sl < nsl; ++sl) {
            const float* ys = us + sl * DEC_M;
            const int* gs = ug + sl * DEC_M;
            int lo = 0, hi = DEC_M;                 // first entry not before (x, g)
            while (lo < hi) {
                const int mid = (lo + hi) >> 1;
                const int g2 = gs[mid];
                const float y = ys[mid];
                const bool before = g2 >= 0 && ((y > x) || (y == x && g2 < g));
                if (before) lo = mid + 1;
                else hi = mid;
            }
            rank += lo;
        }
        if (rank < KC) cg[rank] = g;
        else if (rank == KC) sh_next = x;       // ranks are distinct: one writer
    }
    __syncthreads();
    if (threadIdx.x == 0) sh_tau = fmaxf(sh_tau, sh_next);
    __syncthreads();
    const int nc = sh_nc;
    const float tau = sh_tau;
    const bool complete = sh_cmpl != 0;
    float l1 = 0.f;
    // ---- exact scores, ranking, availability ----
    if ((int)threadIdx.x < nc) es[threadIdx.x] = exact_score(ix, b, cg[threadIdx.x], q_s);
    if (warp == 1) {
        float a = fabsf(q_s[lane]) + fabsf(q_s[lane + 32]);
        for (int off = 16; off > 0; off >>= 1) a += __shfl_xor_sync(FULL, a, off);
        if (lane == 0) sh_exact = __float_as_int(a);    // |q|_1, handed on below
    }
    __syncthreads();
    l1 = __int_as_float(sh_exact);
    if ((int)threadIdx.x < nc) {
        const int c = threadIdx.x;
        int r = 0;
        for (int c2 = 0; c2 < nc; ++c2) r += rank_before(es[c2], cg[c2], es[c], cg[c]);
        order[r] = c;
    }
    FillCtx f;
    f.ix = ix;
    f.bseq = b;
    f.n_blk = n_blk;
    f.pos = pq;
    f.hi = pq - W;
    f.S = S;
    f.open_live = (n_blk * ix.G < ix.NP) && (n_blk > 0) && (n_blk * (int64_t)ix.p * ix.G <= f.hi);
    f.ol_n = 0;
    f.ol_o = open_sm;
    f.ol_g = open_sm + ix.G;
    if (f.open_live) {
        __shared__ int cnt_w[DF_THREADS / 32];
        f.ol_n = build_open_list(ix, b, open_sm, open_sm + ix.G, cnt_w);
    }
    if (threadIdx.x == 0) sh_slow = 0u;
    __syncthreads();
    const int32_t* offs = ix.offsets + b * (ix.NBK + 1);
    const int32_t* mem = ix.members + b * ix.NP;
    const int p = ix.p;
    if ((int)threadIdx.x < nc) {
        const int c = threadIdx.x;
        const int g = cg[c];
        const int o0 = offs[g];
        c_o0[c] = o0;
        if (bucket_full(f, g)) {
            c_full[c] = 1;
            av[c] = (offs[g + 1] - o0) * p;
            avc[c] = av[c];
        } else {
            c_full[c] = 0;
            atomicOr(&sh_slow, 1u << (c & 31));     // marks a group of candidates
            av[c] = -1;
        }
    }
    __syncthreads();
    if (sh_slow) {
        // buckets cut by the window or the sinks, or with open members: a warp each
        for (int c = warp; c < nc; c += DF_THREADS / 32) {
            if (av[c] >= 0) continue;                 // uniform over the warp
            int64_t closed;
            const int64_t a = warp_avail(f, cg[c], &closed);
            if (lane == 0) {
                av[c] = (int)a;
                avc[c] = (int)closed;
            }
        }
        __syncthreads();
    }
    // ---- greedy fill: warp 0, a prefix sum over the ranked candidates ----
    if (warp == 0) {
        constexpr int PL = KC / 32;
        int rc[PL], ra[PL], pre[PL];
        int lsum = 0;
#pragma unroll
        for (int u = 0; u < PL; ++u) {
            const int r = PL * lane + u;
            rc[u] = (r < nc) ? order[r] : -1;
            ra[u] = (rc[u] >= 0) ? av[rc[u]] : 0;
            pre[u] = lsum;
            lsum += ra[u];
        }
        int sc = lsum;
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(FULL, sc, o);
            if (lane >= o) sc += y;
        }
        const int total_av = __shfl_sync(FULL, sc, 31);
        const int lbase = sc - lsum;
        int n_take = 0, cut_c = -1;
#pragma unroll
        for (int u = 0; u < PL; ++u) {
            const int A = lbase + pre[u];
            if (ra[u] > 0 && A < R) {
                ++n_take;
                if (A + ra[u] >= R) cut_c = rc[u];
            }
        }
        int tinc = n_take;
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(FULL, tinc, o);
            if (lane >= o) tinc += y;
        }
        const int nt = __shfl_sync(FULL, tinc, 31);
        int t = tinc - n_take;
#pragma unroll
        for (int u = 0; u < PL; ++u) {
            const int A = lbase + pre[u];
            if (ra[u] > 0 && A < R) {
                const int c = rc[u];
                const int g = cg[c];
                t_g[t] = g;
                t_n[t] = min(ra[u], R - A);
                t_off[t] = A;
                t_o0[t] = c_o0[c];
                t_full[t] = c_full[c];
                ++t;
            }
        }
        const unsigned cb = __ballot_sync(FULL, cut_c >= 0);
        cut_c = cb ? __shfl_sync(FULL, cut_c, __ffs(cb) - 1) : -1;
        bool exact = true;
        if (!complete) {
            const double eps = ldexp((double)l1, -12);
            if (total_av < R) {
                int64_t total = f.hi - S + 1;      // keys in [S, pos - W]
                if (total < 0) total = 0;
                exact = (int64_t)total_av >= total;
            } else if (cut_c >= 0) {
                exact = es[cut_c] > (double)tau + eps;
            }
        }
        __syncwarp();
        if (lane == 0) {
            sh_nt = nt;
            sh_exact = exact ? 1 : 0;
            int acc = 0;                               // members of whole buckets before t
            for (int tt = 0; tt < nt; ++tt) {
                t_mc[tt] = acc;
                if (t_full[tt]) acc += (t_n[tt] + p - 1) / p;
            }
            t_mc[nt] = acc;
            if (!exact) {
                const int slot = atomicAdd(ws.fb_count, 1);
                ws.fb_list[slot] = (int32_t)b;
                atomicAdd(ix.status + 1, 1u);
            }
        }
    }
    __syncthreads();
    if (!sh_exact) return;
    // ---- emission ----
    const int nt = sh_nt;
    int32_t* out = indices + b * (int64_t)s_max;
    const int64_t n_s = (S < pq + 1) ? S : pq + 1;
    for (int64_t x = threadIdx.x; x < n_s; x += DF_THREADS) out[x] = (int32_t)x;
    int32_t* lr = out + n_s;
    const int n_mem = t_mc[nt];
    for (int m = threadIdx.x; m < n_mem; m += DF_THREADS) {
        int lo = 0, hi = nt - 1;                       // last bucket with t_mc <= m
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (t_mc[mid] <= m) lo = mid;
            else hi = mid - 1;
        }
        while (lo + 1 < nt && (!t_full[lo] || t_mc[lo + 1] <= m)) ++lo;
        const int mi = m - t_mc[lo];
        const int32_t mv = __ldg(mem + t_o0[lo] + mi);
        const int k0 = mi * p;
        const int nk = min(p, t_n[lo] - k0);
        for (int q = 0; q < nk; ++q) lr[t_off[lo] + k0 + q] = mv * p + q;
    }
    for (int tt = warp; tt < nt; tt += DF_THREADS / 32)
        if (!t_full[tt]) warp_emit_partial(f, t_g[tt], t_n[tt], lr + t_off[tt]);
    const int64_t n_lr = nt ? (int64_t)t_off[nt - 1] + t_n[nt - 1] : 0;
    cta_emit_tail(pq, W, n_s, n_s + n_lr, s_max, out, counts + b);
}

// ---------------------------------------------------------------------------
// D-LSA Tree nomination, one CTA (TREE_THREADS) per query ("Prefrontal's
// Latent Sparse Attention ...", section "What it changes": the query scores a
// few clusters at each level and walks down).  1. exact binary64 scores of
// every super-centroid (retrieval copy), the `branches` best (score desc,
// lowest id on ties) -- kept per row for the exact fallback; 2. the chosen
// branches' eligible buckets (the universe) with binary32 approximate scores;
// 3. the KC largest of them (radix select) are the row's candidate list, tau
// bounds the rest of the universe (all of it listed: tau = -inf).  A universe
// larger than the shared-memory area gets an empty list with tau = +inf, so
// that the fill sends the row to the fallback.  select_fill_kernel then ranks
// the candidates exactly and fills the budget as Flat does.
// ---------------------------------------------------------------------------
constexpr int TREE_MAX_BR = 256;     // branches walked at most
constexpr int TREE_THREADS = 256;

template <typename T>
__global__ void __launch_bounds__(TREE_THREADS) tree_nominate_kernel(
    IndexView ix, int64_t n_blk, const T* lq, PosSrc pos, int64_t Nq, int W, SelectWs ws,
    const T* sup_rt, int64_t NS, int branches, int u_cap)
{
    extern __shared__ unsigned char tsm[];
    double* es2 = reinterpret_cast<double*>(tsm);               // [NS]
    int32_t* uid = reinterpret_cast<int32_t*>(es2 + NS);        // [u_cap]
    float* usc = reinterpret_cast<float*>(uid + u_cap);         // [u_cap]
    __shared__ float q_s[DL];
    __shared__ int chosen[TREE_MAX_BR];
    __shared__ int n_u;
    __shared__ int cand_s[KC];
    const int64_t b = blockIdx.y, i = blockIdx.x;
    const int64_t row = b * Nq + i;
    const int64_t pq = pos.at(b, Nq, i);
    if (row == 0 && threadIdx.x == 0) *ws.fb_count = 0;
    if (threadIdx.x == 0) n_u = 0;
    load_query(q_s, lq, row);
    __syncthreads();
    // 1. super-centroids, exact (binary64, ascending dimension; 16-byte loads)
    for (int64_t h = threadIdx.x; h < NS; h += TREE_THREADS) {
        double acc = 0.0;
        if (ix.dtype == LSA_BF16) {
            const uint4* r4 = reinterpret_cast<const uint4*>(sup_rt + (b * NS + h) * DL);
#pragma unroll 2
            for (int x = 0; x < DL / 8; ++x) {
                const uint4 raw = __ldg(r4 + x);
                const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 f = __bfloat1622float2(h2[e]);
                    acc = __fma_rn((double)q_s[8 * x + 2 * e], (double)f.x, acc);
                    acc = __fma_rn((double)q_s[8 * x + 2 * e + 1], (double)f.y, acc);
                }
            }
        } else {
            const float4* r4 = reinterpret_cast<const float4*>(sup_rt + (b * NS + h) * DL);
#pragma unroll 2
            for (int x = 0; x < DL / 4; ++x) {
                const float4 f = __ldg(r4 + x);
                acc = __fma_rn((double)q_s[4 * x], (double)f.x, acc);
                acc = __fma_rn((double)q_s[4 * x + 1], (double)f.y, acc);
                acc = __fma_rn((double)q_s[4 * x + 2], (double)f.z, acc);
                acc = __fma_rn((double)q_s[4 * x + 3], (double)f.w, acc);
            }
        }
        es2[h] = acc;
    }
    __syncthreads();
    const int nbr = (int)min((int64_t)branches, NS);
    for (int64_t h = threadIdx.x; h < NS; h += TREE_THREADS) {
        const double e = es2[h];
        int r = 0;                             // rank, counted only while it can be < nbr
        for (int64_t h2 = 0; h2 < NS && r < nbr; ++h2) r += rank_before(es2[h2], (int)h2, e, (int)h);
        if (r < nbr) {
            chosen[r] = (int)h;
            ws.tree_br[row * ws.tree_nbr + r] = (int32_t)h;
        }
    }
    for (int r = nbr + (int)threadIdx.x; r < ws.tree_nbr; r += TREE_THREADS)
        ws.tree_br[row * ws.tree_nbr + r] = -1;
    __syncthreads();
    // 2. the universe: eligible buckets of the chosen branches
    const int64_t nb = eligible_buckets(ix, n_blk, pq, W);
    const int32_t* toff = ws.tree_off + b * (NS + 1);
    const int32_t* tmem = ws.tree_mem + b * ix.NBK;
    // (one shared atomic per warp and chunk: ballot of the eligible members)
    const int lane = threadIdx.x & 31;
    for (int r = 0; r < nbr; ++r) {
        const int h = chosen[r];
        const int32_t x0 = toff[h], x1 = toff[h + 1];
        for (int32_t xb = x0; xb < x1; xb += TREE_THREADS) {
            const int32_t x = xb + threadIdx.x;
            const int32_t g = (x < x1) ? tmem[x] : INT_MAX;
            const bool take = g < nb;
            const unsigned bal = __ballot_sync(0xffffffffu, take);
            int base = 0;
            if (lane == 0 && bal) base = atomicAdd(&n_u, __popc(bal));
            base = __shfl_sync(0xffffffffu, base, 0);
            const int slot = base + __popc(bal & ((1u << lane) - 1u));
            if (take && slot < u_cap) uid[slot] = g;
        }
    }
    __syncthreads();
    const int nu = n_u;
    int32_t* cand = ws.lst_g + row * KC;
    if (nu > u_cap) {                          // too large to rank here: the fallback takes it
        if (threadIdx.x == 0) {
            ws.lst_n[row] = 0;
            ws.lst_tau[row] = INFINITY;
        }
        return;
    }
    if (nu <= KC) {
        for (int x = threadIdx.x; x < KC; x += TREE_THREADS) cand[x] = (x < nu) ? uid[x] : -1;
        if (threadIdx.x == 0) {
            ws.lst_n[row] = nu;
            ws.lst_tau[row] = -INFINITY;
        }
        return;
    }
    // 3. approximate scores of the universe, then its KC best
    for (int u = threadIdx.x; u < nu; u += TREE_THREADS) {
        const int64_t g = uid[u];
        float acc = 0.f;
        if (ix.dtype == LSA_BF16) {
            const uint4* r4 = reinterpret_cast<const uint4*>((const __nv_bfloat16*)ix.cent_rt +
                                                             (b * ix.NBK + g) * DL);
            uint4 raw[DL / 8];
#pragma unroll
            for (int x = 0; x < DL / 8; ++x) raw[x] = __ldg(r4 + x);
#pragma unroll
            for (int x = 0; x < DL / 8; ++x) {
                const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw[x]);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 f = __bfloat1622float2(h2[e]);
                    acc = fmaf(q_s[8 * x + 2 * e], f.x, acc);
                    acc = fmaf(q_s[8 * x + 2 * e + 1], f.y, acc);
                }
            }
        } else {
            const float4* r4 = reinterpret_cast<const float4*>((const float*)ix.cent_rt +
                                                               (b * ix.NBK + g) * DL);
            float4 f[DL / 4];
#pragma unroll
            for (int x = 0; x < DL / 4; ++x) f[x] = __ldg(r4 + x);
#pragma unroll
            for (int x = 0; x < DL / 4; ++x) {
                acc = fmaf(q_s[4 * x], f[x].x, acc);
                acc = fmaf(q_s[4 * x + 1], f[x].y, acc);
                acc = fmaf(q_s[4 * x + 2], f[x].z, acc);
                acc = fmaf(q_s[4 * x + 3], f[x].w, acc);
            }
        }
        usc[u] = acc;
    }
    __syncthreads();
    const float tau = radix_top_kc(usc, nu, cand_s);
    for (int x = threadIdx.x; x < KC; x += TREE_THREADS) cand[x] = uid[cand_s[x]];
    if (threadIdx.x == 0) {
        ws.lst_n[row] = KC;
        ws.lst_tau[row] = tau;
    }
}

// ---------------------------------------------------------------------------
// Exact fallback: persistent CTAs walk the list of flagged queries.  Every
// eligible bucket gets its exact binary64 score; the fill repeatedly takes the
// best remaining bucket (score desc, lowest id) until the budget is met.
// ---------------------------------------------------------------------------
constexpr int FB_THREADS = 256;

template <typename T>
__global__ void __launch_bounds__(FB_THREADS) select_fallback_kernel(IndexView ix, int64_t n_blk,
                                                                     const T* lq, PosSrc pos,
                                                                     int64_t Nq, int R, int W,
                                                                     int S, int s_max,
                                                                     int32_t* indices,
                                                                     int32_t* counts, SelectWs ws)
{
    extern __shared__ int32_t open_sm[];   // [2][G] when the open block exists
    __shared__ int cnt_w[FB_THREADS / 32];
    __shared__ float q_s[DL];
    __shared__ double rs[FB_THREADS / 32];
    __shared__ int64_t rg[FB_THREADS / 32];
    __shared__ int64_t sh_best;
    __shared__ int64_t sh_avail;
    const int n = *ws.fb_count;
    double* sc = ws.fb_scores + (int64_t)blockIdx.x * ix.NBK;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int e = blockIdx.x; e < n; e += gridDim.x) {
        const int64_t row = ws.fb_list[e];
        const int64_t b = row / Nq, i = row % Nq;
        const int64_t pq = pos.at(b, Nq, i);
        const int64_t nb = eligible_buckets(ix, n_blk, pq, W);
        __syncthreads();
        load_query(q_s, lq, row);
        __syncthreads();
        if (!ws.tree_br) {
            for (int64_t g = threadIdx.x; g < nb; g += FB_THREADS) sc[g] = exact_score(ix, b, g, q_s);
        } else {
            // D-LSA Tree: only the buckets of the row's chosen branches compete
            for (int64_t g = threadIdx.x; g < nb; g += FB_THREADS) sc[g] = -INFINITY;
            __syncthreads();
            const int32_t* toff = ws.tree_off + b * (ws.tree_ns + 1);
            const int32_t* tmem = ws.tree_mem + b * ix.NBK;
            for (int r = 0; r < ws.tree_nbr; ++r) {
                const int h = ws.tree_br[row * ws.tree_nbr + r];
                if (h < 0) continue;
                for (int32_t x = toff[h] + threadIdx.x; x < toff[h + 1]; x += FB_THREADS) {
                    const int32_t g = tmem[x];
                    if (g < nb) sc[g] = exact_score(ix, b, g, q_s);
                }
            }
        }
        FillCtx f;
        f.ix = ix;
        f.bseq = b;
        f.n_blk = n_blk;
        f.pos = pq;
        f.hi = pq - W;
        f.S = S;
        f.open_live = (n_blk * ix.G < ix.NP) && (n_blk > 0) && (n_blk * (int64_t)ix.p * ix.G <= f.hi);
        f.ol_n = 0;
        f.ol_o = open_sm;
        f.ol_g = open_sm + ix.G;
        if (f.open_live) f.ol_n = build_open_list(ix, b, open_sm, open_sm + ix.G, cnt_w);
        int32_t* out = indices + row * (int64_t)s_max;
        const int64_t n_s = (S < pq + 1) ? S : pq + 1;
        for (int64_t x = threadIdx.x; x < n_s; x += FB_THREADS) out[x] = (int32_t)x;
        int64_t o = n_s, rem = R;
        __syncthreads();
        while (rem > 0) {
            double bs = -INFINITY;
            int64_t bg = INT64_MAX;
            for (int64_t g = threadIdx.x; g < nb; g += FB_THREADS) {
                const double s = sc[g];
                if (s != -INFINITY && (bs == -INFINITY || s > bs || (s == bs && g < bg))) {
                    bs = s;
                    bg = g;
                }
            }
            for (int off = 16; off > 0; off >>= 1) {
                const double os = __shfl_xor_sync(0xffffffffu, bs, off);
                const int64_t og = __shfl_xor_sync(0xffffffffu, bg, off);
                if (os != -INFINITY && (bs == -INFINITY || os > bs || (os == bs && og < bg))) {
                    bs = os;
                    bg = og;
                }
            }
            if (lane == 0) {
                rs[warp] = bs;
                rg[warp] = bg;
            }
            __syncthreads();
            if (threadIdx.x == 0) {
                for (int w = 1; w < FB_THREADS / 32; ++w)
                    if (rs[w] != -INFINITY && (bs == -INFINITY || rs[w] > bs || (rs[w] == bs && rg[w] < bg))) {
                        bs = rs[w];
                        bg = rg[w];
                    }
                sh_best = (bs == -INFINITY) ? -1 : bg;
            }
            __syncthreads();
            const int64_t g = sh_best;
            if (g < 0) break;
            if (warp == 0) {
                const int64_t a = warp_avail(f, g);
                if (lane == 0) sh_avail = a;
            }
            __syncthreads();
            const int64_t a = sh_avail;
            if (a > 0) {
                const int64_t t = (a <= rem) ? a : rem;
                cta_emit(f, g, t, out + o);
                o += t;
                rem -= t;
            }
            if (threadIdx.x == 0) sc[g] = -INFINITY;
            __syncthreads();
        }
        cta_emit_tail(pq, W, n_s, o, s_max, out, counts + row);
    }
}

// ---------------------------------------------------------------------------
// Decode step, part 1.  grid (B, n_slice): CTA (b, s) scores slice s of
// sequence b's eligible buckets and, when b's new token completes a pooled
// group, searches slice s of the closed buckets for the group's nearest
// centroid.  The two are independent: a pooled group that completes at
// position pos holds keys >= pos - p + 1, which lie inside the recent window
// (W >= p - 1), so no selection made at pos can read them.
// Scores: binary32 FMA over the retrieval copy (16-byte loads, lanes over a
// row's dimensions), then the slice's DEC_M best scores sorted (score desc,
// lower bucket on ties) with their buckets, and the next score as the bound of
// everything the slice leaves out -- the lists decode_fill_kernel merges.
// Append: slice 0 writes the new latent/key/value rows at pos; every slice
// pools the completed group j = (pos+1)/p - 1 (binary32, left to right; the
// group's last row comes from the new latent row itself), normalises it
// (binary64 norm) and takes the closed bucket of largest exact <u, c_g> in its
// range (fp32 centroids, lowest g on ties); the fill takes the best of the
// slices.  A group beyond the open block records DEV_OPEN_FULL.
// ---------------------------------------------------------------------------
constexpr int DEC_THREADS = 256;

template <typename T>
__global__ void __launch_bounds__(DEC_THREADS) decode_prep_kernel(
    IndexView ix, int64_t n_blk, T* latK, T* Kc, T* Vc, const T* nlk, const T* nk, const T* nv,
    const T* lq, const int32_t* pos, int Hkv, int d, int W, SelectWs ws, double* app_score,
    int32_t* app_g, int32_t* app_slot, int n_slice, uint32_t* attn_counter, int counters_per_seq)
{
    __shared__ float q_s[DL];
    __shared__ float x_s[DL];
    __shared__ float sc[DEC_THREADS * 4];          // this slice's fp32 scores (<= 1024)
    __shared__ float tile[64 * (DL + 1)];          // exact search: 64 centroid rows
    __shared__ double nrm_s;
    __shared__ double rs[DEC_THREADS / 32];
    __shared__ int rg[DEC_THREADS / 32];
    const int64_t b = blockIdx.x;
    const int sl = blockIdx.y;
    const int64_t pq = pos[b];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (b == 0 && sl == 0 && threadIdx.x == 0) *ws.fb_count = 0;
    if (pq < 0 || pq >= ix.T_cap) {
        if (sl == 0 && threadIdx.x == 0) {
            dev_error(ix.status, DEV_BAD_INDEX, (uint32_t)b);
            app_slot[b] = -1;
        }
        return;
    }

    // ---------------- scores of this slice ----------------
    {
        const int64_t nb = eligible_buckets(ix, n_blk, pq, W);
        const int64_t per = (((ix.NBK + n_slice - 1) / n_slice) + 31) / 32 * 32;
        const int64_t g0 = sl * per;
        const int64_t g1 = (g0 + per < nb) ? g0 + per : nb;
        if (g0 < g1) {
            load_query(q_s, lq, b);
            __syncthreads();
            // 8 lanes per 128-byte bf16 row (16 lanes per fp32 row), rows of the
            // slice spread over the warps
            const int n = (int)(g1 - g0);
            if (ix.dtype == LSA_BF16) {
                constexpr int LPR = 8, RPI = 32 / LPR;
                const int sub = lane % LPR, rsel = lane / LPR;
                float q[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) q[e] = q_s[sub * 8 + e];
                const uint4* base = reinterpret_cast<const uint4*>(
                    (const __nv_bfloat16*)ix.cent_rt + (b * ix.NBK + g0) * DL);
                // eight rows' loads in flight per lane, then their dot products
                constexpr int RU = 8;
                constexpr int STEP = (DEC_THREADS / 32) * RPI;
                for (int r00 = warp * RPI; r00 < n; r00 += RU * STEP) {
                    uint4 raw[RU];
#pragma unroll
                    for (int u = 0; u < RU; ++u) {
                        const int r = r00 + u * STEP + rsel;
                        raw[u] = (r < n) ? __ldg(base + (int64_t)r * (DL / 8) + sub) : make_uint4(0, 0, 0, 0);
                    }
#pragma unroll
                    for (int u = 0; u < RU; ++u) {
                        const int r = r00 + u * STEP + rsel;
                        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw[u]);
                        float acc = 0.f;
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 f = __bfloat1622float2(h[e]);
                            acc = fmaf(q[2 * e], f.x, acc);
                            acc = fmaf(q[2 * e + 1], f.y, acc);
                        }
#pragma unroll
                        for (int o = LPR / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
                        if (sub == 0 && r < n) sc[r] = acc;
                    }
                }
            } else {
                constexpr int LPR = 16, RPI = 32 / LPR;
                const int sub = lane % LPR, rsel = lane / LPR;
                float q[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) q[e] = q_s[sub * 4 + e];
                const float4* base = reinterpret_cast<const float4*>(
                    (const float*)ix.cent_rt + (b * ix.NBK + g0) * DL);
                for (int r0 = warp * RPI; r0 < n; r0 += (DEC_THREADS / 32) * RPI) {
                    const int r = r0 + rsel;
                    const float4 f = (r < n) ? __ldg(base + (int64_t)r * (DL / 4) + sub) : make_float4(0.f, 0.f, 0.f, 0.f);
                    float acc = fmaf(q[0], f.x, 0.f);
                    acc = fmaf(q[1], f.y, acc);
                    acc = fmaf(q[2], f.z, acc);
                    acc = fmaf(q[3], f.w, acc);
#pragma unroll
                    for (int o = LPR / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
                    if (sub == 0 && r < n) sc[r] = acc;
                }
            }
            __syncthreads();
            // this slice's DEC_M best scores, sorted (ties to the lower
            // bucket), and the next one
            const int64_t ls = b * n_slice + sl;
            for (int t = threadIdx.x; t < n; t += DEC_THREADS) {
                const float x = sc[t];
                int rank = 0;
                for (int u = 0; u < n; ++u) {
                    const float y = sc[u];
                    rank += (y > x) || (y == x && u < t);
                }
                if (rank < DEC_M) {
                    ws.dl_s[ls * DEC_M + rank] = x;
                    ws.dl_g[ls * DEC_M + rank] = (int32_t)(g0 + t);
                } else if (rank == DEC_M) {
                    ws.dl_tau[ls] = x;
                }
            }
            if (threadIdx.x == 0) {
                ws.dl_n[ls] = min(n, DEC_M);
                if (n <= DEC_M) ws.dl_tau[ls] = -INFINITY;
            }
        } else if (threadIdx.x == 0) {
            ws.dl_n[b * n_slice + sl] = 0;
            ws.dl_tau[b * n_slice + sl] = -INFINITY;
        }
    }

    // ---------------- append ----------------
    if (sl == 0) {
        for (int x = threadIdx.x; x < counters_per_seq; x += blockDim.x)
            attn_counter[b * counters_per_seq + x] = 0u;
        T* lrow = latK + (b * ix.T_cap + pq) * DL;
        for (int x = threadIdx.x; x < DL; x += blockDim.x) lrow[x] = nlk[b * DL + x];
        const int64_t kvn = (int64_t)Hkv * d;
        T* krow = Kc + (b * ix.T_cap + pq) * kvn;
        T* vrow = Vc + (b * ix.T_cap + pq) * kvn;
        for (int64_t x = threadIdx.x; x < kvn; x += blockDim.x) {
            krow[x] = nk[b * kvn + x];
            vrow[x] = nv[b * kvn + x];
        }
    }
    const int p = ix.p;
    const int64_t j = (pq + 1) / p - 1;
    const int64_t o = j - n_blk * ix.G;
    if ((pq + 1) % p != 0) {
        if (sl == 0 && threadIdx.x == 0) app_slot[b] = -1;
        return;
    }
    if (n_blk < 1 || o < 0 || o >= ix.G || j >= ix.NP) {
        if (sl == 0 && threadIdx.x == 0) {
            dev_error(ix.status, DEV_OPEN_FULL, (uint32_t)b);
            app_slot[b] = -1;
        }
        return;
    }
    if (threadIdx.x < DL) {
        // rows j*p .. pos-1 from the cache, row pos from the new latent row
        const int i = threadIdx.x;
        const T* rows = latK + (b * ix.T_cap + j * p) * DL;
        float s = (p == 1) ? load_elt(nlk + b * DL + i) : load_elt(rows + i);
        for (int r = 1; r < p; ++r)
            s = __fadd_rn(s, load_elt((r == p - 1) ? nlk + b * DL + i : rows + (int64_t)r * DL + i));
        const float xv = __fdiv_rn(s, (float)p);
        x_s[i] = xv;
        if (sl == 0) ix.pooled[(b * ix.NP + j) * DL + i] = xv;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        double ss = 0.0;
        for (int i = 0; i < DL; ++i) ss = __fma_rn((double)x_s[i], (double)x_s[i], ss);
        nrm_s = __dsqrt_rn(ss);
    }
    __syncthreads();
    if (threadIdx.x < DL) {
        const int i = threadIdx.x;
        const float u = (nrm_s != 0.0) ? __double2float_rn(__ddiv_rn((double)x_s[i], nrm_s)) : 0.f;
        if (sl == 0) ix.unit[(b * ix.NP + j) * DL + i] = u;
        q_s[i] = u;   // reuse as the unit vector
    }
    __syncthreads();
    // Exact scores against this slice of the closed centroids: tiles of 64
    // rows staged with coalesced 16-byte loads (row pitch DL + 1 floats, so
    // that thread t reading row t hits its own bank); one thread per row sums
    // it in ascending dimension.
    const float* cent = ix.cent + b * ix.NBK * DL;
    const int64_t nbk = n_blk * ix.k;
    const int64_t per2 = (nbk + n_slice - 1) / n_slice;
    const int64_t c0 = sl * per2, c1 = (c0 + per2 < nbk) ? c0 + per2 : nbk;
    double bs = -INFINITY;
    int bg = 0x7fffffff;
    for (int64_t t0 = c0; t0 < c1; t0 += 64) {
        const int rows = (int)((c1 - t0) < 64 ? (c1 - t0) : 64);
        __syncthreads();
        const float4* src = reinterpret_cast<const float4*>(cent + t0 * DL);
        {
            // all of the tile's loads in flight (64 rows x 16 float4 over the CTA)
            constexpr int TU = (64 * (DL / 4) + DEC_THREADS - 1) / DEC_THREADS;
            float4 fv[TU];
#pragma unroll
            for (int u = 0; u < TU; ++u) {
                const int x = threadIdx.x + u * DEC_THREADS;
                if (x < rows * (DL / 4)) fv[u] = src[x];
            }
#pragma unroll
            for (int u = 0; u < TU; ++u) {
                const int x = threadIdx.x + u * DEC_THREADS;
                if (x < rows * (DL / 4)) {
                    const int r = x / (DL / 4), c = (x % (DL / 4)) * 4;
                    float* dst = tile + r * (DL + 1) + c;
                    dst[0] = fv[u].x;
                    dst[1] = fv[u].y;
                    dst[2] = fv[u].z;
                    dst[3] = fv[u].w;
                }
            }
        }
        __syncthreads();
        if ((int)threadIdx.x < rows) {
            const float* c = tile + threadIdx.x * (DL + 1);
            double s = 0.0;
#pragma unroll 16
            for (int i = 0; i < DL; ++i) s = __fma_rn((double)q_s[i], (double)c[i], s);
            const int g = (int)(t0 + threadIdx.x);
            if (s > bs || (s == bs && g < bg)) {
                bs = s;
                bg = g;
            }
        }
    }
    for (int off = 16; off > 0; off >>= 1) {
        const double os = __shfl_xor_sync(0xffffffffu, bs, off);
        const int og = __shfl_xor_sync(0xffffffffu, bg, off);
        if (os > bs || (os == bs && og < bg)) {
            bs = os;
            bg = og;
        }
    }
    if (lane == 0) {
        rs[warp] = bs;
        rg[warp] = bg;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < DEC_THREADS / 32; ++w)
            if (rs[w] > bs || (rs[w] == bs && rg[w] < bg)) {
                bs = rs[w];
                bg = rg[w];
            }
        app_score[b * n_slice + sl] = bs;
        app_g[b * n_slice + sl] = bg;
        if (sl == 0) app_slot[b] = (int32_t)o;
    }
}

cudaError_t launch_decode_prep(const IndexView& ix, int64_t n_blk, void* latent_K, void* K,
                               void* V, const void* new_latent_k, const void* new_k,
                               const void* new_v, const void* latent_q, const int32_t* pos,
                               int Hkv, int d, int W, const SelectWs& ws, double* app_score,
                               int32_t* app_g, int32_t* app_slot, int n_slice,
                               uint32_t* attn_counter, int counters_per_seq, cudaStream_t st)
{
    if (n_slice < 1 || (ix.NBK + n_slice - 1) / n_slice > DEC_THREADS * 4 - 31)
        return cudaErrorInvalidValue;   // a slice's scores must fit the shared buffer
    dim3 grid((unsigned)ix.B, (unsigned)n_slice);
    if (ix.dtype == LSA_BF16) {
        typedef __nv_bfloat16 T;
        decode_prep_kernel<T><<<grid, DEC_THREADS, 0, st>>>(
            ix, n_blk, (T*)latent_K, (T*)K, (T*)V, (const T*)new_latent_k, (const T*)new_k,
            (const T*)new_v, (const T*)latent_q, pos, Hkv, d, W, ws, app_score, app_g, app_slot,
            n_slice, attn_counter, counters_per_seq);
    } else {
        typedef float T;
        decode_prep_kernel<T><<<grid, DEC_THREADS, 0, st>>>(
            ix, n_blk, (T*)latent_K, (T*)K, (T*)V, (const T*)new_latent_k, (const T*)new_k,
            (const T*)new_v, (const T*)latent_q, pos, Hkv, d, W, ws, app_score, app_g, app_slot,
            n_slice, attn_counter, counters_per_seq);
    }
    note_launch();
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Workspace and launch.
// ---------------------------------------------------------------------------
static inline size_t al256(size_t x) { return (x + 255) & ~(size_t)255; }

bool select_uses_tc(const IndexView& ix, int64_t Nq)
{
    return ix.dtype == LSA_BF16 && Nq >= 128 && tc_scoring_available();
}

// Candidate lists per row: one per tensor-core split, or one of KC from the
// SIMT nominator.
static void list_shape(const IndexView& ix, int64_t Nq, int* n_lst, int* cap, bool one_list = false)
{
    if (!one_list && select_uses_tc(ix, Nq)) {
        *n_lst = tc_split_plan(ix, Nq, 0).n_split;
        *cap = TC_LIST_CAP;
    } else {
        *n_lst = 1;
        *cap = KC;
    }
}

// Group maxima per row of the tensor-core path (0 otherwise).
static int64_t n_grp_of(const IndexView& ix, int64_t Nq, bool one_list = false)
{
    return (!one_list && select_uses_tc(ix, Nq)) ? tc_split_plan(ix, Nq, 0).n_grp : 0;
}

// one_list: a single list of KC candidates per row (SIMT-style nominators:
// the tree's), whatever the tensor-core scorer would use.
static size_t ws_bytes_shape(const IndexView& ix, int64_t Nq, bool one_list)
{
    const size_t rows = (size_t)ix.B * (size_t)Nq;
    int nl, cap;
    list_shape(ix, Nq, &nl, &cap, one_list);
    const size_t ng = (size_t)n_grp_of(ix, Nq, one_list);
    size_t n = al256(rows * nl * cap * 4) + al256(rows * nl * 4) + al256(rows * nl * 4) +
               al256(rows * 4) + al256(4) + al256((size_t)FB_CTAS * (size_t)ix.NBK * 8);
    if (ng) n += al256(rows * ng * 2) + al256(rows * 4);
    return n;
}

size_t select_ws_bytes(const IndexView& ix, int64_t Nq) { return ws_bytes_shape(ix, Nq, false); }

static SelectWs carve_shape(void* ws, const IndexView& ix, int64_t Nq, bool one_list)
{
    const size_t rows = (size_t)ix.B * (size_t)Nq;
    int nl, cap;
    list_shape(ix, Nq, &nl, &cap, one_list);
    char* p = (char*)ws;
    SelectWs w;
    w.n_lst = nl;
    w.lst_cap = cap;
    w.lst_g = (int32_t*)p;
    p += al256(rows * nl * cap * 4);
    w.lst_n = (int32_t*)p;
    p += al256(rows * nl * 4);
    w.lst_tau = (float*)p;
    p += al256(rows * nl * 4);
    w.fb_list = (int32_t*)p;
    p += al256(rows * 4);
    w.fb_count = (int32_t*)p;
    p += al256(4);
    w.fb_scores = (double*)p;
    p += al256((size_t)FB_CTAS * (size_t)ix.NBK * 8);
    w.dl_s = nullptr;
    w.dl_g = nullptr;
    w.dl_n = nullptr;
    w.dl_tau = nullptr;
    w.n_slice = 0;
    w.tree_br = nullptr;
    w.tree_off = nullptr;
    w.tree_mem = nullptr;
    w.tree_nbr = 0;
    w.tree_ns = 0;
    w.n_grp = n_grp_of(ix, Nq, one_list);
    w.gmax = nullptr;
    w.theta = nullptr;
    if (w.n_grp) {
        w.gmax = (uint16_t*)p;
        p += al256(rows * (size_t)w.n_grp * 2);
        w.theta = (float*)p;
        p += al256(rows * 4);
    }
    w.plan = BucketPlan{};
    w.app_score = nullptr;
    w.app_g = nullptr;
    w.app_slot = nullptr;
    w.app_n = 0;
    return w;
}

SelectWs select_ws_carve(void* ws, const IndexView& ix, int64_t Nq)
{
    return carve_shape(ws, ix, Nq, false);
}

cudaError_t launch_score_lists_tc(const IndexView& ix, int64_t n_blk, const void* latent_Q,
                                  PosSrc pos, int64_t Nq, int W, const SelectWs& ws,
                                  cudaStream_t st);

template <typename T>
static cudaError_t launch_finish_t(const IndexView& ix, int64_t n_blk, const T* lq, PosSrc pos,
                                   int64_t Nq, lsa_select_params sp, int32_t* indices,
                                   int32_t* counts, int s_max, const SelectWs& ws, cudaStream_t st)
{
    dim3 grid((unsigned)Nq, (unsigned)ix.B);
    // the compacted open list, when the index has an open block
    const size_t osm = (n_blk > 0 && n_blk * ix.G < ix.NP) ? (size_t)ix.G * 2 * sizeof(int32_t) : 0;
    if (ws.n_lst < 1 || ws.n_lst > FILL_THREADS || ws.lst_cap < 1) return cudaErrorInvalidValue;
    const int64_t rows_all = ix.B * Nq;
    const size_t wsm = (size_t)FW_WARPS * osm;   // one open list per warp
    if (rows_all >= FW_MIN_ROWS && ws.n_lst <= FW_LISTS && wsm <= FW_DSMEM_MAX) {
        // many rows: a warp per row
        const void* kern = (const void*)select_fill_warp_kernel<T>;
        cudaError_t e = ensure_smem_attr(kern, FW_DSMEM_MAX);
        if (e != cudaSuccess) return e;
        select_fill_warp_kernel<T><<<(unsigned)((rows_all + FW_WARPS - 1) / FW_WARPS),
                                     32 * FW_WARPS, wsm, st>>>(ix, n_blk, lq, pos, Nq, sp.budget,
                                                               sp.window, sp.sinks, s_max,
                                                               indices, counts, ws);
    } else {
        select_fill_kernel<T><<<grid, FILL_THREADS, osm, st>>>(
            ix, n_blk, lq, pos, Nq, sp.budget, sp.window, sp.sinks, s_max, indices, counts, ws);
    }
    note_launch();
    const int64_t rows = ix.B * Nq;
    const unsigned fb_grid = (unsigned)(rows < FB_CTAS ? rows : FB_CTAS);
    select_fallback_kernel<T><<<fb_grid, FB_THREADS, osm, st>>>(ix, n_blk, lq, pos, Nq, sp.budget,
                                                                sp.window, sp.sinks, s_max,
                                                                indices, counts, ws);
    note_launch();
    return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_select_t(const IndexView& ix, int64_t n_blk, const T* lq, PosSrc pos,
                                   int64_t Nq, lsa_select_params sp, int32_t* indices,
                                   int32_t* counts, int s_max, const SelectWs& ws, bool use_tc,
                                   cudaStream_t st)
{
    dim3 grid((unsigned)Nq, (unsigned)ix.B);
    cudaError_t e;
    if (use_tc) {
        e = launch_score_lists_tc(ix, n_blk, lq, pos, Nq, sp.window, ws, st);
        if (e != cudaSuccess) return e;
    } else {
        const size_t smem = (size_t)n_blk * ix.k * sizeof(float);
        e = ensure_smem_attr((const void*)score_topk_simt_kernel<T>, (int)SIMT_SMEM_MAX);
        if (e != cudaSuccess) return e;
        score_topk_simt_kernel<T><<<grid, SIMT_THREADS, smem, st>>>(ix, n_blk, lq, pos, Nq,
                                                                    sp.window, ws);
        note_launch();
    }
    return launch_finish_t(ix, n_blk, lq, pos, Nq, sp, indices, counts, s_max, ws, st);
}

cudaError_t launch_select(const IndexView& ix, int64_t n_blk, const void* latent_Q, PosSrc pos,
                          int64_t Nq, lsa_select_params sp, int32_t* indices, int32_t* counts,
                          int s_max, const SelectWs& ws, bool use_tc, cudaStream_t st)
{
    if (Nq <= 0) return cudaSuccess;
    if (ix.dtype == LSA_BF16)
        return launch_select_t(ix, n_blk, (const __nv_bfloat16*)latent_Q, pos, Nq, sp, indices,
                               counts, s_max, ws, use_tc, st);
    return launch_select_t(ix, n_blk, (const float*)latent_Q, pos, Nq, sp, indices, counts, s_max,
                           ws, false, st);
}

template <typename T>
static cudaError_t launch_decode_finish_t(const IndexView& ix, int64_t n_blk, const T* lq,
                                          const int32_t* pos, lsa_select_params sp,
                                          int32_t* indices, int32_t* counts, int s_max,
                                          const SelectWs& ws, cudaStream_t st)
{
    if (ws.n_slice < 1 || ws.n_slice > DEC_MAX_SLICES || !ws.dl_s) return cudaErrorInvalidValue;
    const size_t osm = (n_blk > 0 && n_blk * ix.G < ix.NP) ? (size_t)ix.G * 2 * sizeof(int32_t) : 0;
    decode_fill_kernel<T><<<(unsigned)ix.B, DF_THREADS, osm, st>>>(
        ix, n_blk, lq, pos, sp.budget, sp.window, sp.sinks, s_max, indices, counts, ws);
    note_launch();
    const unsigned fb_grid = (unsigned)(ix.B < FB_CTAS ? ix.B : FB_CTAS);
    select_fallback_kernel<T><<<fb_grid, FB_THREADS, osm, st>>>(ix, n_blk, lq, PosSrc{pos, 0}, 1,
                                                                sp.budget, sp.window, sp.sinks,
                                                                s_max, indices, counts, ws);
    note_launch();
    return cudaGetLastError();
}

static int tree_u_cap(const IndexView& ix, int64_t NS, int branches)
{
    // room for the chosen branches' buckets: three times the mean branch size
    // per branch (larger universes take the exact fallback), within what
    // shared memory holds after the super scores
    const int64_t mean = (ix.NBK + NS - 1) / NS;
    int64_t cap = 3 * mean * branches + KC;
    const int64_t avail = (200 * 1024 - NS * 8) / 8;
    if (cap > avail) cap = avail;
    if (cap > ix.NBK) cap = ix.NBK;
    return (int)(cap < 0 ? 0 : cap);
}

size_t tree_select_ws_bytes(const IndexView& ix, int64_t Nq, int branches)
{
    return ws_bytes_shape(ix, Nq, true) + al256((size_t)ix.B * Nq * branches * 4);
}

template <typename T>
static cudaError_t launch_tree_t(const IndexView& ix, int64_t n_blk, const void* tree_buf,
                                 int64_t NS, int branches, const T* lq, const int32_t* positions,
                                 int64_t Nq, lsa_select_params sp, int32_t* indices,
                                 int32_t* counts, int s_max, void* ws_buf, cudaStream_t st)
{
    SelectWs ws = carve_shape(ws_buf, ix, Nq, true);
    ws.tree_br = (int32_t*)((char*)ws_buf + ws_bytes_shape(ix, Nq, true));
    ws.tree_nbr = branches;
    ws.tree_ns = NS;
    const void* sup_rt;
    tree_select_arrays(ix, tree_buf, NS, &sup_rt, &ws.tree_off, &ws.tree_mem);
    const int u_cap = tree_u_cap(ix, NS, branches);
    const size_t smem = (size_t)NS * 8 + (size_t)u_cap * 8;
    cudaError_t e = ensure_smem_attr((const void*)tree_nominate_kernel<T>, 200 * 1024);
    if (e != cudaSuccess) return e;
    const PosSrc pos{positions, 0};
    tree_nominate_kernel<T><<<dim3((unsigned)Nq, (unsigned)ix.B), TREE_THREADS, smem, st>>>(
        ix, n_blk, lq, pos, Nq, sp.window, ws, (const T*)sup_rt, NS, branches, u_cap);
    note_launch();
    return launch_finish_t(ix, n_blk, lq, pos, Nq, sp, indices, counts, s_max, ws, st);
}

cudaError_t launch_tree_select(const IndexView& ix, int64_t n_blk, const void* tree_buf,
                               int64_t NS, int branches, const void* latent_Q,
                               const int32_t* positions, int64_t Nq, lsa_select_params sp,
                               int32_t* indices, int32_t* counts, int s_max, void* ws,
                               cudaStream_t st)
{
    if (Nq <= 0) return cudaSuccess;
    if (branches < 1 || branches > TREE_MAX_BR || NS < 1 || NS * 8 > 100 * 1024 ||
        tree_u_cap(ix, NS, branches) < (ix.NBK < KC ? ix.NBK : KC))
        return cudaErrorInvalidValue;
    if (ix.dtype == LSA_BF16)
        return launch_tree_t(ix, n_blk, tree_buf, NS, branches, (const __nv_bfloat16*)latent_Q,
                             positions, Nq, sp, indices, counts, s_max, ws, st);
    return launch_tree_t(ix, n_blk, tree_buf, NS, branches, (const float*)latent_Q, positions,
                         Nq, sp, indices, counts, s_max, ws, st);
}

cudaError_t launch_decode_finish(const IndexView& ix, int64_t n_blk, const void* latent_q,
                                 const int32_t* pos, lsa_select_params sp, int32_t* indices,
                                 int32_t* counts, int s_max, const SelectWs& ws, cudaStream_t st)
{
    if (ix.dtype == LSA_BF16)
        return launch_decode_finish_t(ix, n_blk, (const __nv_bfloat16*)latent_q, pos, sp, indices,
                                      counts, s_max, ws, st);
    return launch_decode_finish_t(ix, n_blk, (const float*)latent_q, pos, sp, indices, counts,
                                  s_max, ws, st);
}

cudaError_t launch_select_finish(const IndexView& ix, int64_t n_blk, const void* latent_Q,
                                 PosSrc pos, int64_t Nq, lsa_select_params sp, int32_t* indices,
                                 int32_t* counts, int s_max, const SelectWs& ws, cudaStream_t st)
{
    if (ix.dtype == LSA_BF16)
        return launch_finish_t(ix, n_blk, (const __nv_bfloat16*)latent_Q, pos, Nq, sp, indices,
                               counts, s_max, ws, st);
    return launch_finish_t(ix, n_blk, (const float*)latent_Q, pos, Nq, sp, indices, counts, s_max,
                           ws, st);
}

}  // namespace lsa
