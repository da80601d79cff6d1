// k_attn_bucket.cu -- bucket-major exact sparse attention for prefill chunks.
//
// Method: "Latent Sparse Attention: un indice gerarchico per contesti lunghi",
// paragraph on retrieval: a query attends exactly over the keys of the
// buckets it took (the last one cut to the budget), its sinks and its recent
// window.  "Prefrontal's Latent Sparse Attention speeds up one attention layer
// 72x at 10M tokens ...", section "What it changes": only the choice of keys
// changes, the attention itself is exact softmax attention.
//
// The queries of one prefill chunk take many of the same buckets.  Instead of
// gathering every query's keys separately, this path groups the work by key
// set: a tile is one bucket (or one run of consecutive queries' sinks and
// windows) with up to BA_Q queries that read it, for one KV head.  A tile's
// key rows are streamed through shared memory once and serve all of its
// queries; each query keeps an fp32 online-softmax state for the keys of its
// own range and writes an unnormalised partial (acc, max, sum).  A merge then
// combines each query's partials (one per taken bucket plus one for sinks and
// window) into the output -- the same softmax, summed in another order.
//
// Pipeline of one tile (persistent CTAs, work items from an atomic counter):
// all 8 warps issue 16-byte cp.async copies of the next stages' K and V rows
// (64 keys per stage, one KV head: 256 B per key at d = 128) into an
// XOR-swizzled layout (16-byte chunk c of row r stored at chunk c ^ (r & 7)),
// so the ldmatrix reads of 8 consecutive keys hit 8 different bank groups.
// Warp w owns queries 2w and 2w+1: it computes S^T = K Q^T for both from the
// same K fragments (keys on the MMA M dimension, the query heads of the KV head
// on N), masks keys outside each query's ranges, and accumulates
// O^T = V^T P^T, again sharing the V fragments.
#include <limits.h>
#include <math.h>

#include "attn_bucket.cuh"
#include "lsa_internal.cuh"
#include "ptx.cuh"

namespace lsa {

#ifndef LSA_BA_STAGES
#define LSA_BA_STAGES 3
#endif
#ifndef LSA_BA_MIN_BLOCKS
#define LSA_BA_MIN_BLOCKS 2     // resident CTAs per SM the register budget is sized for
#endif
constexpr int BA_K = 64;          // keys per pipeline stage
constexpr int BA_STAGES = LSA_BA_STAGES;
constexpr int BA_WARPS = 8;       // two queries each
constexpr int BA_THREADS = BA_WARPS * 32;
constexpr int PLAN_THREADS = 1024;

template <int D>
struct BaCfg {
    static constexpr int ROWB = D * 2;          // bytes of one key's row of one KV head
    static constexpr int CH = ROWB / 16;        // 16-byte chunks per row
    static constexpr int TILE = BA_K * ROWB;    // K (or V) bytes of a stage
    static constexpr int STAGE = 2 * TILE;
    static constexpr int RING = BA_STAGES * STAGE;
};


// ---------------------------------------------------------------------------
// Plan: one CTA scans the per-bucket entry counts into each bucket's first
// sorted position and lists the tiles (bucket, tile number) in bucket order.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(PLAN_THREADS) bucket_plan_kernel(BucketPlan P, int64_t nbt)
{
    __shared__ long long we[PLAN_THREADS / 32], wt[PLAN_THREADS / 32];
    __shared__ long long tot_t;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t chunk = (nbt + PLAN_THREADS - 1) / PLAN_THREADS;
    const int64_t g0 = min(nbt, (int64_t)tid * chunk), g1 = min(nbt, g0 + chunk);
    long long se = 0, st = 0;
    for (int64_t g = g0; g < g1; ++g) {
        const int c = P.bucket_cnt[g];
        se += c;
        st += (c + BA_Q - 1) / BA_Q;
    }
    long long ie = se, it = st;   // inclusive scans inside the warp
    for (int o = 1; o < 32; o <<= 1) {
        const long long ye = __shfl_up_sync(0xffffffffu, ie, o);
        const long long yt = __shfl_up_sync(0xffffffffu, it, o);
        if (lane >= o) {
            ie += ye;
            it += yt;
        }
    }
    if (lane == 31) {
        we[warp] = ie;
        wt[warp] = it;
    }
    __syncthreads();
    if (warp == 0) {
        const long long ve = we[lane], vt = wt[lane];
        long long xe = ve, xt = vt;
        for (int o = 1; o < 32; o <<= 1) {
            const long long ye = __shfl_up_sync(0xffffffffu, xe, o);
            const long long yt = __shfl_up_sync(0xffffffffu, xt, o);
            if (lane >= o) {
                xe += ye;
                xt += yt;
            }
        }
        we[lane] = xe - ve;   // exclusive warp offsets
        wt[lane] = xt - vt;
        if (lane == 31) tot_t = xt;
    }
    __syncthreads();
    long long eo = we[warp] + ie - se, to = wt[warp] + it - st;
    for (int64_t g = g0; g < g1; ++g) {
        const int c = P.bucket_cnt[g];
        P.bucket_off[g] = (int32_t)eo;
        eo += c;
        const int nt = (c + BA_Q - 1) / BA_Q;
        for (int j = 0; j < nt; ++j, ++to)
            if (to < P.tile_cap) P.tiles[to] = make_int2((int)g, j);
    }
    if (tid == 0) {
        P.ctr[CTR_TILES] = (int32_t)(tot_t < P.tile_cap ? tot_t : P.tile_cap);
        P.ctr[CTR_WORK] = 0;
    }
}

// Every granted bucket entry goes to its bucket's sorted run, at its rank.
__global__ void __launch_bounds__(256) bucket_scatter_kernel(BucketPlan P)
{
    const int64_t n = P.ctr[CTR_VALID_END];
    for (int64_t x = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; x < n;
         x += (int64_t)gridDim.x * blockDim.x) {
        const int4 e = P.ent[x];
        if (e.y >= 0) P.sorted[P.bucket_off[e.y] + P.ent2[x].x] = (int32_t)x;
    }
}

// One warp per tile: the tile descriptions the tensor-core kernel's planner
// warp copies in one piece (instead of following the plan's pointers).
__global__ void __launch_bounds__(256) bucket_tile_records_kernel(BaArgs a, int align)
{
    const int64_t n_tiles = a.n_wt + a.P.ctr[CTR_TILES];
    TileInfo* recs = reinterpret_cast<TileInfo*>(a.P.recs);
    const int lane = threadIdx.x & 31;
    for (int64_t t = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < n_tiles;
         t += ((int64_t)gridDim.x * blockDim.x) >> 5) {
        TileInfo* T = recs + t;
        ba_tile_setup(a, t * a.Hkv, align, T);
        __syncwarp();
        if (lane == 0) {
            const int nk = T->kend - T->kbeg;
            T->n_st = (nk > 0) ? (nk + align - 1) / align : 1;
            if (T->kend <= T->kbeg) T->kend = T->kbeg + 1;   // one masked key
        }
        __syncwarp();
    }
}

cudaError_t launch_tile_records(const BaArgs& a, int align, cudaStream_t st)
{
    bucket_tile_records_kernel<<<(unsigned)(sm_count() * 8), 256, 0, st>>>(a, align);
    note_launch();
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// The tile kernel.
// ---------------------------------------------------------------------------

// One 16-key online-softmax step for one query (heads h0 = 2*(lane&3) and
// h0+1 of the thread's accumulator columns); returns P^T as the B fragments
// of O^T = V^T P^T.
template <int KSTEPS>
__device__ __forceinline__ void ba_softmax(const float (&s)[4], int key_lo, const QRange& r,
                                           bool all_in, float scale_log2, float& m0, float& m1,
                                           float& l0, float& l1, float (&o)[KSTEPS][4],
                                           uint32_t& pb0, uint32_t& pb1)
{
    const int key_hi = key_lo + 8;
    const bool v_lo = all_in || r.has(key_lo), v_hi = all_in || r.has(key_hi);
    const float z0 = v_lo ? s[0] * scale_log2 : -INFINITY;
    const float z1 = v_lo ? s[1] * scale_log2 : -INFINITY;
    const float z2 = v_hi ? s[2] * scale_log2 : -INFINITY;
    const float z3 = v_hi ? s[3] * scale_log2 : -INFINITY;
    float tm0 = fmaxf(z0, z2), tm1 = fmaxf(z1, z3);
#pragma unroll
    for (int o_ = 4; o_ < 32; o_ <<= 1) {
        tm0 = fmaxf(tm0, __shfl_xor_sync(0xffffffffu, tm0, o_));
        tm1 = fmaxf(tm1, __shfl_xor_sync(0xffffffffu, tm1, o_));
    }
    const float mn0 = fmaxf(m0, tm0), mn1 = fmaxf(m1, tm1);
    const float al0 = (m0 == -INFINITY) ? 0.f : exp2f(m0 - mn0);
    const float al1 = (m1 == -INFINITY) ? 0.f : exp2f(m1 - mn1);
    const float mu0 = (mn0 == -INFINITY) ? 0.f : mn0;
    const float mu1 = (mn1 == -INFINITY) ? 0.f : mn1;
    const float p0 = exp2f(z0 - mu0), p1 = exp2f(z1 - mu1);
    const float p2 = exp2f(z2 - mu0), p3 = exp2f(z3 - mu1);
    // the accumulator needs rescaling only where a running max moved after
    // something was accumulated (before that it is exactly zero)
    const bool moved = (al0 != 1.f && m0 != -INFINITY) || (al1 != 1.f && m1 != -INFINITY);
    m0 = mn0;
    m1 = mn1;
    l0 = l0 * al0 + (p0 + p2);
    l1 = l1 * al1 + (p1 + p3);
    if (__any_sync(0xffffffffu, moved)) {
#pragma unroll
        for (int mt = 0; mt < KSTEPS; ++mt) {
            o[mt][0] *= al0;
            o[mt][1] *= al1;
            o[mt][2] *= al0;
            o[mt][3] *= al1;
        }
    }
    pb0 = ptx::movmatrix_t(ptx::pack_bf16(p0, p1));
    pb1 = ptx::movmatrix_t(ptx::pack_bf16(p2, p3));
}

// Writes one query's partial for the query heads of KV head h: per head the
// accumulator normalised by its own sum, as bf16 (po [hpg][D]), and the
// (max in log2 units, sum) pair (pml [hpg]).
template <int KSTEPS>
__device__ __forceinline__ void ba_write_partial(__nv_bfloat16* po, float2* pml, int hpg, float m0,
                                                 float m1, float l0, float l1,
                                                 const float (&o)[KSTEPS][4])
{
    constexpr int D = KSTEPS * 16;
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o_ = 4; o_ < 32; o_ <<= 1) {
        l0 += __shfl_xor_sync(0xffffffffu, l0, o_);
        l1 += __shfl_xor_sync(0xffffffffu, l1, o_);
    }
    const float i0 = (l0 > 0.f) ? 1.f / l0 : 0.f, i1 = (l1 > 0.f) ? 1.f / l1 : 0.f;
    const int h0 = 2 * (lane & 3), dr = lane >> 2;
#pragma unroll
    for (int mt = 0; mt < KSTEPS; ++mt) {
        if (h0 < hpg) {
            po[h0 * D + mt * 16 + dr] = __float2bfloat16_rn(o[mt][0] * i0);
            po[h0 * D + mt * 16 + dr + 8] = __float2bfloat16_rn(o[mt][2] * i0);
        }
        if (h0 + 1 < hpg) {
            po[(h0 + 1) * D + mt * 16 + dr] = __float2bfloat16_rn(o[mt][1] * i1);
            po[(h0 + 1) * D + mt * 16 + dr + 8] = __float2bfloat16_rn(o[mt][3] * i1);
        }
    }
    if (dr == 0) {
        if (h0 < hpg) pml[h0] = make_float2(m0, l0);
        if (h0 + 1 < hpg) pml[h0 + 1] = make_float2(m1, l1);
    }
}

template <int D>
__global__ void __launch_bounds__(BA_THREADS, LSA_BA_MIN_BLOCKS) bucket_attn_kernel(BaArgs a)
{
    using C = BaCfg<D>;
    constexpr int KSTEPS = D / 16;
    extern __shared__ __align__(128) unsigned char smem[];
    int32_t* mem_list = reinterpret_cast<int32_t*>(smem + C::RING);    // [G] closed members
    int32_t* open_list = mem_list + a.ix.G;                             // [G] open members
    __shared__ TileInfo ti;
    __shared__ int sh_work;
    __shared__ int ws_cnt[BA_THREADS / 32];

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const IndexView& ix = a.ix;
    const int p = ix.p;
    const int lp = ((p & (p - 1)) == 0) ? __ffs(p) - 1 : -1;
    const int64_t n_work = (a.n_wt + a.P.ctr[CTR_TILES]) * a.Hkv;
    int w_next = 0;
    if (tid == 0) w_next = atomicAdd(a.P.ctr + CTR_WORK, 1);

    for (;;) {
        if (tid == 0) {
            sh_work = w_next;
            w_next = atomicAdd(a.P.ctr + CTR_WORK, 1);   // consumed by the next item
        }
        __syncthreads();
        const int64_t w = sh_work;
        if (w >= n_work) break;
        if (warp == 0) ba_tile_setup(a, w, 16, &ti);
        __syncthreads();
        const int h = ti.h;
        const long long b = ti.b;
        const int kbeg = ti.kbeg, kend = ti.kend;

        // the bucket's closed members (pooled ids, ascending) into shared memory
        if (ti.kind == 1) {
            const int32_t* mem = ix.members + b * ix.NP + ti.o0;
            for (int x = tid; x < ti.nclosed / p; x += BA_THREADS) mem_list[x] = mem[x];
            if (ti.any_open)
                ba_open_list(ix, a.n_blk, b, ti.g, tid, BA_THREADS, ws_cnt, open_list,
                             [] { __syncthreads(); });
        }
        __syncthreads();   // member lists visible to every thread

        const int n_st = (kend > kbeg) ? (kend - kbeg + BA_K - 1) / BA_K : 0;
        const size_t tstride = (size_t)a.Hkv * D;   // elements between consecutive tokens
        const __nv_bfloat16* Kb = a.K + ((size_t)b * ix.T_cap * a.Hkv + h) * D;
        const __nv_bfloat16* Vb = a.V + ((size_t)b * ix.T_cap * a.Hkv + h) * D;
        auto issue = [&](int s) {
            unsigned char* kt = smem + (s % BA_STAGES) * C::STAGE;
            const int kb = kbeg + s * BA_K;
            int32_t tok[BA_K * C::CH / BA_THREADS];   // tokens < T_cap < 2^31
#pragma unroll
            for (int i = 0; i < BA_K * C::CH / BA_THREADS; ++i) {
                const int r = (tid + i * BA_THREADS) / C::CH;
                int k = kb + r;
                if (k >= kend) k = kend - 1;   // padding rows repeat a real key (masked)
                const int64_t t = ba_token(ti, k, p, lp, mem_list, open_list);
                tok[i] = (int32_t)t;
                if (t < 0 || t >= ix.T_cap) {
                    dev_error(ix.status, DEV_BAD_INDEX, (uint32_t)t);
                    tok[i] = 0;
                }
            }
#pragma unroll
            for (int i = 0; i < BA_K * C::CH / BA_THREADS; ++i) {
                const int x = tid + i * BA_THREADS;
                const int r = x / C::CH, c = x % C::CH;
                const size_t goff = (size_t)tok[i] * tstride + c * 8;
                const int soff = r * C::ROWB + ((c ^ (r & 7)) << 4);
                ptx::cp_async16(kt + soff, Kb + goff);
                ptx::cp_async16(kt + C::TILE + soff, Vb + goff);
            }
        };

        // this warp's two queries
        const int qa = 2 * warp, qb = qa + 1;
        const bool liveA = ti.slot[qa] >= 0, liveB = ti.slot[qb] >= 0;
        const QRange ra = ti.rng[qa], rb = ti.rng[qb];
        uint32_t qfa[KSTEPS][2], qfb[KSTEPS][2];
        {
            const int hh = lane >> 2;
            const bool hl = hh < a.hpg;
            const __nv_bfloat16* qra =
                a.Q + ((size_t)ti.row[qa] * a.Hq + (size_t)h * a.hpg + (hl ? hh : 0)) * D;
            const __nv_bfloat16* qrb =
                a.Q + ((size_t)ti.row[qb] * a.Hq + (size_t)h * a.hpg + (hl ? hh : 0)) * D;
#pragma unroll
            for (int kk = 0; kk < KSTEPS; ++kk) {
                const int c = kk * 16 + 2 * (lane & 3);
                qfa[kk][0] = (liveA && hl) ? *reinterpret_cast<const uint32_t*>(qra + c) : 0u;
                qfa[kk][1] = (liveA && hl) ? *reinterpret_cast<const uint32_t*>(qra + c + 8) : 0u;
                qfb[kk][0] = (liveB && hl) ? *reinterpret_cast<const uint32_t*>(qrb + c) : 0u;
                qfb[kk][1] = (liveB && hl) ? *reinterpret_cast<const uint32_t*>(qrb + c + 8) : 0u;
            }
        }
        float ma0 = -INFINITY, ma1 = -INFINITY, la0 = 0.f, la1 = 0.f;
        float mb0 = -INFINITY, mb1 = -INFINITY, lb0 = 0.f, lb1 = 0.f;
        float oa[KSTEPS][4], ob[KSTEPS][4];
#pragma unroll
        for (int mt = 0; mt < KSTEPS; ++mt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                oa[mt][e] = 0.f;
                ob[mt][e] = 0.f;
            }

#pragma unroll
        for (int s = 0; s < BA_STAGES - 1; ++s) {
            if (s < n_st) issue(s);
            ptx::cp_async_commit();
        }
        const int xk = (lane >> 4) ^ (lane & 7);          // K fragment rows: chunk 2kk ^ xk
        const int xv = ((lane >> 3) & 1) ^ (lane & 7);    // V^T fragment rows: chunk 2mt ^ xv
        for (int s = 0; s < n_st; ++s) {
            ptx::cp_async_wait<BA_STAGES - 2>();
            __syncthreads();
            if (s + BA_STAGES - 1 < n_st) issue(s + BA_STAGES - 1);
            ptx::cp_async_commit();
            const unsigned char* kt = smem + (s % BA_STAGES) * C::STAGE;
            const unsigned char* vt = kt + C::TILE;
            const int kb = kbeg + s * BA_K;
#pragma unroll 1
            for (int sub = 0; sub < BA_K / 16; ++sub) {
                const int k0 = kb + sub * 16;
                if (k0 >= kend) break;
                const bool actA = liveA && ra.meets(k0, k0 + 16);
                const bool actB = liveB && rb.meets(k0, k0 + 16);
                if (!actA && !actB) continue;
                // two accumulation chains per query (even and odd k-steps)
                float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
                float sa2[4] = {0.f, 0.f, 0.f, 0.f}, sb2[4] = {0.f, 0.f, 0.f, 0.f};
                {
                    const unsigned char* rowp = kt + (sub * 16 + (lane & 15)) * C::ROWB;
#pragma unroll
                    for (int kk = 0; kk < KSTEPS; ++kk) {
                        uint32_t a0, a1, a2, a3;
                        ptx::ldsm_x4(a0, a1, a2, a3, rowp + (((2 * kk) ^ xk) << 4));
                        float* ca = (kk & 1) ? sa2 : sa;
                        float* cb = (kk & 1) ? sb2 : sb;
                        if (actA) ptx::mma_bf16_16816(ca, a0, a1, a2, a3, qfa[kk][0], qfa[kk][1]);
                        if (actB) ptx::mma_bf16_16816(cb, a0, a1, a2, a3, qfb[kk][0], qfb[kk][1]);
                    }
                }
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    sa[e] += sa2[e];
                    sb[e] += sb2[e];
                }
                const int key_lo = k0 + (lane >> 2);
                uint32_t pa0 = 0, pa1 = 0, pb0 = 0, pb1 = 0;
                if (actA)
                    ba_softmax<KSTEPS>(sa, key_lo, ra, ra.covers(k0, k0 + 16), a.scale_log2, ma0,
                                       ma1, la0, la1, oa, pa0, pa1);
                if (actB)
                    ba_softmax<KSTEPS>(sb, key_lo, rb, rb.covers(k0, k0 + 16), a.scale_log2, mb0,
                                       mb1, lb0, lb1, ob, pb0, pb1);
                {
                    const int r = (lane & 7) + 8 * ((lane >> 4) & 1);
                    const unsigned char* rowp = vt + (sub * 16 + r) * C::ROWB;
#pragma unroll
                    for (int mt = 0; mt < KSTEPS; ++mt) {
                        uint32_t a0, a1, a2, a3;
                        ptx::ldsm_x4_t(a0, a1, a2, a3, rowp + (((2 * mt) ^ xv) << 4));
                        if (actA) ptx::mma_bf16_16816(oa[mt], a0, a1, a2, a3, pa0, pa1);
                        if (actB) ptx::mma_bf16_16816(ob[mt], a0, a1, a2, a3, pb0, pb1);
                    }
                }
            }
        }
        ptx::cp_async_wait<0>();

        if (liveA) {
            const size_t ph = (size_t)ti.slot[qa] * a.Hq + (size_t)h * a.hpg;
            ba_write_partial<KSTEPS>(a.P.part_o + ph * D, a.P.part_ml + ph, a.hpg, ma0, ma1, la0,
                                     la1, oa);
        }
        if (liveB) {
            const size_t ph = (size_t)ti.slot[qb] * a.Hq + (size_t)h * a.hpg;
            ba_write_partial<KSTEPS>(a.P.part_o + ph * D, a.P.part_ml + ph, a.hpg, mb0, mb1, lb0,
                                     lb1, ob);
        }
        __syncthreads();   // the next tile rewrites the ring and the tile's shared state
    }
}

// ---------------------------------------------------------------------------
// Merge: one CTA per listed query row combines the row's nt + 1 partials.
// Partial s holds O_s / l_s (bf16) with its max m_s and sum l_s per query
// head: with M the head's largest max and w_s = l_s exp2(m_s - M), the output
// is sum_s w_s (O_s / l_s) / sum_s w_s.  A row's partial slots are
// consecutive, so the (max, sum) pairs of all its slots and heads are one
// contiguous block, and each slot's outputs for all heads are another
// (Hq * d bf16, 8 KB at 32 x 128): every load is coalesced.
// ---------------------------------------------------------------------------
constexpr int MERGE_THREADS = 256;
constexpr int MERGE_MAX_SLOTS = KC + 1;
constexpr int MERGE_MAX_HEADS = 64;

__global__ void __launch_bounds__(MERGE_THREADS) bucket_merge_kernel(BucketPlan P, int Hq, int D,
                                                                     __nv_bfloat16* O)
{
    // (max, sum) per [slot][head]; the normalised weight then replaces the max
    __shared__ float2 ml_s[MERGE_MAX_SLOTS * MERGE_MAX_HEADS];
    const int64_t row = blockIdx.x;
    const int nt = P.row_n[row];
    if (nt < 0) return;                        // gather row: written by the per-query kernel
    const int ns = nt + 1;
    const int64_t base = (int64_t)P.row_base[row] * Hq;   // first (slot, head)
    const float2* ml = P.part_ml + base;
    // every (slot, head) pair of the row in one coalesced pass
    for (int x = threadIdx.x; x < ns * Hq; x += MERGE_THREADS) ml_s[x] = __ldcg(&ml[x]);
    __syncthreads();
    // weights exp2(m - M) * sum: one pass per head over its slots
    for (int h = threadIdx.x; h < Hq; h += MERGE_THREADS) {
        float M = -INFINITY;
        for (int sl = 0; sl < ns; ++sl) M = fmaxf(M, ml_s[sl * Hq + h].x);
        float L = 0.f;
        for (int sl = 0; sl < ns; ++sl) {
            const float2 v = ml_s[sl * Hq + h];
            const float wv = (v.x == -INFINITY) ? 0.f : v.y * exp2f(v.x - M);
            ml_s[sl * Hq + h].x = wv;
            L += wv;
        }
        const float inv = 1.f / L;
        for (int sl = 0; sl < ns; ++sl) ml_s[sl * Hq + h].x *= inv;
    }
    __syncthreads();
    const int n8 = Hq * D / 8;                 // 16-byte groups of the row's output
    const __nv_bfloat16* src = P.part_o + base * D;
    __nv_bfloat16* dst = O + row * (int64_t)Hq * D;
    for (int c = threadIdx.x; c < n8; c += MERGE_THREADS) {
        const int h = (c * 8) / D;
        float acc[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll 4
        for (int sl = 0; sl < ns; ++sl) {
            const uint4 u = __ldcg(reinterpret_cast<const uint4*>(src + (int64_t)sl * Hq * D) + c);
            const float wv = ml_s[sl * Hq + h].x;
            const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 f = __bfloat1622float2(b2[e]);
                acc[2 * e] = fmaf(f.x, wv, acc[2 * e]);
                acc[2 * e + 1] = fmaf(f.y, wv, acc[2 * e + 1]);
            }
        }
        uint4 out;
        uint32_t* o32 = reinterpret_cast<uint32_t*>(&out);
#pragma unroll
        for (int e = 0; e < 4; ++e) o32[e] = ptx::pack_bf16(acc[2 * e], acc[2 * e + 1]);
        reinterpret_cast<uint4*>(dst)[c] = out;
    }
}

bool bucket_attn_supported(int Hq, int Hkv, int d)
{
    return (d == 64 || d == 128) && Hkv >= 1 && Hq % Hkv == 0 && Hq / Hkv <= 8 &&
           Hq <= MERGE_MAX_HEADS;
}

template <int D>
static cudaError_t launch_tiles(const BaArgs& a, cudaStream_t st)
{
    using C = BaCfg<D>;
    auto kern = bucket_attn_kernel<D>;
    const int smem = C::RING + 2 * a.ix.G * 4;
    // the limit is raised once per device, for the largest block (4096 groups)
    cudaError_t e = ensure_smem_attr((const void*)kern, C::RING + 2 * 4096 * 4);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, BA_THREADS, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    kern<<<(unsigned)(sm_count() * per_sm), BA_THREADS, smem, st>>>(a);
    note_launch();
    return cudaGetLastError();
}

cudaError_t launch_bucket_attn(const IndexView& ix, int64_t n_blk, const BucketPlan& P,
                               const void* Q, const void* K, const void* V, int64_t Nq, int Hq,
                               int Hkv, int d, PosSrc pos, int W, int S, const int32_t* indices,
                               const int32_t* counts, int s_max, float scale, void* O,
                               cudaStream_t st)
{
    if (ix.B * Nq == 0) return cudaSuccess;
    const int64_t nbt = ix.B * ix.NBK;
    bucket_plan_kernel<<<1, PLAN_THREADS, 0, st>>>(P, nbt);
    note_launch();
    bucket_scatter_kernel<<<(unsigned)(sm_count() * 4), 256, 0, st>>>(P);
    note_launch();
    BaArgs a;
    a.Q = (const __nv_bfloat16*)Q;
    a.K = (const __nv_bfloat16*)K;
    a.V = (const __nv_bfloat16*)V;
    a.Nq = Nq;
    a.Hq = Hq;
    a.Hkv = Hkv;
    a.hpg = Hq / Hkv;
    a.ix = ix;
    a.n_blk = n_blk;
    a.pos = pos;
    a.W = W;
    a.S = S;
    a.P = P;
    a.wt_per_seq = (Nq + BA_Q - 1) / BA_Q;
    a.n_wt = ix.B * a.wt_per_seq;
    a.scale_log2 = scale * 1.4426950408889634f;
    cudaError_t e;
    if (bucket_attn_tc_supported(Hq, Hkv, d, ix.G)) {
        e = launch_tile_records(a, 64, st);
        if (e != cudaSuccess) return e;
        e = launch_bucket_attn_tc(a, d, st);
    } else
        e = (d == 128) ? launch_tiles<128>(a, st) : launch_tiles<64>(a, st);
    if (e != cudaSuccess) return e;
    e = launch_attn_rows(Q, K, V, ix.B, Nq, ix.T_cap, Hq, Hkv, d, indices, counts, s_max, scale, O,
                         ix.status, P.gather_rows, P.ctr + CTR_GATHER, st);
    if (e != cudaSuccess) return e;
    bucket_merge_kernel<<<(unsigned)(ix.B * Nq), MERGE_THREADS, 0, st>>>(P, Hq, d,
                                                                        (__nv_bfloat16*)O);
    note_launch();
    return cudaGetLastError();
}

}  // namespace lsa
