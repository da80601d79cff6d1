// attn_bucket.cuh -- tile description shared by the two bucket-major
// attention kernels (k_attn_bucket.cu: warp MMA; k_attn_bucket_tc.cu:
// tcgen05).  A tile is one bucket (or one run of consecutive queries' sinks
// and recent windows) with up to BA_Q queries that read it, for one KV head.
// Its keys form a list -- the bucket's closed members expanded to keys,
// then its open-block members; or the sinks, then the union of the windows --
// and each query reads at most two ranges of that list.
#pragma once

#include <limits.h>

#include "lsa_internal.cuh"

namespace lsa {

struct BaArgs {
    const __nv_bfloat16* Q;
    const __nv_bfloat16* K;
    const __nv_bfloat16* V;
    int64_t Nq;
    int Hq, Hkv, hpg;
    IndexView ix;
    int64_t n_blk;
    PosSrc pos;
    int W, S;
    BucketPlan P;
    int64_t wt_per_seq;   // window tiles per sequence
    int64_t n_wt;         // window tiles of all sequences
    float scale_log2;
};

struct QRange {
    int lo0, hi0, lo1, hi1;   // key-list index ranges [lo0, hi0) and [lo1, hi1)
    __device__ __forceinline__ bool has(int k) const
    {
        return (k >= lo0 && k < hi0) || (k >= lo1 && k < hi1);
    }
    __device__ __forceinline__ bool meets(int a, int b) const   // [a, b) intersects
    {
        return (lo0 < hi0 && lo0 < b && a < hi0) || (lo1 < hi1 && lo1 < b && a < hi1);
    }
    __device__ __forceinline__ bool covers(int a, int b) const  // [a, b) inside one range
    {
        return (lo0 <= a && b <= hi0) || (lo1 <= a && b <= hi1);
    }
};

struct __align__(16) TileInfo {
    QRange rng[BA_Q];
    int row[BA_Q];       // query row (b * Nq + i)
    int slot[BA_Q];      // partial slot, -1 for an empty query position
    int kind;            // 0 sinks + windows, 1 bucket
    int kbeg, kend;      // key-list range the tile walks
    int nsA;             // window tiles: sink keys at the head of the list
    int o0, nclosed;     // bucket tiles: first CSR position, closed keys
    int any_open;        // bucket tiles: some query reads open-block keys
    int h;               // KV head
    int n_st;            // stages (set by the kernel)
    long long b, wlo, g; // sequence; first window token; bucket in the sequence
};
static_assert(sizeof(TileInfo) == TILE_REC_BYTES, "tile record size");

// Fills ti for work item w (tile t = w / Hkv, KV head w % Hkv).  Executed by
// one whole warp; lanes < BA_Q own the tile's query positions.  kbeg is rounded
// down to a multiple of `align`, so that how a query's keys fall into steps --
// and so its fp32 summation order -- does not depend on which other queries
// share the tile.
__device__ __forceinline__ void ba_tile_setup(const BaArgs& a, int64_t w, int align, TileInfo* ti)
{
    const int lane = threadIdx.x & 31;
    const IndexView& ix = a.ix;
    const int h = (int)(w % a.Hkv);
    const int64_t t = w / a.Hkv;
    int live = 0, row = 0, slot = -1, n_open = 0;
    QRange r{0, 0, 0, 0};
    if (t < a.n_wt) {
        // sinks + recent windows of BA_Q consecutive queries
        const int64_t b = t / a.wt_per_seq;
        const int64_t i = (t % a.wt_per_seq) * BA_Q + lane;
        int64_t pq = 0, n_s = 0, w0 = 0;
        if (lane < BA_Q && i < a.Nq) {
            row = (int)(b * a.Nq + i);
            const int rn = a.P.row_n[row];
            if (rn >= 0) {
                live = 1;
                slot = a.P.row_base[row] + rn;
                pq = a.pos.at(b, a.Nq, i);
                n_s = (a.S < pq + 1) ? a.S : pq + 1;
                w0 = pq - a.W + 1;
                if (w0 < n_s) w0 = n_s;
            }
        }
        long long nsA = live ? n_s : 0, wmin = live ? w0 : LLONG_MAX,
                  whi = live ? pq + 1 : LLONG_MIN;
        for (int o = 16; o > 0; o >>= 1) {
            nsA = max(nsA, __shfl_xor_sync(0xffffffffu, nsA, o));
            wmin = min(wmin, __shfl_xor_sync(0xffffffffu, wmin, o));
            whi = max(whi, __shfl_xor_sync(0xffffffffu, whi, o));
        }
        const long long wlo = max(wmin, nsA);
        if (live) {
            r.lo0 = 0;
            r.hi0 = (int)n_s;
            if (pq + 1 > w0) {
                r.lo1 = (int)(nsA + (w0 - wlo));
                r.hi1 = (int)(nsA + (pq + 1 - wlo));
            }
        }
        if (lane == 0) {
            ti->kind = 0;
            ti->b = b;
            ti->g = 0;
            ti->nsA = (int)nsA;
            ti->wlo = (whi == LLONG_MIN) ? 0 : wlo;
            ti->o0 = 0;
            ti->nclosed = 0;
            ti->kbeg = 0;
            ti->kend = (whi == LLONG_MIN) ? 0 : (int)(nsA + (whi - wlo));
            ti->any_open = 0;
        }
    } else {
        // one tile of a bucket's queries
        const int2 tj = a.P.tiles[t - a.n_wt];
        const int64_t gg = tj.x;
        const int64_t b = gg / ix.NBK, g = gg % ix.NBK;
        const int cnt = a.P.bucket_cnt[gg];
        const int nq = min(BA_Q, cnt - tj.y * BA_Q);
        const int32_t* off = ix.offsets + b * (ix.NBK + 1);
        const int o0 = off[g];
        const int nclosed = (off[g + 1] - o0) * ix.p;
        if (lane < nq) {
            const int pidx = a.P.sorted[a.P.bucket_off[gg] + tj.y * BA_Q + lane];
            const int4 e = a.P.ent[pidx];
            n_open = a.P.ent2[pidx].y;
            live = 1;
            row = e.x;
            slot = pidx;
            r.lo0 = e.z;
            r.hi0 = e.w;
            r.lo1 = nclosed;
            r.hi1 = nclosed + n_open;
        }
        int kb = live ? ((r.hi0 > r.lo0) ? r.lo0 : r.lo1) : INT_MAX;
        int ke = live ? ((n_open > 0) ? r.hi1 : r.hi0) : 0;
        int any_open = n_open;
        for (int o = 16; o > 0; o >>= 1) {
            kb = min(kb, __shfl_xor_sync(0xffffffffu, kb, o));
            ke = max(ke, __shfl_xor_sync(0xffffffffu, ke, o));
            any_open = max(any_open, __shfl_xor_sync(0xffffffffu, any_open, o));
        }
        if (lane == 0) {
            ti->kind = 1;
            ti->b = b;
            ti->g = g;
            ti->nsA = 0;
            ti->wlo = 0;
            ti->o0 = o0;
            ti->nclosed = nclosed;
            ti->kbeg = (kb == INT_MAX) ? 0 : (kb / align) * align;
            ti->kend = (kb == INT_MAX) ? 0 : ke;
            ti->any_open = any_open > 0;
        }
    }
    if (lane < BA_Q) {
        ti->rng[lane] = r;
        ti->row[lane] = row;
        ti->slot[lane] = live ? slot : -1;
    }
    if (lane == 0) ti->h = h;
}

// Token of key-list index k of a tile (closed and open member lists in
// shared memory; lp = log2(p) when p is a power of two, else -1).
__device__ __forceinline__ int64_t ba_token(const TileInfo& ti, int k, int p, int lp,
                                            const int32_t* mem_list, const int32_t* open_list)
{
    if (ti.kind == 0) return (k < ti.nsA) ? (int64_t)k : (int64_t)ti.wlo + (k - ti.nsA);
    const bool closed = k < ti.nclosed;
    const int kk = closed ? k : k - ti.nclosed;
    const int q = (lp >= 0) ? (kk >> lp) : kk / p;
    const int rr = kk - q * p;
    return (int64_t)(closed ? mem_list[q] : open_list[q]) * p + rr;
}

// The bucket's open-block members (pooled ids, ascending) into open_list, by
// an ordered compaction over the open block.  Executed by nthreads threads
// (whole warps, ids 0 .. nthreads-1 via `tid`); cnt_s holds one int per warp;
// bar() synchronises exactly those threads.
template <typename Bar>
__device__ __forceinline__ void ba_open_list(const IndexView& ix, int64_t n_blk, long long b,
                                             long long g, int tid, int nthreads, int* cnt_s,
                                             int32_t* open_list, Bar bar)
{
    const int32_t* open = ix.open_bucket + b * ix.G;
    const int lane = tid & 31, warp = tid >> 5, nw = nthreads >> 5;
    constexpr int U = 8;   // loads in flight per thread
    int base = 0;
    for (int x00 = 0; x00 < ix.G; x00 += U * nthreads) {
        int32_t bk[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int x = x00 + u * nthreads + tid;
            bk[u] = (x < ix.G) ? open[x] : -1;
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            if (x00 + u * nthreads >= ix.G) break;   // uniform over the threads
            const int x = x00 + u * nthreads + tid;
            const bool hit = x < ix.G && bk[u] == g;
            const unsigned bal = __ballot_sync(0xffffffffu, hit);
            if (lane == 0) cnt_s[warp] = __popc(bal);
            bar();
            int before = base;
            for (int w2 = 0; w2 < warp; ++w2) before += cnt_s[w2];
            if (hit) open_list[before + __popc(bal & ((1u << lane) - 1u))] = (int32_t)(n_blk * ix.G + x);
            for (int w2 = 0; w2 < nw; ++w2) base += cnt_s[w2];
            bar();
        }
    }
}

// Writes the description of every tile (window tiles first, then bucket
// tiles) to P.recs, with n_st counted in `align`-key stages; a tile whose
// queries read nothing still walks one (masked) key.
cudaError_t launch_tile_records(const BaArgs& a, int align, cudaStream_t st);

// The tensor-core tile kernel (k_attn_bucket_tc.cu) and the shapes it serves.
bool bucket_attn_tc_supported(int Hq, int Hkv, int d, int G);
cudaError_t launch_bucket_attn_tc(const BaArgs& a, int d, cudaStream_t st);

}  // namespace lsa
