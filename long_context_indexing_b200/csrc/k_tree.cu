// k_tree.cu -- level 2 of the D-LSA Tree: spherical k-means of each
// sequence's closed-bucket centroids into super-buckets.
//
// Method: "Prefrontal's Latent Sparse Attention speeds up one attention layer
// 72x at 10M tokens; end to end, the gain is 9x", section "What it changes":
// clusters are grouped into a hierarchy that a query walks down, scoring a
// few clusters at each level.  "Latent Sparse Attention: un indice gerarchico
// per contesti lunghi", paragraph on Flat vs Tree.  The construction is this
// library's reading: the buckets' fp32 centroids are clustered exactly like a
// block's unit vectors -- init c2_h = c[floor(h * NB / NS)], L Lloyd
// iterations of {assign each centroid to the super-centroid of largest exact
// <c, c2_h> (binary64 sum in ascending dimension, ties to the lowest h);
// c2_h = normalised binary64 sum of its members in ascending bucket order, an
// empty super-bucket keeps its centroid} -- and the final assignment becomes
// a CSR list per super-bucket (bucket ids ascending) with a retrieval copy of
// the super-centroids (bf16 for bf16 indices).
//
// Kernels per Lloyd iteration: assign (a thread per centroid, super-centroids
// staged in shared memory; per CTA of 256 centroids, one thread then walks
// them in order to give each its rank among the CTA's centroids of the same
// super-bucket and the CTA's counts), scan (a thread per super-bucket: its
// per-CTA bases and its CSR offset), scatter (stable: bucket ids land in
// ascending order), update (a CTA per super-bucket, a thread per dimension,
// eight member rows in flight).  All arithmetic that decides an integer is
// binary64 with exact products, so the result is reproducible bit for bit.
#include <math.h>

#include "lsa_internal.cuh"

namespace lsa {

constexpr int TR_PTS = 256;          // centroids per assign CTA
constexpr int TR_TILE = 256;         // super-centroids staged per pass

// Storage of a tree (one caller buffer; every array on a 256-byte boundary).
struct TreeView {
    int64_t B, NBK, NS;
    float* sup;          // [B][NS][64] fp32 super-centroids
    void* sup_rt;        // [B][NS][64] retrieval copy (index dtype)
    int32_t* off;        // [B][NS + 1] CSR offsets
    int32_t* mem;        // [B][NBK] bucket ids, ascending inside a super-bucket
    int32_t* asg;        // [B][NBK] super-bucket of every bucket
    int32_t* rank;       // [B][NBK] rank among its CTA's buckets of the same super-bucket
    int32_t* hist;       // [B][n_cta][NS] per-CTA counts, then per-CTA bases
};

static inline size_t al256t(size_t x) { return (x + 255) & ~(size_t)255; }

static TreeView tree_view(const IndexView& ix, void* buf, int64_t NS)
{
    TreeView t;
    t.B = ix.B;
    t.NBK = ix.NBK;
    t.NS = NS;
    const size_t es = (ix.dtype == LSA_BF16) ? 2 : 4;
    const int64_t n_cta = (ix.NBK + TR_PTS - 1) / TR_PTS;
    char* p = (char*)buf;
    t.sup = (float*)p;     p += al256t((size_t)ix.B * NS * DL * 4);
    t.sup_rt = p;          p += al256t((size_t)ix.B * NS * DL * es);
    t.off = (int32_t*)p;   p += al256t((size_t)ix.B * (NS + 1) * 4);
    t.mem = (int32_t*)p;   p += al256t((size_t)ix.B * ix.NBK * 4);
    t.asg = (int32_t*)p;   p += al256t((size_t)ix.B * ix.NBK * 4);
    t.rank = (int32_t*)p;  p += al256t((size_t)ix.B * ix.NBK * 4);
    t.hist = (int32_t*)p;  p += al256t((size_t)ix.B * n_cta * NS * 4);
    return t;
}

size_t tree_bytes(const IndexView& ix, int64_t NS)
{
    const size_t es = (ix.dtype == LSA_BF16) ? 2 : 4;
    const int64_t n_cta = (ix.NBK + TR_PTS - 1) / TR_PTS;
    return al256t((size_t)ix.B * NS * DL * 4) + al256t((size_t)ix.B * NS * DL * es) +
           al256t((size_t)ix.B * (NS + 1) * 4) + 3 * al256t((size_t)ix.B * ix.NBK * 4) +
           al256t((size_t)ix.B * n_cta * NS * 4);
}

// c2_h = c[floor(h * NB / NS)]
__global__ void tree_init_kernel(IndexView ix, TreeView t, int64_t NB)
{
    const int64_t b = blockIdx.y;
    for (int64_t x = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; x < t.NS * DL;
         x += (int64_t)gridDim.x * blockDim.x) {
        const int64_t h = x / DL, i = x % DL;
        const int64_t src = (h * NB) / t.NS;
        t.sup[(b * t.NS + h) * DL + i] = ix.cent[(b * ix.NBK + src) * DL + i];
    }
}

// assign + per-CTA ranks and counts
__global__ void __launch_bounds__(TR_PTS) tree_assign_kernel(IndexView ix, TreeView t, int64_t NB)
{
    extern __shared__ float tile[];                  // [TR_TILE][DL + 1]
    __shared__ int32_t asg_s[TR_PTS];
    const int64_t b = blockIdx.y;
    const int64_t cta = blockIdx.x;
    const int64_t g = cta * TR_PTS + threadIdx.x;
    const bool live = g < NB;
    float c[DL];
    if (live) {
        const float4* row = reinterpret_cast<const float4*>(ix.cent + (b * ix.NBK + g) * DL);
#pragma unroll
        for (int x = 0; x < DL / 4; ++x) {
            const float4 f = row[x];
            c[4 * x] = f.x;
            c[4 * x + 1] = f.y;
            c[4 * x + 2] = f.z;
            c[4 * x + 3] = f.w;
        }
    }
    double best = -INFINITY;
    int bh = 0;
    for (int64_t h0 = 0; h0 < t.NS; h0 += TR_TILE) {
        const int nh = (int)((t.NS - h0) < TR_TILE ? (t.NS - h0) : TR_TILE);
        __syncthreads();
        for (int x = threadIdx.x; x < nh * DL; x += blockDim.x)
            tile[(x / DL) * (DL + 1) + x % DL] = t.sup[(b * t.NS + h0) * DL + x];
        __syncthreads();
        if (live) {
            for (int hh = 0; hh < nh; ++hh) {
                const float* s = tile + hh * (DL + 1);
                double acc = 0.0;
#pragma unroll 16
                for (int i = 0; i < DL; ++i) acc = __fma_rn((double)c[i], (double)s[i], acc);
                if (acc > best) {                    // ties keep the lower h
                    best = acc;
                    bh = (int)(h0 + hh);
                }
            }
        }
    }
    asg_s[threadIdx.x] = live ? bh : -1;
    __syncthreads();
    if (threadIdx.x == 0) {
        // ranks among this CTA's buckets of the same super-bucket, in bucket order
        int32_t* hist = t.hist + (b * gridDim.x + cta) * t.NS;
        for (int64_t h = 0; h < t.NS; ++h) hist[h] = 0;
        for (int j = 0; j < TR_PTS; ++j) {
            const int h = asg_s[j];
            if (h < 0) break;
            t.rank[b * t.NBK + cta * TR_PTS + j] = hist[h]++;
        }
    }
    if (live) t.asg[b * t.NBK + g] = bh;
}

// a thread per super-bucket: per-CTA bases (in place of the counts), then the
// CSR offsets by a block-wide exclusive scan of the totals
__global__ void __launch_bounds__(1024) tree_scan_kernel(TreeView t, int64_t n_cta)
{
    __shared__ int32_t tot_s[1024];
    __shared__ int32_t carry;
    const int64_t b = blockIdx.x;
    int32_t* hist = t.hist + b * n_cta * t.NS;
    if (threadIdx.x == 0) carry = 0;
    for (int64_t h0 = 0; h0 < t.NS; h0 += blockDim.x) {
        const int64_t h = h0 + threadIdx.x;
        int32_t tot = 0;
        if (h < t.NS) {
            for (int64_t c = 0; c < n_cta; ++c) {
                const int32_t n = hist[c * t.NS + h];
                hist[c * t.NS + h] = tot;            // base of CTA c inside super-bucket h
                tot += n;
            }
        }
        tot_s[threadIdx.x] = tot;
        __syncthreads();
        if (threadIdx.x == 0) {
            int32_t run = carry;
            const int n = (int)((t.NS - h0) < blockDim.x ? (t.NS - h0) : blockDim.x);
            for (int x = 0; x < n; ++x) {
                const int32_t v = tot_s[x];
                tot_s[x] = run;
                run += v;
            }
            carry = run;
        }
        __syncthreads();
        if (h < t.NS) t.off[b * (t.NS + 1) + h] = tot_s[threadIdx.x];
        __syncthreads();
    }
    if (threadIdx.x == 0) t.off[b * (t.NS + 1) + t.NS] = carry;
}

__global__ void tree_scatter_kernel(TreeView t, int64_t NB, int64_t n_cta)
{
    const int64_t b = blockIdx.y;
    const int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (g >= NB) return;
    const int h = t.asg[b * t.NBK + g];
    const int64_t c = g / TR_PTS;
    const int32_t at = t.off[b * (t.NS + 1) + h] + t.hist[(b * n_cta + c) * t.NS + h] +
                       t.rank[b * t.NBK + g];
    t.mem[b * t.NBK + at] = (int32_t)g;
}

// a CTA per super-bucket, a thread per dimension: binary64 sum of the member
// centroids in ascending bucket order, norm, write (empty: unchanged)
__global__ void __launch_bounds__(DL) tree_update_kernel(IndexView ix, TreeView t, int last)
{
    __shared__ double v_s[DL];
    __shared__ double nrm_s;
    const int64_t b = blockIdx.y, h = blockIdx.x;
    const int i = threadIdx.x;
    const int32_t o0 = t.off[b * (t.NS + 1) + h], o1 = t.off[b * (t.NS + 1) + h + 1];
    const int32_t* mem = t.mem + b * t.NBK;
    const float* cent = ix.cent + b * ix.NBK * DL;
    double v = 0.0;
    constexpr int U = 8;
    for (int32_t x0 = o0; x0 < o1; x0 += U) {
        float f[U];
#pragma unroll
        for (int u = 0; u < U; ++u)
            f[u] = (x0 + u < o1) ? cent[(int64_t)mem[x0 + u] * DL + i] : 0.f;
#pragma unroll
        for (int u = 0; u < U; ++u)
            if (x0 + u < o1) v = v + (double)f[u];
    }
    v_s[i] = v;
    __syncthreads();
    if (i == 0) {
        double ss = 0.0;
        for (int d = 0; d < DL; ++d) ss = __dadd_rn(ss, __dmul_rn(v_s[d], v_s[d]));
        nrm_s = __dsqrt_rn(ss);
    }
    __syncthreads();
    float* s = t.sup + (b * t.NS + h) * DL;
    if (o1 > o0 && nrm_s != 0.0) s[i] = __double2float_rn(__ddiv_rn(v, nrm_s));
    if (last) {
        __syncthreads();
        const float c = s[i];
        const int64_t x = (b * t.NS + h) * DL + i;
        if (ix.dtype == LSA_BF16) ((__nv_bfloat16*)t.sup_rt)[x] = __float2bfloat16_rn(c);
        else ((float*)t.sup_rt)[x] = c;
    }
}

cudaError_t launch_tree_build(const IndexView& ix, int64_t n_blk, void* buf, int64_t NS, int L,
                              cudaStream_t st)
{
    const int64_t NB = n_blk * ix.k;
    if (NS < 1 || NS > NB || L < 1) return cudaErrorInvalidValue;
    const TreeView t = tree_view(ix, buf, NS);
    const int64_t n_cta = (NB + TR_PTS - 1) / TR_PTS;
    const int smem = TR_TILE * (DL + 1) * 4;
    cudaError_t e = ensure_smem_attr((const void*)tree_assign_kernel, smem);
    if (e != cudaSuccess) return e;
    tree_init_kernel<<<dim3(64, (unsigned)ix.B), 256, 0, st>>>(ix, t, NB);
    note_launch();
    for (int it = 0; it < L; ++it) {
        tree_assign_kernel<<<dim3((unsigned)n_cta, (unsigned)ix.B), TR_PTS, smem, st>>>(ix, t, NB);
        note_launch();
        tree_scan_kernel<<<(unsigned)ix.B, 1024, 0, st>>>(t, n_cta);
        note_launch();
        tree_scatter_kernel<<<dim3((unsigned)((NB + 255) / 256), (unsigned)ix.B), 256, 0, st>>>(
            t, NB, n_cta);
        note_launch();
        tree_update_kernel<<<dim3((unsigned)NS, (unsigned)ix.B), DL, 0, st>>>(ix, t,
                                                                            it == L - 1 ? 1 : 0);
        note_launch();
    }
    return cudaGetLastError();
}

cudaError_t tree_export(const IndexView& ix, const void* buf, int64_t NS, float* sup,
                        void* sup_rt, int32_t* off, int32_t* mem, cudaStream_t st)
{
    const TreeView t = tree_view(ix, const_cast<void*>(buf), NS);
    const size_t es = (ix.dtype == LSA_BF16) ? 2 : 4;
    cudaError_t e = cudaSuccess;
    if (sup) e = cudaMemcpyAsync(sup, t.sup, (size_t)ix.B * NS * DL * 4, cudaMemcpyDeviceToDevice, st);
    if (e == cudaSuccess && sup_rt)
        e = cudaMemcpyAsync(sup_rt, t.sup_rt, (size_t)ix.B * NS * DL * es, cudaMemcpyDeviceToDevice, st);
    if (e == cudaSuccess && off)
        e = cudaMemcpyAsync(off, t.off, (size_t)ix.B * (NS + 1) * 4, cudaMemcpyDeviceToDevice, st);
    if (e == cudaSuccess && mem)
        e = cudaMemcpyAsync(mem, t.mem, (size_t)ix.B * ix.NBK * 4, cudaMemcpyDeviceToDevice, st);
    return e;
}

// Pointers the selection needs (offsets, members, retrieval copy).
void tree_select_arrays(const IndexView& ix, const void* buf, int64_t NS, const void** sup_rt,
                        const int32_t** off, const int32_t** mem)
{
    const TreeView t = tree_view(ix, const_cast<void*>(buf), NS);
    *sup_rt = t.sup_rt;
    *off = t.off;
    *mem = t.mem;
}

}  // namespace lsa
