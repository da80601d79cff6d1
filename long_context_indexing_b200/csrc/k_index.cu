// k_index.cu -- content index kernels (pooling, spherical k-means, CSR,
// open-block assignment).
//
// Method: "Latent Sparse Attention: un indice gerarchico per contesti
// lunghi", paragraph on index construction: consecutive keys are pooled in
// small groups, the pooled sequence is cut into blocks and, inside each block,
// similar representations are grouped into buckets that keep a centroid and
// the indices of the original keys.
//
// Reproducibility: every decision (assignment argmax, centroid bits) is made
// on exactly the values a sequential binary64 evaluation produces:
//   * pooling sums the p rows left to right with __fadd_rn and divides with
//     __fdiv_rn (binary32);
//   * dot products of binary32 data use __fma_rn in binary64 in ascending
//     dimension; a product of two binary32 values is exact in binary64, so
//     each step is "exact product, then one rounding of the sum";
//   * sums of binary64 values (centroid norms) use __dmul_rn then __dadd_rn,
//     never a contracted FMA;
//   * sqrt and division are the correctly rounded __dsqrt_rn / __ddiv_rn.
#include "lsa_internal.cuh"

namespace lsa {

// ---------------------------------------------------------------------------
// Pool + normalise.  One warp per 32 consecutive pooled groups.
//   phase 1 x = (((r0 + r1) + r2) + ...) / p, writes pooled: bf16 rows with
//            p in {1, 2, 4, 8} are read as one contiguous run per group with
//            16-byte lanes and summed after shuffles; otherwise lanes =
//            dimension pairs;
//   phase 2 (lane = group): ss = sum_i x_i^2 in ascending i (binary64),
//            nrm = sqrt(ss);
//   phase 3 (lanes = dimension pairs): u_i = x_i / nrm, writes unit.
// ---------------------------------------------------------------------------
constexpr int POOL_WARPS = 4;

// P > 0: bf16 rows with P rows per group (vectorised path); P = 0: any dtype
// and pool size.
template <typename T, int P>
__global__ void __launch_bounds__(POOL_WARPS * 32) pool_unit_kernel(IndexView ix,
                                                                    const T* __restrict__ lat,
                                                                    int64_t j0, int64_t j1)
{
    __shared__ float xs[POOL_WARPS][32][DL + 1];
    __shared__ double nrm_s[POOL_WARPS][32];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t b = blockIdx.y;
    const int64_t jw = j0 + ((int64_t)blockIdx.x * POOL_WARPS + warp) * 32;
    if (jw >= j1) return;
    const int n = (int)((j1 - jw) < 32 ? (j1 - jw) : 32);
    const int p = ix.p;
    const T* seq = lat + b * ix.T_cap * DL;
    float* pooled = ix.pooled + b * ix.NP * DL;
    float* unit = ix.unit + b * ix.NP * DL;

    if (P > 0) {
        // bf16 rows, P rows per group: the group's P consecutive 128-byte rows
        // are one contiguous run, read with 16-byte lanes (8 lanes per row),
        // four groups' loads in flight; lane L < 8 then gathers dimensions
        // 8L .. 8L+7 of rows 0 .. P-1 by shuffles and sums them in row order
        constexpr int CH = P * 8;                   // 16-byte chunks per group
        constexpr int NU = (CH + 31) / 32 > 0 ? (CH + 31) / 32 : 1;   // loads per lane per group
        constexpr int GU = 4;                       // groups per batch
        const int L = lane & 7;
        for (int g0 = 0; g0 < n; g0 += GU) {
            uint4 v[GU][NU];
#pragma unroll
            for (int gg = 0; gg < GU; ++gg) {
                const uint4* src = reinterpret_cast<const uint4*>(seq + (jw + g0 + gg) * P * DL);
#pragma unroll
                for (int u = 0; u < NU; ++u) {
                    const int c = lane + 32 * u;
                    v[gg][u] = (g0 + gg < n && c < CH) ? __ldg(src + c) : make_uint4(0u, 0u, 0u, 0u);
                }
            }
#pragma unroll
            for (int gg = 0; gg < GU; ++gg) {
                float sacc[8];
#pragma unroll
                for (int r = 0; r < P; ++r) {
                    const uint4 w = v[gg][r / 4];
                    const int srcl = (r % 4) * 8 + L;
                    uint4 y;
                    y.x = __shfl_sync(0xffffffffu, w.x, srcl);
                    y.y = __shfl_sync(0xffffffffu, w.y, srcl);
                    y.z = __shfl_sync(0xffffffffu, w.z, srcl);
                    y.w = __shfl_sync(0xffffffffu, w.w, srcl);
                    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&y);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 f = __bfloat1622float2(h[e]);
                        if (r == 0) {
                            sacc[2 * e] = f.x;
                            sacc[2 * e + 1] = f.y;
                        } else {
                            sacc[2 * e] = __fadd_rn(sacc[2 * e], f.x);
                            sacc[2 * e + 1] = __fadd_rn(sacc[2 * e + 1], f.y);
                        }
                    }
                }
                const int g = g0 + gg;
                if (lane < 8 && g < n) {
                    const float fp = (float)P;
                    float xv[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        xv[e] = __fdiv_rn(sacc[e], fp);
                        xs[warp][g][8 * L + e] = xv[e];
                    }
                    float4* dst = reinterpret_cast<float4*>(pooled + (jw + g) * DL + 8 * L);
                    dst[0] = make_float4(xv[0], xv[1], xv[2], xv[3]);
                    dst[1] = make_float4(xv[4], xv[5], xv[6], xv[7]);
                }
            }
        }
    } else {
        for (int g = 0; g < n; ++g) {
            const int64_t j = jw + g;
            const T* row = seq + (j * p) * DL;
            float s0 = load_elt(row + 2 * lane), s1 = load_elt(row + 2 * lane + 1);
            for (int r = 1; r < p; ++r) {
                s0 = __fadd_rn(s0, load_elt(row + (int64_t)r * DL + 2 * lane));
                s1 = __fadd_rn(s1, load_elt(row + (int64_t)r * DL + 2 * lane + 1));
            }
            const float fp = (float)p;
            const float x0 = __fdiv_rn(s0, fp), x1 = __fdiv_rn(s1, fp);
            *reinterpret_cast<float2*>(pooled + j * DL + 2 * lane) = make_float2(x0, x1);
            xs[warp][g][2 * lane] = x0;
            xs[warp][g][2 * lane + 1] = x1;
        }
    }
    __syncwarp();
    if (lane < n) {
        double ss = 0.0;
#pragma unroll 8
        for (int i = 0; i < DL; ++i) {
            const double xi = (double)xs[warp][lane][i];
            ss = __fma_rn(xi, xi, ss);  // exact product, one rounding of the sum
        }
        nrm_s[warp][lane] = __dsqrt_rn(ss);
    }
    __syncwarp();
    for (int g = 0; g < n; ++g) {
        const int64_t j = jw + g;
        const double nr = nrm_s[warp][g];
        float u0 = 0.f, u1 = 0.f;
        if (nr != 0.0) {
            u0 = __double2float_rn(__ddiv_rn((double)xs[warp][g][2 * lane], nr));
            u1 = __double2float_rn(__ddiv_rn((double)xs[warp][g][2 * lane + 1], nr));
        }
        *reinterpret_cast<float2*>(unit + j * DL + 2 * lane) = make_float2(u0, u1);
    }
}

cudaError_t launch_pool_unit(const IndexView& ix, const void* latent_K, int64_t j0, int64_t j1,
                             cudaStream_t st)
{
    if (j1 <= j0) return cudaSuccess;
    const int64_t groups = j1 - j0;
    const int per_cta = POOL_WARPS * 32;
    dim3 grid((unsigned)((groups + per_cta - 1) / per_cta), (unsigned)ix.B);
    if (ix.dtype == LSA_BF16) {
        typedef __nv_bfloat16 B;
        const B* lk = (const B*)latent_K;
        switch (ix.p) {
        case 1: pool_unit_kernel<B, 1><<<grid, per_cta, 0, st>>>(ix, lk, j0, j1); break;
        case 2: pool_unit_kernel<B, 2><<<grid, per_cta, 0, st>>>(ix, lk, j0, j1); break;
        case 4: pool_unit_kernel<B, 4><<<grid, per_cta, 0, st>>>(ix, lk, j0, j1); break;
        case 8: pool_unit_kernel<B, 8><<<grid, per_cta, 0, st>>>(ix, lk, j0, j1); break;
        default: pool_unit_kernel<B, 0><<<grid, per_cta, 0, st>>>(ix, lk, j0, j1); break;
        }
    } else {
        pool_unit_kernel<float, 0><<<grid, per_cta, 0, st>>>(ix, (const float*)latent_K, j0, j1);
    }
    note_launch();
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// k-means assign.  CTA = 128 pooled groups of one block (blockIdx.x = block
// offset * splits + split).  Centroids of the block in shared memory; each
// thread holds its unit vector in registers and evaluates <u, c_m> for
// m = 0..k-1 in binary64 (ascending dimension), argmax with ties to the
// lowest m.  With init != 0 the centroids are the evenly spaced rows
// u[bG + floor(m*G/k)], and split 0 also stores them as the current centroids.
// ---------------------------------------------------------------------------
constexpr int ASSIGN_THREADS = 128;

__global__ void __launch_bounds__(ASSIGN_THREADS) kmeans_assign_kernel(IndexView ix, int64_t b0,
                                                                       int splits, int init)
{
    __shared__ float cs[MAX_K][DL];
    __shared__ float us[ASSIGN_THREADS][DL + 1];
    const int64_t bseq = blockIdx.y;
    const int64_t blk = b0 + blockIdx.x / splits;
    const int split = blockIdx.x % splits;
    const int G = ix.G, k = ix.k;
    const float* unit = ix.unit + bseq * ix.NP * DL;
    float* cent = ix.cent + bseq * ix.NBK * DL;
    const int64_t jb = blk * G;  // first pooled id of the block

    for (int x = threadIdx.x; x < k * DL; x += ASSIGN_THREADS) {
        const int m = x / DL, i = x % DL;
        float c;
        if (init) {
            const int64_t src = jb + ((int64_t)m * G) / k;
            c = unit[src * DL + i];
            if (split == 0) cent[(blk * k + m) * DL + i] = c;
        } else {
            c = cent[(blk * k + m) * DL + i];
        }
        cs[m][i] = c;
    }
    const int j_lo = split * ASSIGN_THREADS;
    const int nj = min(ASSIGN_THREADS, G - j_lo);
    for (int x = threadIdx.x; x < nj * DL; x += ASSIGN_THREADS) {
        const int r = x / DL, i = x % DL;
        us[r][i] = unit[(jb + j_lo + r) * DL + i];
    }
    __syncthreads();
    if ((int)threadIdx.x >= nj) return;
    float u[DL];
#pragma unroll
    for (int i = 0; i < DL; ++i) u[i] = us[threadIdx.x][i];
    double best = -INFINITY;
    int bm = 0;
    // Two independent ascending chains at a time (ILP); each chain is the
    // sequential binary64 sum of exact products.
    for (int m = 0; m < k; m += 2) {
        const int m2 = (m + 1 < k) ? m + 1 : m;
        double s = 0.0, s2 = 0.0;
#pragma unroll
        for (int i = 0; i < DL; ++i) {
            s = __fma_rn((double)u[i], (double)cs[m][i], s);
            s2 = __fma_rn((double)u[i], (double)cs[m2][i], s2);
        }
        if (s > best) {
            best = s;
            bm = m;
        }
        if (m2 != m && s2 > best) {
            best = s2;
            bm = m2;
        }
    }
    ix.assign[bseq * ix.NP + jb + j_lo + threadIdx.x] = (int16_t)bm;
}

// ---------------------------------------------------------------------------
// k-means update (+ CSR and retrieval copy on the last iteration).
// CTA = one block, 1024 threads.
//   1. stable counting sort of the block's assignments: warp w < k walks the
//      G assignments in order with ballots, so members come out ascending;
//   2. thread (m, i): v_mi = sum over members of u_j[i], ascending j
//      (binary64 __dadd_rn);
//   3. thread m: ss = sum_i v_mi * v_mi ascending (__dmul_rn, __dadd_rn),
//      nrm = sqrt(ss);
//   4. thread (m, i): c_mi = binary32(v_mi / nrm) unless the bucket is empty
//      or nrm == 0 (then the centroid is kept).
// ---------------------------------------------------------------------------
constexpr int UPDATE_THREADS = 1024;
constexpr int MAX_G = 4096;

__global__ void __launch_bounds__(UPDATE_THREADS) kmeans_update_kernel(IndexView ix, int64_t b0,
                                                                       int last)
{
    __shared__ int16_t mem_s[MAX_G];
    __shared__ int cnt_s[MAX_K];
    __shared__ int off_s[MAX_K + 1];
    __shared__ double v_s[MAX_K][DL];
    __shared__ double nrm_s[MAX_K];
    const int64_t bseq = blockIdx.y;
    const int64_t blk = b0 + blockIdx.x;
    const int G = ix.G, k = ix.k;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int16_t* assign = ix.assign + bseq * ix.NP + blk * G;
    const float* unit = ix.unit + bseq * ix.NP * DL;
    float* cent = ix.cent + bseq * ix.NBK * DL;
    const int64_t jb = blk * G;

    // 1. counts
    for (int m = warp; m < k; m += UPDATE_THREADS / 32) {
        int c = 0;
        for (int j = lane; j < G; j += 32) c += (assign[j] == m);
        for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
        if (lane == 0) cnt_s[m] = c;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int acc = 0;
        for (int m = 0; m < k; ++m) {
            off_s[m] = acc;
            acc += cnt_s[m];
        }
        off_s[k] = acc;
    }
    __syncthreads();
    // stable placement (ascending j inside each bucket)
    for (int m = warp; m < k; m += UPDATE_THREADS / 32) {
        int base = off_s[m];
        for (int j0 = 0; j0 < G; j0 += 32) {
            const int j = j0 + lane;
            const bool hit = (j < G) && (assign[j] == m);
            const unsigned bal = __ballot_sync(0xffffffffu, hit);
            if (hit) mem_s[base + __popc(bal & ((1u << lane) - 1u))] = (int16_t)j;
            base += __popc(bal);
        }
    }
    __syncthreads();

    // 2. member sums
    for (int x = threadIdx.x; x < k * DL; x += UPDATE_THREADS) {
        const int m = x / DL, i = x % DL;
        double v = 0.0;
        for (int e = off_s[m]; e < off_s[m + 1]; ++e)
            v = __dadd_rn(v, (double)unit[(jb + mem_s[e]) * DL + i]);
        v_s[m][i] = v;
    }
    __syncthreads();
    // 3. norms
    if ((int)threadIdx.x < k) {
        const int m = threadIdx.x;
        double ss = 0.0;
        for (int i = 0; i < DL; ++i) ss = __dadd_rn(ss, __dmul_rn(v_s[m][i], v_s[m][i]));
        nrm_s[m] = __dsqrt_rn(ss);
    }
    __syncthreads();
    // 4. centroids (+ retrieval copy)
    for (int x = threadIdx.x; x < k * DL; x += UPDATE_THREADS) {
        const int m = x / DL, i = x % DL;
        const int64_t gi = (blk * k + m) * DL + i;
        float c = cent[gi];
        if (cnt_s[m] > 0 && nrm_s[m] != 0.0) {
            c = __double2float_rn(__ddiv_rn(v_s[m][i], nrm_s[m]));
            cent[gi] = c;
        }
        if (last) {
            if (ix.dtype == LSA_BF16)
                ((__nv_bfloat16*)ix.cent_rt)[bseq * ix.NBK * DL + gi] = __float2bfloat16_rn(c);
            else
                ((float*)ix.cent_rt)[bseq * ix.NBK * DL + gi] = c;
        }
    }
    if (last) {
        int32_t* offsets = ix.offsets + bseq * (ix.NBK + 1);
        int32_t* members = ix.members + bseq * ix.NP;
        for (int m = threadIdx.x; m <= k; m += UPDATE_THREADS)
            offsets[blk * k + m] = (int32_t)(jb + off_s[m]);
        for (int e = threadIdx.x; e < G; e += UPDATE_THREADS)
            members[jb + e] = (int32_t)(jb + mem_s[e]);
    }
}

cudaError_t launch_kmeans(const IndexView& ix, int64_t b0, int64_t b1, cudaStream_t st)
{
    if (b1 <= b0) return cudaSuccess;
    const int64_t nb = b1 - b0;
    const int splits = (ix.G + ASSIGN_THREADS - 1) / ASSIGN_THREADS;
    for (int it = 0; it < ix.L; ++it) {
        kmeans_assign_kernel<<<dim3((unsigned)(nb * splits), (unsigned)ix.B), ASSIGN_THREADS, 0,
                               st>>>(ix, b0, splits, it == 0);
        note_launch();
        kmeans_update_kernel<<<dim3((unsigned)nb, (unsigned)ix.B), UPDATE_THREADS, 0, st>>>(
            ix, b0, it == ix.L - 1);
        note_launch();
    }
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Open block: CTA per open slot o (blockIdx.x) and sequence (blockIdx.y).
// Slots below n_done get the nearest closed centroid (exact binary64 score,
// ties to the lowest g); the others are reset to -1.
// ---------------------------------------------------------------------------
__device__ __forceinline__ bool better(double s, int g, double bs, int bg)
{
    return s > bs || (s == bs && g < bg);
}

__global__ void __launch_bounds__(256) open_assign_kernel(IndexView ix, int64_t n_blk,
                                                          int64_t n_done)
{
    __shared__ float u_s[DL];
    __shared__ double rs[8];
    __shared__ int rg[8];
    const int64_t bseq = blockIdx.y;
    const int o = blockIdx.x;
    int32_t* open = ix.open_bucket + bseq * ix.G;
    if (o >= n_done) {
        if (threadIdx.x == 0) open[o] = -1;
        return;
    }
    const int64_t j = n_blk * ix.G + o;
    if (threadIdx.x < DL) u_s[threadIdx.x] = ix.unit[(bseq * ix.NP + j) * DL + threadIdx.x];
    __syncthreads();
    const float* cent = ix.cent + bseq * ix.NBK * DL;
    const int64_t nb = n_blk * ix.k;
    double bs = -INFINITY;
    int bg = 0x7fffffff;
    for (int64_t g = threadIdx.x; g < nb; g += 256) {
        const float* c = cent + g * DL;
        double s = 0.0;
#pragma unroll 16
        for (int i = 0; i < DL; ++i) s = __fma_rn((double)u_s[i], (double)c[i], s);
        if (better(s, (int)g, bs, bg)) {
            bs = s;
            bg = (int)g;
        }
    }
    for (int off = 16; off > 0; off >>= 1) {
        const double os = __shfl_xor_sync(0xffffffffu, bs, off);
        const int og = __shfl_xor_sync(0xffffffffu, bg, off);
        if (better(os, og, bs, bg)) {
            bs = os;
            bg = og;
        }
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) {
        rs[warp] = bs;
        rg[warp] = bg;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < 8; ++w)
            if (better(rs[w], rg[w], bs, bg)) {
                bs = rs[w];
                bg = rg[w];
            }
        open[o] = bg;
    }
}

cudaError_t launch_open_assign(const IndexView& ix, int64_t n_blk, int64_t j_end, cudaStream_t st)
{
    const int64_t jo = n_blk * ix.G;
    int64_t n_done = j_end - jo;
    if (n_done < 0) n_done = 0;
    if (n_done > ix.G) n_done = ix.G;
    // the open block holds the pooled groups after the closed blocks, as far
    // as the index's capacity reaches (a partial block when T_cap is not a
    // whole number of blocks)
    if (n_done > ix.NP - jo) n_done = ix.NP - jo;
    if (n_blk == 0 || n_done < 0) n_done = 0;
    open_assign_kernel<<<dim3((unsigned)ix.G, (unsigned)ix.B), 256, 0, st>>>(ix, n_blk, n_done);
    note_launch();
    return cudaGetLastError();
}

}  // namespace lsa
