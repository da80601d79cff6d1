// k_cp.cu -- the KV cache held in shards of whole blocks (context parallel):
// attention over the selected keys that fall in one shard, and the
// LSE-weighted merge of the shards' partial results.
//
// Method: "Latent Sparse Attention: un indice gerarchico per contesti
// lunghi", paragraph on memory: with context parallelism every rank keeps its
// share of the KV cache and a full copy of the bucket index, so every rank
// makes the same selection and reads the selected keys it holds.  The
// attention over the union of the shards' keys is the softmax over all of
// them: with o_r and lse_r the output and log-sum-exp of shard r's keys,
//   o = sum_r exp(lse_r - L) o_r,   L = log sum_r exp(lse_r).
#include <math.h>

#include "lsa_internal.cuh"

namespace lsa {

// ---------------------------------------------------------------------------
// A warp per query row: the row's selected positions inside [lo, hi), in
// their order, as shard-local rows (t - lo), and their count.  Entries past
// the row's count (or -1) are not read.
// ---------------------------------------------------------------------------
constexpr int RF_WARPS = 8;

__global__ void __launch_bounds__(32 * RF_WARPS) range_filter_kernel(
    const int32_t* __restrict__ indices, const int32_t* __restrict__ counts, int64_t rows,
    int s_max, int64_t lo, int64_t hi, int32_t* __restrict__ loc_idx, int32_t* __restrict__ loc_cnt)
{
    const int lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * RF_WARPS + (threadIdx.x >> 5);
    if (row >= rows) return;                         // warp-uniform
    const int32_t* in = indices + row * (int64_t)s_max;
    int32_t* out = loc_idx + row * (int64_t)s_max;
    const int n = min(counts[row], s_max);
    int m = 0;
    for (int x0 = 0; x0 < n; x0 += 32) {
        const int x = x0 + lane;
        const int32_t t = (x < n) ? in[x] : -1;
        const bool keep = t >= 0 && t >= lo && t < hi;
        const unsigned bal = __ballot_sync(0xffffffffu, keep);
        if (keep) out[m + __popc(bal & ((1u << lane) - 1u))] = (int32_t)(t - lo);
        m += __popc(bal);
    }
    if (lane == 0) loc_cnt[row] = m;
}

cudaError_t launch_range_filter(const int32_t* indices, const int32_t* counts, int64_t rows,
                                int s_max, int64_t lo, int64_t hi, int32_t* loc_idx,
                                int32_t* loc_cnt, cudaStream_t st)
{
    if (rows <= 0) return cudaSuccess;
    const unsigned grid = (unsigned)((rows + RF_WARPS - 1) / RF_WARPS);
    range_filter_kernel<<<grid, 32 * RF_WARPS, 0, st>>>(indices, counts, rows, s_max, lo, hi,
                                                        loc_idx, loc_cnt);
    note_launch();
    return cudaGetLastError();
}

// Rows with no key in the shard: output 0 and lse = -inf (what the merge
// weighs with 0), whatever the attention kernel left for an empty row.
template <typename T>
__global__ void __launch_bounds__(256) range_empty_kernel(const int32_t* __restrict__ loc_cnt,
                                                          int64_t rows, int Hq, int d, T* O,
                                                          float* lse)
{
    const int64_t row = blockIdx.x;
    if (row >= rows || loc_cnt[row] != 0) return;           // CTA-uniform
    for (int x = threadIdx.x; x < Hq * d; x += blockDim.x) O[row * Hq * d + x] = (T)0.f;
    for (int h = threadIdx.x; h < Hq; h += blockDim.x) lse[row * Hq + h] = -INFINITY;
}

cudaError_t launch_range_empty(const int32_t* loc_cnt, int64_t rows, int Hq, int d, lsa_dtype dt,
                               void* O, float* lse, cudaStream_t st)
{
    if (rows <= 0) return cudaSuccess;
    if (dt == LSA_BF16)
        range_empty_kernel<__nv_bfloat16><<<(unsigned)rows, 256, 0, st>>>(
            loc_cnt, rows, Hq, d, (__nv_bfloat16*)O, lse);
    else
        range_empty_kernel<float><<<(unsigned)rows, 256, 0, st>>>(loc_cnt, rows, Hq, d, (float*)O,
                                                                  lse);
    note_launch();
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// LSE-weighted merge: a warp per (row, query head).  Lane r < n_parts reads
// part r's log-sum-exp; M = the largest, w_r = exp(lse_r - M) (0 for a part
// without keys, whose output is never read), L = sum w_r.  Every lane then
// sums w_r o_r over the parts for its d/32 dimensions and divides by L.
// ---------------------------------------------------------------------------
constexpr int MP_WARPS = 8;
constexpr int MP_MAX_PARTS = 32;

__device__ __forceinline__ float mp_load(const float* p) { return *p; }
__device__ __forceinline__ float mp_load(const __nv_bfloat16* p) { return __bfloat162float(*p); }
__device__ __forceinline__ void mp_store(float* p, float v) { *p = v; }
__device__ __forceinline__ void mp_store(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }

template <typename T>
__global__ void __launch_bounds__(32 * MP_WARPS) merge_partials_kernel(
    const T* __restrict__ parts, const float* __restrict__ lse_parts, int n_parts, int64_t n_heads,
    int d, T* __restrict__ O, float* lse)
{
    const int lane = threadIdx.x & 31;
    const int64_t wid = (int64_t)blockIdx.x * MP_WARPS + (threadIdx.x >> 5);   // (row, head)
    if (wid >= n_heads) return;                                            // warp-uniform
    const float ls = (lane < n_parts) ? lse_parts[(int64_t)lane * n_heads + wid] : -INFINITY;
    float M = ls;
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    const float w = (ls == -INFINITY) ? 0.f : expf(ls - M);
    float L = w;
    for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
    for (int c = lane; c < d; c += 32) {
        float acc = 0.f;
        for (int r = 0; r < n_parts; ++r) {
            const float wr = __shfl_sync(0xffffffffu, w, r);
            if (wr > 0.f) acc += wr * mp_load(parts + ((int64_t)r * n_heads + wid) * d + c);
        }
        mp_store(O + wid * d + c, (L > 0.f) ? acc / L : 0.f);
    }
    if (lane == 0 && lse) lse[wid] = (L > 0.f) ? M + logf(L) : -INFINITY;
}

cudaError_t launch_merge_partials(const void* parts, const float* lse_parts, lsa_dtype dt,
                                  int n_parts, int64_t rows, int Hq, int d, void* O, float* lse,
                                  cudaStream_t st)
{
    if (n_parts < 1 || n_parts > MP_MAX_PARTS) return cudaErrorInvalidValue;
    const int64_t n = rows * Hq;
    if (n <= 0) return cudaSuccess;
    const unsigned grid = (unsigned)((n + MP_WARPS - 1) / MP_WARPS);
    if (dt == LSA_BF16)
        merge_partials_kernel<__nv_bfloat16><<<grid, 32 * MP_WARPS, 0, st>>>(
            (const __nv_bfloat16*)parts, lse_parts, n_parts, n, d, (__nv_bfloat16*)O, lse);
    else
        merge_partials_kernel<float><<<grid, 32 * MP_WARPS, 0, st>>>(
            (const float*)parts, lse_parts, n_parts, n, d, (float*)O, lse);
    note_launch();
    return cudaGetLastError();
}

}  // namespace lsa
