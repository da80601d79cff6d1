// k_attn_bwd.cu -- gradients of the sparse attention over stored selections.
//
// Method: "Latent Sparse Attention: un indice gerarchico per contesti
// lunghi", paragraph on N-LSA's memory: the selected indices are kept for the
// backward pass.  The attention is softmax attention over each query's
// selected keys, so with z_t = scale <q, k_t>, p_t = exp(z_t - lse) (lse from
// the forward pass) and an upstream gradient dO:
//   D = <dO, O>,  dP_t = <dO, v_t>,  dS_t = p_t (dP_t - D),
//   dQ = scale sum_t dS_t k_t,  dK_t += scale dS_t q,  dV_t += p_t dO.
//
// One CTA per (query row, KV head): the group's query heads, their dO rows
// and D in shared memory; the row's keys in tiles of 32 (K and V rows of the
// KV head, fp32 in shared memory).  Per tile: z, dP, p and dS for every
// (head, key); dQ accumulates in registers; the tile's dK and dV rows, summed
// over the group's heads, are added to fp32 accumulators with atomics (keys
// read by several queries receive several additions, in no fixed order).
#include <math.h>

#include "lsa_internal.cuh"

namespace lsa {

constexpr int BW_THREADS = 128;
constexpr int BW_TK = 32;          // keys per tile
constexpr int BW_MAX_D = 128;
constexpr int BW_MAX_HPG = 8;
constexpr int BW_QPT = BW_MAX_HPG * BW_MAX_D / BW_THREADS;   // (head, dim) pairs per thread

__device__ __forceinline__ float bw_load(const float* p) { return *p; }
__device__ __forceinline__ float bw_load(const __nv_bfloat16* p) { return __bfloat162float(*p); }
__device__ __forceinline__ void bw_store(float* p, float v) { *p = v; }
__device__ __forceinline__ void bw_store(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }

template <typename T>
__global__ void __launch_bounds__(BW_THREADS) attn_backward_kernel(
    const T* __restrict__ Q, const T* __restrict__ K, const T* __restrict__ V,
    const T* __restrict__ O, const float* __restrict__ lse, const T* __restrict__ dO, int64_t Nq,
    int64_t T_cap, int Hq, int Hkv, int d, const int32_t* __restrict__ indices,
    const int32_t* __restrict__ counts, int s_max, float scale, T* dQ, float* dK, float* dV,
    uint32_t* status)
{
    __shared__ float q_s[BW_MAX_HPG][BW_MAX_D];
    __shared__ float g_s[BW_MAX_HPG][BW_MAX_D];        // dO
    __shared__ float k_s[BW_TK][BW_MAX_D + 1];
    __shared__ float v_s[BW_TK][BW_MAX_D + 1];
    __shared__ float p_s[BW_MAX_HPG][BW_TK];
    __shared__ float ds_s[BW_MAX_HPG][BW_TK];
    __shared__ float D_s[BW_MAX_HPG], L_s[BW_MAX_HPG];
    __shared__ int32_t t_s[BW_TK];
    const int hpg = Hq / Hkv;
    const int64_t row = blockIdx.x / Hkv;
    const int g = blockIdx.x % Hkv;
    const int64_t b = row / Nq;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t hbase = row * Hq + (int64_t)g * hpg;             // first query head of the group
    for (int x = threadIdx.x; x < hpg * d; x += BW_THREADS) {
        const int h = x / d, c = x % d;
        q_s[h][c] = bw_load(Q + (hbase + h) * d + c);
        g_s[h][c] = bw_load(dO + (hbase + h) * d + c);
    }
    __syncthreads();
    // D = <dO, O> per head (a warp per head), the forward's lse
    for (int h = warp; h < hpg; h += BW_THREADS / 32) {
        float s = 0.f;
        for (int c = lane; c < d; c += 32) s += g_s[h][c] * bw_load(O + (hbase + h) * d + c);
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (lane == 0) {
            D_s[h] = s;
            L_s[h] = lse[hbase + h];
        }
    }
    float dq[BW_QPT];
#pragma unroll
    for (int j = 0; j < BW_QPT; ++j) dq[j] = 0.f;
    const int32_t* idx = indices + row * (int64_t)s_max;
    const int n = min(counts[row], s_max);
    for (int k0 = 0; k0 < n; k0 += BW_TK) {
        __syncthreads();                       // the previous tile is consumed
        if (threadIdx.x < BW_TK) {
            const int kk = k0 + threadIdx.x;
            int32_t t = -1;
            if (kk < n) {
                t = idx[kk];
                if (t < 0 || t >= T_cap) {
                    if (status) dev_error(status, DEV_BAD_INDEX, (uint32_t)t);
                    t = -1;
                }
            }
            t_s[threadIdx.x] = t;
        }
        __syncthreads();
        for (int x = threadIdx.x; x < BW_TK * d; x += BW_THREADS) {
            const int r = x / d, c = x % d;
            const int32_t t = t_s[r];
            float kv = 0.f, vv = 0.f;
            if (t >= 0) {
                const int64_t off = ((b * T_cap + t) * Hkv + g) * d + c;
                kv = bw_load(K + off);
                vv = bw_load(V + off);
            }
            k_s[r][c] = kv;
            v_s[r][c] = vv;
        }
        __syncthreads();
        // p and dS of every (head, key) of the tile
        for (int x = threadIdx.x; x < hpg * BW_TK; x += BW_THREADS) {
            const int h = x / BW_TK, r = x % BW_TK;
            float p = 0.f, ds = 0.f;
            if (t_s[r] >= 0) {
                float z = 0.f, dp = 0.f;
                for (int c = 0; c < d; ++c) {
                    z = fmaf(q_s[h][c], k_s[r][c], z);
                    dp = fmaf(g_s[h][c], v_s[r][c], dp);
                }
                p = expf(z * scale - L_s[h]);
                ds = p * (dp - D_s[h]);
            }
            p_s[h][r] = p;
            ds_s[h][r] = ds;
        }
        __syncthreads();
        // dQ: this thread's (head, dim) pairs
#pragma unroll
        for (int j = 0; j < BW_QPT; ++j) {
            const int e = threadIdx.x + BW_THREADS * j;
            if (e < hpg * d) {
                const int h = e / d, c = e % d;
                float a = dq[j];
                for (int r = 0; r < BW_TK; ++r) a = fmaf(ds_s[h][r], k_s[r][c], a);
                dq[j] = a;
            }
        }
        // dK, dV rows of the tile's keys, summed over the group's heads
        for (int x = threadIdx.x; x < BW_TK * d; x += BW_THREADS) {
            const int r = x / d, c = x % d;
            const int32_t t = t_s[r];
            if (t < 0) continue;
            float gk = 0.f, gv = 0.f;
            for (int h = 0; h < hpg; ++h) {
                gk = fmaf(ds_s[h][r], q_s[h][c], gk);
                gv = fmaf(p_s[h][r], g_s[h][c], gv);
            }
            const int64_t off = ((b * T_cap + t) * Hkv + g) * d + c;
            atomicAdd(dK + off, gk * scale);
            atomicAdd(dV + off, gv);
        }
    }
#pragma unroll
    for (int j = 0; j < BW_QPT; ++j) {
        const int e = threadIdx.x + BW_THREADS * j;
        if (e < hpg * d) {
            const int h = e / d, c = e % d;
            bw_store(dQ + (hbase + h) * d + c, dq[j] * scale);
        }
    }
}

bool attn_backward_supported(int Hq, int Hkv, int d)
{
    return Hkv >= 1 && Hq % Hkv == 0 && Hq / Hkv <= BW_MAX_HPG && d >= 1 && d <= BW_MAX_D;
}

cudaError_t launch_attn_backward(const void* Q, const void* K, const void* V, const void* O,
                                 const float* lse, const void* dO, lsa_dtype dt, int64_t B,
                                 int64_t Nq, int64_t T_cap, int Hq, int Hkv, int d,
                                 const int32_t* indices, const int32_t* counts, int s_max,
                                 float scale, void* dQ, float* dK, float* dV, uint32_t* status,
                                 cudaStream_t st)
{
    const int64_t ctas = B * Nq * Hkv;
    if (ctas <= 0) return cudaSuccess;
    if (dt == LSA_BF16)
        attn_backward_kernel<__nv_bfloat16><<<(unsigned)ctas, BW_THREADS, 0, st>>>(
            (const __nv_bfloat16*)Q, (const __nv_bfloat16*)K, (const __nv_bfloat16*)V,
            (const __nv_bfloat16*)O, lse, (const __nv_bfloat16*)dO, Nq, T_cap, Hq, Hkv, d, indices,
            counts, s_max, scale, (__nv_bfloat16*)dQ, dK, dV, status);
    else
        attn_backward_kernel<float><<<(unsigned)ctas, BW_THREADS, 0, st>>>(
            (const float*)Q, (const float*)K, (const float*)V, (const float*)O, lse,
            (const float*)dO, Nq, T_cap, Hq, Hkv, d, indices, counts, s_max, scale, (float*)dQ,
            dK, dV, status);
    note_launch();
    return cudaGetLastError();
}

}  // namespace lsa
