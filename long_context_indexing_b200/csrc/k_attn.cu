// k_attn.cu -- exact softmax attention over each query's selected keys.
//
// Method: "Prefrontal's Latent Sparse Attention speeds up one attention layer
// 72x at 10M tokens; end to end, the gain is 9x", section "What it changes":
// the attention kernel is unchanged, LSA only decides which keys are read.
// "Latent Sparse Attention: un indice gerarchico per contesti lunghi",
// paragraph on retrieval: attention runs on the selected keys and values; the
// KV cache keeps the original representations.
//
// The selection is shared by every query head; query head h reads KV head
// h / (Hq/Hkv).  Both kernels use an fp32 online softmax.
//
// bf16 kernel (the hot one).  One CTA per (query, KV head), 4 warps; warp w
// takes the 16-key tiles w, w+4, w+8, ... of the query's selection and keeps
// its own online-softmax state; the warps merge at the end.  Each warp owns a
// STAGES-deep ring of K and V tiles filled by per-row bulk copies
// (cp.async.bulk, one per key row of d bf16) into padded shared-memory rows
// (pitch = 2d + 16 bytes, so ldmatrix rows fall in distinct banks), completed
// on one mbarrier per stage.  The logits are computed transposed,
// S^T = K Q^T (keys on the MMA M dimension, the <= 8 heads of the KV group on
// N), so no MMA row is padding; P^T is turned into the B operand of
// O^T = V^T P^T with movmatrix, and V^T comes from ldmatrix.trans.
#include <math.h>

#include "lsa_internal.cuh"
#include "ptx.cuh"

namespace lsa {

constexpr uint32_t WAIT_LIMIT = 1u << 24;

__device__ __forceinline__ int32_t checked_index(int32_t t, int64_t T_cap, uint32_t* status)
{
    if (t < 0 || t >= T_cap) {
        if (status) dev_error(status, DEV_BAD_INDEX, (uint32_t)t);
        return 0;
    }
    return t;
}

// ---------------------------------------------------------------------------
// fp32 kernel: CTA per (query, KV head), 128 threads, 32-key tiles.
// ---------------------------------------------------------------------------
template <int HPG, int D>
__global__ void __launch_bounds__(128) attn_f32_kernel(const float* __restrict__ Q,
                                                       const float* __restrict__ K,
                                                       const float* __restrict__ V, int64_t Nq,
                                                       int64_t T_cap, int Hq, int Hkv,
                                                       const int32_t* __restrict__ indices,
                                                       const int32_t* __restrict__ counts,
                                                       int s_max, float scale, float* O, float* lse,
                                                       uint32_t* status)
{
    constexpr int TK = 32;
    constexpr int PER = (HPG * D + 127) / 128;
    __shared__ float q_s[HPG][D];
    __shared__ float k_s[TK][D + 1];
    __shared__ float v_s[TK][D];
    __shared__ float p_s[HPG][TK];
    __shared__ float alpha_s[HPG];
    __shared__ int32_t t_s[TK];
    const int64_t row = blockIdx.x / Hkv;
    const int g = blockIdx.x % Hkv;
    const int64_t b = row / Nq;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int32_t* idx = indices + row * (int64_t)s_max;
    const int n = min(counts[row], s_max);  // never read past the row
    for (int x = threadIdx.x; x < HPG * D; x += 128)
        q_s[x / D][x % D] = Q[(row * Hq + (int64_t)g * HPG + x / D) * D + x % D];
    float m_h = -INFINITY, l_h = 0.f;  // valid in warp w for heads w, w+4 (lane 0 copy)
    float m_h2 = -INFINITY, l_h2 = 0.f;
    float acc[PER];
#pragma unroll
    for (int e = 0; e < PER; ++e) acc[e] = 0.f;

    for (int t0 = 0; t0 < n; t0 += TK) {
        __syncthreads();
        if (threadIdx.x < TK) {
            const int kk = t0 + threadIdx.x;
            t_s[threadIdx.x] = (kk < n) ? checked_index(idx[kk], T_cap, status) : -1;
        }
        __syncthreads();
        for (int x = threadIdx.x; x < TK * D; x += 128) {
            const int r = x / D, c = x % D;
            const int32_t t = t_s[r];
            float kv = 0.f, vv = 0.f;
            if (t >= 0) {
                const int64_t off = ((b * T_cap + t) * Hkv + g) * D + c;
                kv = K[off];
                vv = V[off];
            }
            k_s[r][c] = kv;
            v_s[r][c] = vv;
        }
        __syncthreads();
        for (int x = threadIdx.x; x < HPG * TK; x += 128) {
            const int h = x / TK, r = x % TK;
            float s = -INFINITY;
            if (t_s[r] >= 0) {
                float a = 0.f;
#pragma unroll 16
                for (int c = 0; c < D; ++c) a = fmaf(q_s[h][c], k_s[r][c], a);
                s = a * scale;
            }
            p_s[h][r] = s;
        }
        __syncthreads();
        for (int h = warp; h < HPG; h += 4) {
            const float s = p_s[h][lane];
            float mx = s;
            for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            const float m_old = (h == warp) ? m_h : m_h2;
            const float m_new = fmaxf(m_old, mx);
            const float alpha = (m_old == -INFINITY) ? 0.f : expf(m_old - m_new);
            const float pv = (s == -INFINITY) ? 0.f : expf(s - m_new);
            float sum = pv;
            for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
            p_s[h][lane] = pv;
            if (h == warp) {
                m_h = m_new;
                l_h = l_h * alpha + sum;
            } else {
                m_h2 = m_new;
                l_h2 = l_h2 * alpha + sum;
            }
            if (lane == 0) alpha_s[h] = alpha;
        }
        __syncthreads();
#pragma unroll
        for (int e = 0; e < PER; ++e) {
            const int x = threadIdx.x + e * 128;
            if (x < HPG * D) {
                const int h = x / D, c = x % D;
                float a = acc[e] * alpha_s[h];
                for (int r = 0; r < TK; ++r) a = fmaf(p_s[h][r], v_s[r][c], a);
                acc[e] = a;
            }
        }
    }
    __syncthreads();
    __shared__ float l_fin[HPG], m_fin[HPG];
    for (int h = warp; h < HPG; h += 4)
        if (lane == 0) {
            l_fin[h] = (h == warp) ? l_h : l_h2;
            m_fin[h] = (h == warp) ? m_h : m_h2;
        }
    __syncthreads();
#pragma unroll
    for (int e = 0; e < PER; ++e) {
        const int x = threadIdx.x + e * 128;
        if (x < HPG * D) {
            const int h = x / D, c = x % D;
            O[(row * Hq + (int64_t)g * HPG + h) * D + c] = acc[e] / l_fin[h];
        }
    }
    if (lse && threadIdx.x < HPG)
        lse[row * Hq + (int64_t)g * HPG + threadIdx.x] =
            m_fin[threadIdx.x] + logf(l_fin[threadIdx.x]);
}

// ---------------------------------------------------------------------------
// bf16 tensor-core kernel.
// ---------------------------------------------------------------------------
constexpr int ATT_WARPS = 4;

template <int D, int STAGES>
struct AttnSmem {
    static constexpr int ROWB = D * 2;            // bytes of one key row of one KV head
    static constexpr int PITCH = ROWB + 16;       // padded shared-memory row
    static constexpr int TILE = 16 * PITCH;       // one 16-key tile of K (or V)
    static constexpr int WARP_BYTES = STAGES * 2 * TILE;
    static constexpr int MERGE_BYTES = ATT_WARPS * 8 * (D + 2) * 4;
    static constexpr int RING = ATT_WARPS * WARP_BYTES;
    static constexpr int BYTES = (RING > MERGE_BYTES ? RING : MERGE_BYTES) + ATT_WARPS * STAGES * 8;
};

template <int D, int STAGES>
__global__ void __launch_bounds__(ATT_WARPS * 32) attn_bf16_kernel(
    const __nv_bfloat16* __restrict__ Q, const __nv_bfloat16* __restrict__ K,
    const __nv_bfloat16* __restrict__ V, int64_t Nq, int64_t T_cap, int Hq, int Hkv, int hpg,
    const int32_t* __restrict__ indices, const int32_t* __restrict__ counts, int s_max,
    float scale_log2, __nv_bfloat16* O, float* lse, uint32_t* status)
{
    using SM = AttnSmem<D, STAGES>;
    constexpr int KSTEPS = D / 16;
    extern __shared__ __align__(128) unsigned char smem[];
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (SM::BYTES - ATT_WARPS * STAGES * 8));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t row = blockIdx.x / Hkv;
    const int g = blockIdx.x % Hkv;
    const int64_t b = row / Nq;
    const int32_t* idx = indices + row * (int64_t)s_max;
    const int n = min(counts[row], s_max);  // never read past the row
    unsigned char* ring = smem + warp * SM::WARP_BYTES;
    uint64_t* wbar = bars + warp * STAGES;

    if (lane == 0)
        for (int s = 0; s < STAGES; ++s) ptx::mbar_init(&wbar[s], 1);
    ptx::fence_mbar_init();
    __syncwarp();

    // Q^T fragments (B operand): head n = lane/4, dims 2*(lane%4) + {0,1} (+8).
    uint32_t qf[KSTEPS][2];
    {
        const int h = lane >> 2;
        const bool live = h < hpg;
        const __nv_bfloat16* qrow = Q + (row * Hq + (int64_t)g * hpg + (live ? h : 0)) * D;
#pragma unroll
        for (int kk = 0; kk < KSTEPS; ++kk) {
            const int c = kk * 16 + 2 * (lane & 3);
            qf[kk][0] = live ? *reinterpret_cast<const uint32_t*>(qrow + c) : 0u;
            qf[kk][1] = live ? *reinterpret_cast<const uint32_t*>(qrow + c + 8) : 0u;
        }
    }

    const int n_tiles = (n + 15) >> 4;
    // tiles of this warp: t = warp + ATT_WARPS * j
    const int my_tiles = (n_tiles > warp) ? (n_tiles - warp + ATT_WARPS - 1) / ATT_WARPS : 0;
    const int32_t last_valid = (n > 0) ? n - 1 : 0;
    bool timed_out = false;

    auto issue = [&](int j) {
        const int s = j % STAGES;
        const int t = warp + ATT_WARPS * j;
        unsigned char* kt = ring + s * 2 * SM::TILE;
        unsigned char* vt = kt + SM::TILE;
        if (lane == 0) ptx::mbar_arrive_expect_tx(&wbar[s], 2u * 16u * SM::ROWB);
        __syncwarp();
        const int r = lane & 15;
        int key = t * 16 + r;
        if (key > last_valid) key = last_valid;
        const int32_t kidx = checked_index(idx[key], T_cap, status);
        const int64_t off = ((b * T_cap + kidx) * Hkv + g) * (int64_t)D;
        if (lane < 16)
            ptx::bulk_g2s(kt + r * SM::PITCH, K + off, SM::ROWB, &wbar[s]);
        else
            ptx::bulk_g2s(vt + r * SM::PITCH, V + off, SM::ROWB, &wbar[s]);
    };

    for (int j = 0; j < STAGES && j < my_tiles; ++j) issue(j);

    float oacc[KSTEPS][4];
#pragma unroll
    for (int mt = 0; mt < KSTEPS; ++mt)
#pragma unroll
        for (int e = 0; e < 4; ++e) oacc[mt][e] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;

    int j_stop = my_tiles;
    for (int j = 0; j < my_tiles; ++j) {
        const int s = j % STAGES;
        const uint32_t parity = (uint32_t)((j / STAGES) & 1);
        if (!ptx::mbar_wait_bounded(&wbar[s], parity, WAIT_LIMIT)) {
            timed_out = true;
            j_stop = j;
            break;
        }
        const unsigned char* kt = ring + s * 2 * SM::TILE;
        const unsigned char* vt = kt + SM::TILE;
        const int t = warp + ATT_WARPS * j;

        // S^T[16 keys][8 heads] = K[16][D] Q^T[D][8]
        float sacc[4] = {0.f, 0.f, 0.f, 0.f};
        {
            const unsigned char* base = kt + (lane & 15) * SM::PITCH + (lane >> 4) * 16;
#pragma unroll
            for (int kk = 0; kk < KSTEPS; ++kk) {
                uint32_t a0, a1, a2, a3;
                ptx::ldsm_x4(a0, a1, a2, a3, base + kk * 32);
                ptx::mma_bf16_16816(sacc, a0, a1, a2, a3, qf[kk][0], qf[kk][1]);
            }
        }
        // online softmax in log2 units; keys beyond n are masked
        const int key_lo = t * 16 + (lane >> 2), key_hi = key_lo + 8;
        float z0 = (key_lo < n) ? sacc[0] * scale_log2 : -INFINITY;
        float z1 = (key_lo < n) ? sacc[1] * scale_log2 : -INFINITY;
        float z2 = (key_hi < n) ? sacc[2] * scale_log2 : -INFINITY;
        float z3 = (key_hi < n) ? sacc[3] * scale_log2 : -INFINITY;
        float tm0 = fmaxf(z0, z2), tm1 = fmaxf(z1, z3);
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
            tm0 = fmaxf(tm0, __shfl_xor_sync(0xffffffffu, tm0, o));
            tm1 = fmaxf(tm1, __shfl_xor_sync(0xffffffffu, tm1, o));
        }
        const float mn0 = fmaxf(m0, tm0), mn1 = fmaxf(m1, tm1);
        const float al0 = (m0 == -INFINITY) ? 0.f : exp2f(m0 - mn0);
        const float al1 = (m1 == -INFINITY) ? 0.f : exp2f(m1 - mn1);
        const float mu0 = (mn0 == -INFINITY) ? 0.f : mn0;
        const float mu1 = (mn1 == -INFINITY) ? 0.f : mn1;
        const float p0 = exp2f(z0 - mu0), p1 = exp2f(z1 - mu1);
        const float p2 = exp2f(z2 - mu0), p3 = exp2f(z3 - mu1);
        m0 = mn0;
        m1 = mn1;
        l0 = l0 * al0 + (p0 + p2);
        l1 = l1 * al1 + (p1 + p3);
#pragma unroll
        for (int mt = 0; mt < KSTEPS; ++mt) {
            oacc[mt][0] *= al0;
            oacc[mt][1] *= al1;
            oacc[mt][2] *= al0;
            oacc[mt][3] *= al1;
        }
        // P^T (C layout) -> B operand of O^T = V^T P^T
        const uint32_t pb0 = ptx::movmatrix_t(ptx::pack_bf16(p0, p1));
        const uint32_t pb1 = ptx::movmatrix_t(ptx::pack_bf16(p2, p3));
        {
            const int mi = lane >> 3, r = lane & 7;
            const unsigned char* base = vt + (r + 8 * (mi >> 1)) * SM::PITCH + (mi & 1) * 16;
#pragma unroll
            for (int mt = 0; mt < KSTEPS; ++mt) {
                uint32_t a0, a1, a2, a3;
                ptx::ldsm_x4_t(a0, a1, a2, a3, base + mt * 32);
                ptx::mma_bf16_16816(oacc[mt], a0, a1, a2, a3, pb0, pb1);
            }
        }
        __syncwarp();
        if (j + STAGES < my_tiles) issue(j + STAGES);
    }

    // After a timeout, give the copies this warp still has in flight a
    // bounded chance to land before the ring is reused.
    if (timed_out)
        for (int j = j_stop; j < my_tiles && j < j_stop + STAGES; ++j)
            ptx::mbar_wait_bounded(&wbar[j % STAGES], (uint32_t)((j / STAGES) & 1), WAIT_LIMIT);

    // reduce l over the lanes sharing the same heads
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
        l0 += __shfl_xor_sync(0xffffffffu, l0, o);
        l1 += __shfl_xor_sync(0xffffffffu, l1, o);
    }
    __syncthreads();  // every warp is done with its ring: reuse it for the merge
    float* mw = reinterpret_cast<float*>(smem);            // [ATT_WARPS][8]
    float* lw = mw + ATT_WARPS * 8;                         // [ATT_WARPS][8]
    float* ow = lw + ATT_WARPS * 8;                         // [ATT_WARPS][8][D]
    if (lane < 4) {
        mw[warp * 8 + 2 * lane] = m0;
        mw[warp * 8 + 2 * lane + 1] = m1;
        lw[warp * 8 + 2 * lane] = l0;
        lw[warp * 8 + 2 * lane + 1] = l1;
    }
    {
        const int h0 = 2 * (lane & 3), dr = lane >> 2;
#pragma unroll
        for (int mt = 0; mt < KSTEPS; ++mt) {
            float* o = ow + (warp * 8) * D;
            o[h0 * D + mt * 16 + dr] = oacc[mt][0];
            o[(h0 + 1) * D + mt * 16 + dr] = oacc[mt][1];
            o[h0 * D + mt * 16 + dr + 8] = oacc[mt][2];
            o[(h0 + 1) * D + mt * 16 + dr + 8] = oacc[mt][3];
        }
    }
    __shared__ int any_timeout;
    if (threadIdx.x == 0) any_timeout = 0;
    __syncthreads();
    if (timed_out) any_timeout = 1;
    __syncthreads();
    if (any_timeout && threadIdx.x == 0 && status) dev_error(status, DEV_TIMEOUT, (uint32_t)row);
    for (int x = threadIdx.x; x < hpg * D; x += ATT_WARPS * 32) {
        const int h = x / D, c = x % D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < ATT_WARPS; ++w) M = fmaxf(M, mw[w * 8 + h]);
        float L = 0.f, acc = 0.f;
#pragma unroll
        for (int w = 0; w < ATT_WARPS; ++w) {
            const float sc = (mw[w * 8 + h] == -INFINITY) ? 0.f : exp2f(mw[w * 8 + h] - M);
            L += lw[w * 8 + h] * sc;
            acc += ow[(w * 8 + h) * D + c] * sc;
        }
        float o = acc / L;
        if (any_timeout) o = __int_as_float(0x7fc00000);
        O[(row * Hq + (int64_t)g * hpg + h) * D + c] = __float2bfloat16_rn(o);
        if (c == 0 && lse) {
            float v = (M + log2f(L)) * 0.69314718055994531f;
            if (any_timeout) v = __int_as_float(0x7fc00000);
            lse[row * Hq + (int64_t)g * hpg + h] = v;
        }
    }
}

template <int D, int STAGES>
static cudaError_t launch_bf16(const void* Q, const void* K, const void* V, int64_t B, int64_t Nq,
                               int64_t T_cap, int Hq, int Hkv, const int32_t* indices,
                               const int32_t* counts, int s_max, float scale, void* O, float* lse,
                               uint32_t* status, cudaStream_t st)
{
    using SM = AttnSmem<D, STAGES>;
    auto kern = attn_bf16_kernel<D, STAGES>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SM::BYTES);
    if (e != cudaSuccess) return e;
    const int64_t ctas = B * Nq * Hkv;
    kern<<<(unsigned)ctas, ATT_WARPS * 32, SM::BYTES, st>>>(
        (const __nv_bfloat16*)Q, (const __nv_bfloat16*)K, (const __nv_bfloat16*)V, Nq, T_cap, Hq,
        Hkv, Hq / Hkv, indices, counts, s_max, scale * 1.4426950408889634f, (__nv_bfloat16*)O, lse,
        status);
    return cudaGetLastError();
}

template <int HPG, int D>
static cudaError_t launch_f32(const void* Q, const void* K, const void* V, int64_t B, int64_t Nq,
                              int64_t T_cap, int Hq, int Hkv, const int32_t* indices,
                              const int32_t* counts, int s_max, float scale, void* O, float* lse,
                              uint32_t* status, cudaStream_t st)
{
    const int64_t ctas = B * Nq * Hkv;
    attn_f32_kernel<HPG, D><<<(unsigned)ctas, 128, 0, st>>>(
        (const float*)Q, (const float*)K, (const float*)V, Nq, T_cap, Hq, Hkv, indices, counts,
        s_max, scale, (float*)O, lse, status);
    return cudaGetLastError();
}

cudaError_t launch_attn_status(const void* Q, const void* K, const void* V, lsa_dtype dt, int64_t B,
                               int64_t Nq, int64_t T_cap, int Hq, int Hkv, int d,
                               const int32_t* indices, const int32_t* counts, int s_max, float scale,
                               void* O, float* lse, uint32_t* status, cudaStream_t st)
{
    if (B * Nq == 0) return cudaSuccess;
    const int hpg = Hq / Hkv;
    if (dt == LSA_BF16) {
        if (d == 128) return launch_bf16<128, 3>(Q, K, V, B, Nq, T_cap, Hq, Hkv, indices, counts,
                                                 s_max, scale, O, lse, status, st);
        return launch_bf16<64, 4>(Q, K, V, B, Nq, T_cap, Hq, Hkv, indices, counts, s_max, scale, O,
                                  lse, status, st);
    }
#define LSA_F32_CASE(H, DD)                                                                      \
    if (hpg == H && d == DD)                                                                     \
        return launch_f32<H, DD>(Q, K, V, B, Nq, T_cap, Hq, Hkv, indices, counts, s_max, scale, O, \
                                 lse, status, st);
    LSA_F32_CASE(1, 64)
    LSA_F32_CASE(2, 64)
    LSA_F32_CASE(4, 64)
    LSA_F32_CASE(8, 64)
    LSA_F32_CASE(1, 128)
    LSA_F32_CASE(2, 128)
    LSA_F32_CASE(4, 128)
    LSA_F32_CASE(8, 128)
#undef LSA_F32_CASE
    return cudaErrorInvalidValue;
}

cudaError_t launch_attn(const void* Q, const void* K, const void* V, lsa_dtype dt, int64_t B,
                        int64_t Nq, int64_t T_cap, int Hq, int Hkv, int d,
                        const int32_t* indices, const int32_t* counts, int s_max, float scale,
                        void* O, float* lse, cudaStream_t st)
{
    return launch_attn_status(Q, K, V, dt, B, Nq, T_cap, Hq, Hkv, d, indices, counts, s_max, scale,
                              O, lse, nullptr, st);
}

}  // namespace lsa
