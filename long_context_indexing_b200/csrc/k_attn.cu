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
// bf16 kernel (the hot one): see the comment above attn_bf16_kernel.  The
// logits are computed transposed, S^T = K Q^T (keys on the MMA M dimension,
// the <= 8 query heads of a KV head on N), so no MMA row is padding; P^T
// becomes the B operand of O^T = V^T P^T through movmatrix, and V^T comes
// from ldmatrix.trans.
#include <math.h>

#include <mutex>

#include "lsa_internal.cuh"
#include "ptx.cuh"

namespace lsa {

constexpr uint32_t WAIT_LIMIT = 1u << 24;

// Polls each bounded wait of the bf16 attention kernel makes before it gives
// up.  A test hook (lsa_set_wait_limit) lowers it to make the waits run out;
// the drain of copies in flight on the way out always allows WAIT_LIMIT.
__device__ uint32_t g_attn_wait = WAIT_LIMIT;

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
//
// CTA = one query row and one group of HG <= 4 KV heads (and one key split
// when split-KV is on).  Warp 4 is the producer: for every stage it copies the
// KT selected keys' rows for the whole head group (HG*d bf16, contiguous in
// the token-major cache) for K and for V with one bulk copy each into padded
// shared-memory rows, completing on the stage's "full" mbarrier.  Warps 0-3
// consume: warp w serves KV head w % HG and the 16-key slice w / HG of every
// stage (KT = 16 * 4 / HG keys per stage), then arrives on the stage's
// "empty" mbarrier.  At the end the warps of each head merge their
// online-softmax states.  With NS > 1 splits, each CTA writes an fp32
// partial (max, sum, unnormalised output) per query head; the last CTA of a
// (row, head group) to finish -- an atomic counter, no waiting -- combines them.
// ---------------------------------------------------------------------------
constexpr int CONS_WARPS = 4;
constexpr int ATT_THREADS = (CONS_WARPS + 1) * 32;

template <int D, int HG, int STAGES>
struct AttnCfg {
    static constexpr int WPG = CONS_WARPS / HG;     // warps per KV head
    static constexpr int KT = 16 * WPG;             // keys per stage
    static constexpr int RB = HG * D * 2;           // bytes of one key's head-group row
    static constexpr int PITCH = RB + 16;           // padded shared-memory row
    static constexpr int TILE = KT * PITCH;         // K (or V) bytes of a stage
    static constexpr int STAGE = 2 * TILE;
    static constexpr int RING = STAGES * STAGE;
    static constexpr int MERGE = CONS_WARPS * 8 * (D + 2) * 4;
    static constexpr int BODY = RING > MERGE ? RING : MERGE;
    static constexpr int BYTES = BODY + 2 * STAGES * 8 + 16;
};

struct SplitKV {
    int ns;              // splits per (row, head group); 1 = off
    int keys_per_split;  // multiple of the stage size
    float* part;         // [rows][ns][Hq][D + 4]  (acc[D], max, sum, pad)
    uint32_t* counter;   // [rows * n_hgroups], zero before the launch
    const int32_t* row_list;   // optional: CTA i serves row row_list[i] ...
    const int32_t* row_count;  // ... for i < *row_count (the rest exit)
};

template <int D, int HG, int STAGES>
__global__ void __launch_bounds__(ATT_THREADS) attn_bf16_kernel(
    const __nv_bfloat16* __restrict__ Q, const __nv_bfloat16* __restrict__ K,
    const __nv_bfloat16* __restrict__ V, int64_t Nq, int64_t T_cap, int Hq, int Hkv, int hpg,
    const int32_t* __restrict__ indices, const int32_t* __restrict__ counts, int s_max,
    float scale_log2, __nv_bfloat16* O, float* lse, uint32_t* status, SplitKV sk)
{
    using C = AttnCfg<D, HG, STAGES>;
    constexpr int KSTEPS = D / 16;
    extern __shared__ __align__(128) unsigned char smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::BODY);
    uint64_t* empty = full + STAGES;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + STAGES);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_hg = Hkv / HG;
    const int64_t unit = blockIdx.x / sk.ns;        // (row, head group)
    const int split = blockIdx.x % sk.ns;
    int64_t row = unit / n_hg;
    if (sk.row_list) {
        if (row >= *sk.row_count) return;   // the whole CTA leaves before any barrier
        row = sk.row_list[row];
    }
    const int g0 = (int)(unit % n_hg) * HG;           // first KV head of the group
    const int64_t b = row / Nq;
    const int32_t* idx = indices + row * (int64_t)s_max;
    const int n_all = min(counts[row], s_max);        // never read past the row
    const int k_lo = split * sk.keys_per_split;
    const int k_hi = min(n_all, k_lo + sk.keys_per_split);
    const int n = max(0, k_hi - k_lo);               // keys of this CTA
    const int n_st = (n + C::KT - 1) / C::KT;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            ptx::mbar_init(&full[s], 1);
            ptx::mbar_init(&empty[s], CONS_WARPS);
        }
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    __syncthreads();

    const uint32_t wl = g_attn_wait;
    int issued = 0;                      // stages the producer warp has issued
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    float oacc[KSTEPS][4];
#pragma unroll
    for (int mt = 0; mt < KSTEPS; ++mt)
#pragma unroll
        for (int e = 0; e < 4; ++e) oacc[mt][e] = 0.f;

    if (warp == CONS_WARPS) {
        // ---------------- producer ----------------
        const int32_t last = (n_all > 0) ? idx[n_all - 1] : 0;
        // this lane's key ids of the next stage are read before the wait for
        // a free slot, so the index loads overlap the copies in flight
        constexpr int XPL = (2 * C::KT + 31) / 32;   // copies per lane per stage
        int32_t tn[XPL];
        auto load_tok = [&](int j) {
#pragma unroll
            for (int u = 0; u < XPL; ++u) {
                const int x = lane + 32 * u;
                const int key = k_lo + j * C::KT + x % C::KT;
                tn[u] = (x < 2 * C::KT && key < k_hi) ? idx[key] : last;
            }
        };
        if (n_st > 0) load_tok(0);
        for (int j = 0; j < n_st; ++j) {
            const int s = j % STAGES;
            const uint32_t ph = (uint32_t)((j / STAGES) & 1);
            int32_t tc[XPL];
#pragma unroll
            for (int u = 0; u < XPL; ++u) tc[u] = tn[u];
            if (j + 1 < n_st) load_tok(j + 1);
            // the warp agrees on every decision, so it never diverges here
            if (__any_sync(0xffffffffu, *abort_flag != 0)) break;
            if (!__all_sync(0xffffffffu, ptx::mbar_wait_bounded(&empty[s], ph ^ 1u, wl))) {
                if (lane == 0) {
                    *abort_flag = 1;
                    if (status) dev_error(status, DEV_TIMEOUT, (uint32_t)row);
                }
                break;
            }
            if (lane == 0) ptx::mbar_arrive_expect_tx(&full[s], 2u * C::KT * C::RB);
            __syncwarp();
            unsigned char* kt = smem + s * C::STAGE;
#pragma unroll
            for (int u = 0; u < XPL; ++u) {
                const int x = lane + 32 * u;
                if (x >= 2 * C::KT) break;
                const int r = x % C::KT;
                const int32_t t = checked_index(tc[u], T_cap, status);
                const int64_t off = ((b * T_cap + t) * Hkv + g0) * (int64_t)D;
                if (x < C::KT)
                    ptx::bulk_g2s(kt + r * C::PITCH, K + off, C::RB, &full[s]);
                else
                    ptx::bulk_g2s(kt + C::TILE + r * C::PITCH, V + off, C::RB, &full[s]);
            }
            issued = j + 1;
        }
    } else {
        // ---------------- consumers ----------------
        const int hl = warp % HG;              // KV head inside the group
        const int sub = warp / HG;             // 16-key slice of every stage
        const int g = g0 + hl;
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
        const int hoff = hl * D * 2;             // byte offset of this head in a row
        for (int j = 0; j < n_st; ++j) {
            const int s = j % STAGES;
            const uint32_t ph = (uint32_t)((j / STAGES) & 1);
            if (__any_sync(0xffffffffu, *abort_flag != 0)) break;
            if (!__all_sync(0xffffffffu, ptx::mbar_wait_bounded(&full[s], ph, wl))) {
                if (lane == 0) {
                    *abort_flag = 1;
                    if (status) dev_error(status, DEV_TIMEOUT, (uint32_t)row);
                }
                break;
            }
            const unsigned char* kt = smem + s * C::STAGE + sub * 16 * C::PITCH + hoff;
            const unsigned char* vt = kt + C::TILE;
            const int kbase = j * C::KT + sub * 16;   // key offset inside this CTA's keys
            if (kbase < n) {
                float sacc[4] = {0.f, 0.f, 0.f, 0.f};
                {
                    const unsigned char* base = kt + (lane & 15) * C::PITCH + (lane >> 4) * 16;
#pragma unroll
                    for (int kk = 0; kk < KSTEPS; ++kk) {
                        uint32_t a0, a1, a2, a3;
                        ptx::ldsm_x4(a0, a1, a2, a3, base + kk * 32);
                        ptx::mma_bf16_16816(sacc, a0, a1, a2, a3, qf[kk][0], qf[kk][1]);
                    }
                }
                const int key_lo = kbase + (lane >> 2), key_hi = key_lo + 8;
                const float z0 = (key_lo < n) ? sacc[0] * scale_log2 : -INFINITY;
                const float z1 = (key_lo < n) ? sacc[1] * scale_log2 : -INFINITY;
                const float z2 = (key_hi < n) ? sacc[2] * scale_log2 : -INFINITY;
                const float z3 = (key_hi < n) ? sacc[3] * scale_log2 : -INFINITY;
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
                const uint32_t pb0 = ptx::movmatrix_t(ptx::pack_bf16(p0, p1));
                const uint32_t pb1 = ptx::movmatrix_t(ptx::pack_bf16(p2, p3));
                {
                    const int mi = lane >> 3, r = lane & 7;
                    const unsigned char* base = vt + (r + 8 * (mi >> 1)) * C::PITCH + (mi & 1) * 16;
#pragma unroll
                    for (int mt = 0; mt < KSTEPS; ++mt) {
                        uint32_t a0, a1, a2, a3;
                        ptx::ldsm_x4_t(a0, a1, a2, a3, base + mt * 32);
                        ptx::mma_bf16_16816(oacc[mt], a0, a1, a2, a3, pb0, pb1);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&empty[s]);
        }
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
            l0 += __shfl_xor_sync(0xffffffffu, l0, o);
            l1 += __shfl_xor_sync(0xffffffffu, l1, o);
        }
    }
    // Copies of an aborted stage may still be in flight: the latest issue of
    // every ring slot gets a bounded chance to land before the ring is reused
    // for the merge (slots never issued are not waited for).
    if (*abort_flag && warp == CONS_WARPS)
        for (int j = (issued > STAGES ? issued - STAGES : 0); j < issued; ++j)
            ptx::mbar_wait_bounded(&full[j % STAGES], (uint32_t)((j / STAGES) & 1), WAIT_LIMIT);
    __syncthreads();

    // ---------------- merge the warps of each head ----------------
    float* mw = reinterpret_cast<float*>(smem);         // [CONS_WARPS][8]
    float* lw = mw + CONS_WARPS * 8;                    // [CONS_WARPS][8]
    float* ow = lw + CONS_WARPS * 8;                    // [CONS_WARPS][8][D]
    if (warp < CONS_WARPS) {
        if (lane < 4) {
            mw[warp * 8 + 2 * lane] = m0;
            mw[warp * 8 + 2 * lane + 1] = m1;
            lw[warp * 8 + 2 * lane] = l0;
            lw[warp * 8 + 2 * lane + 1] = l1;
        }
        const int h0 = 2 * (lane & 3), dr = lane >> 2;
        float* o = ow + (warp * 8) * D;
#pragma unroll
        for (int mt = 0; mt < KSTEPS; ++mt) {
            o[h0 * D + mt * 16 + dr] = oacc[mt][0];
            o[(h0 + 1) * D + mt * 16 + dr] = oacc[mt][1];
            o[h0 * D + mt * 16 + dr + 8] = oacc[mt][2];
            o[(h0 + 1) * D + mt * 16 + dr + 8] = oacc[mt][3];
        }
    }
    __syncthreads();
    const bool aborted = *abort_flag != 0;
    const int nq_heads = HG * hpg;                     // query heads of this CTA
    const float nanf_ = __int_as_float(0x7fc00000);
    if (sk.ns == 1) {
        for (int x = threadIdx.x; x < nq_heads * D; x += ATT_THREADS) {
            const int qh = x / D, c = x % D;
            const int hl = qh / hpg, h = qh % hpg;
            float M = -INFINITY;
            for (int sb = 0; sb < CONS_WARPS / HG; ++sb) M = fmaxf(M, mw[(sb * HG + hl) * 8 + h]);
            float L = 0.f, acc = 0.f;
            for (int sb = 0; sb < CONS_WARPS / HG; ++sb) {
                const int w = sb * HG + hl;
                const float sc = (mw[w * 8 + h] == -INFINITY) ? 0.f : exp2f(mw[w * 8 + h] - M);
                L += lw[w * 8 + h] * sc;
                acc += ow[(w * 8 + h) * D + c] * sc;
            }
            const int64_t oh = row * Hq + (int64_t)g0 * hpg + qh;
            O[oh * D + c] = __float2bfloat16_rn(aborted ? nanf_ : acc / L);
            if (c == 0 && lse) lse[oh] = aborted ? nanf_ : (M + log2f(L)) * 0.69314718055994531f;
        }
        return;
    }
    // split-KV: write this split's partial per query head as
    // [acc[0..D) | max | sum | 2 pad] (stride D + 4 floats, 16-byte aligned)
    constexpr int PS = D + 4;
    for (int x = threadIdx.x; x < nq_heads * (D + 2); x += ATT_THREADS) {
        const int qh = x / (D + 2), c = x % (D + 2);
        const int hl = qh / hpg, h = qh % hpg;
        float M = -INFINITY;
        for (int sb = 0; sb < CONS_WARPS / HG; ++sb) M = fmaxf(M, mw[(sb * HG + hl) * 8 + h]);
        float v = 0.f;
        if (c == D) {
            v = M;
        } else {
            for (int sb = 0; sb < CONS_WARPS / HG; ++sb) {
                const int w = sb * HG + hl;
                const float sc = (mw[w * 8 + h] == -INFINITY) ? 0.f : exp2f(mw[w * 8 + h] - M);
                v += (c == D + 1 ? lw[w * 8 + h] : ow[(w * 8 + h) * D + c]) * sc;
            }
        }
        const int64_t qhg = (int64_t)g0 * hpg + qh;
        sk.part[((row * sk.ns + split) * Hq + qhg) * PS + c] = aborted ? nanf_ : v;
    }
    if (!sk.counter) return;   // partials only: attn_combine_kernel merges them
    __threadfence();
    __syncthreads();
    __shared__ uint32_t sh_last;
    if (threadIdx.x == 0) {
        const uint32_t prev = atomicAdd(&sk.counter[unit], 1u);
        sh_last = (prev == (uint32_t)sk.ns - 1) ? 1u : 0u;
    }
    __syncthreads();
    if (!sh_last) return;
    __threadfence();
    // Combine: per query head the global max M over splits and each split's
    // weight exp2(m_s - M) / L (L = sum of the rescaled partial sums), then
    // every output element is one weighted sum over splits.  Partials of other
    // CTAs are read through L2 (__ldcg), never through a stale L1 line.
    float* m_sp = reinterpret_cast<float*>(smem);           // [nq_heads][ns]
    float* w_sp = m_sp + nq_heads * sk.ns;                   // [nq_heads][ns]
    const int64_t sstride = (int64_t)Hq * PS;
    const float* pbase = sk.part + (row * sk.ns * Hq + (int64_t)g0 * hpg) * PS;
    for (int x = threadIdx.x; x < nq_heads * sk.ns; x += ATT_THREADS) {
        const int qh = x / sk.ns, sp = x % sk.ns;
        const float2 ml = __ldcg(reinterpret_cast<const float2*>(pbase + sp * sstride +
                                                                 (int64_t)qh * PS + D));
        m_sp[x] = ml.x;
        w_sp[x] = ml.y;   // partial sum for now
    }
    __syncthreads();
    for (int qh = threadIdx.x; qh < nq_heads; qh += ATT_THREADS) {
        float M = -INFINITY;
        for (int sp = 0; sp < sk.ns; ++sp) M = fmaxf(M, m_sp[qh * sk.ns + sp]);
        float L = 0.f;
        for (int sp = 0; sp < sk.ns; ++sp) {
            const float ms = m_sp[qh * sk.ns + sp];
            const float e = (ms == -INFINITY) ? 0.f : exp2f(ms - M);
            m_sp[qh * sk.ns + sp] = e;                       // reuse as the rescale
            L += w_sp[qh * sk.ns + sp] * e;
        }
        for (int sp = 0; sp < sk.ns; ++sp) w_sp[qh * sk.ns + sp] = m_sp[qh * sk.ns + sp] / L;
        if (lse) lse[row * Hq + (int64_t)g0 * hpg + qh] = (M + log2f(L)) * 0.69314718055994531f;
    }
    __syncthreads();
    // every output element is one weighted sum over splits; 4 dims per thread,
    // several splits' loads in flight at once
    for (int x = threadIdx.x; x < nq_heads * (D / 4); x += ATT_THREADS) {
        const int qh = x / (D / 4), c = (x % (D / 4)) * 4;
        const float* pp = pbase + (int64_t)qh * PS + c;
        const float* wq = w_sp + qh * sk.ns;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
        for (int sp = 0; sp < sk.ns; ++sp) {
            const float4 v = __ldcg(reinterpret_cast<const float4*>(pp + sp * sstride));
            const float w = wq[sp];
            acc.x += v.x * w;
            acc.y += v.y * w;
            acc.z += v.z * w;
            acc.w += v.w * w;
        }
        __nv_bfloat16* o = O + (row * Hq + (int64_t)g0 * hpg + qh) * D + c;
        o[0] = __float2bfloat16_rn(acc.x);
        o[1] = __float2bfloat16_rn(acc.y);
        o[2] = __float2bfloat16_rn(acc.z);
        o[3] = __float2bfloat16_rn(acc.w);
    }
    if (threadIdx.x == 0) sk.counter[unit] = 0;   // ready for the next launch
}

// ---------------------------------------------------------------------------
// Split-KV combine: one CTA (CB_WARPS warps) per (query row, query head), so
// that every split's partial is in flight at once (the combine is short and
// latency-bound).  The (max, sum) of every split go to shared memory first:
// M = the largest max, w_s = exp2(m_s - M), L = sum of w_s * sum_s.  Warp w
// then accumulates splits w, w + CB_WARPS, ... (lane = 4 output dimensions,
// 16-byte loads, all of the warp's splits issued before they are summed), the
// warps' sums meet in shared memory, and O = sum / L.
// ---------------------------------------------------------------------------
constexpr int CB_WARPS = 8;
constexpr int CB_MAX_SPLITS = 128;
constexpr int CB_PER_WARP = CB_MAX_SPLITS / CB_WARPS;   // splits per warp at most

template <int D>
__global__ void __launch_bounds__(32 * CB_WARPS) attn_combine_kernel(const float* __restrict__ part,
                                                                     int ns, int Hq,
                                                                     __nv_bfloat16* O, float* lse)
{
    constexpr int PS = D + 4;
    __shared__ float w_s[CB_MAX_SPLITS];
    __shared__ float4 acc_s[CB_WARPS][D / 4];
    __shared__ float sh_M, sh_L;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t wid = blockIdx.x;                  // (row, head)
    const int64_t row = wid / Hq, h = wid % Hq;
    const float* base = part + (row * ns * Hq + h) * PS;
    const int64_t sstride = (int64_t)Hq * PS;
    // every warp's splits, loaded before anything waits on them
    const bool live = lane < D / 4;
    float4 v[CB_PER_WARP];
#pragma unroll
    for (int u = 0; u < CB_PER_WARP; ++u) {
        const int sp = warp + CB_WARPS * u;
        v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (live && sp < ns) v[u] = __ldcg(reinterpret_cast<const float4*>(base + sp * sstride) + lane);
    }
    // (max, sum) of every split
    float m = -INFINITY;
    for (int sp = threadIdx.x; sp < ns; sp += 32 * CB_WARPS) {
        const float2 ml = __ldcg(reinterpret_cast<const float2*>(base + sp * sstride + D));
        w_s[sp] = ml.x;
        m = fmaxf(m, ml.x);
    }
    __shared__ float m_w[CB_WARPS];
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) m_w[warp] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        float M = m_w[0];
        for (int x = 1; x < CB_WARPS; ++x) M = fmaxf(M, m_w[x]);
        sh_M = M;
    }
    __syncthreads();
    const float M = sh_M;
    float lsum = 0.f;
    for (int sp = threadIdx.x; sp < ns; sp += 32 * CB_WARPS) {
        const float ms = w_s[sp];
        const float w = (ms == -INFINITY) ? 0.f : exp2f(ms - M);
        w_s[sp] = w;
        lsum += __ldcg(base + sp * sstride + D + 1) * w;
    }
    for (int o = 16; o > 0; o >>= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, o);
    __syncthreads();                                 // w_s complete; m_w free
    if (lane == 0) m_w[warp] = lsum;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int u = 0; u < CB_PER_WARP; ++u) {
        const int sp = warp + CB_WARPS * u;
        if (sp < ns) {
            const float w = w_s[sp];
            acc.x += v[u].x * w;
            acc.y += v[u].y * w;
            acc.z += v[u].z * w;
            acc.w += v[u].w * w;
        }
    }
    if (live) acc_s[warp][lane] = acc;
    __syncthreads();
    if (threadIdx.x == 0) {
        float L = 0.f;
        for (int x = 0; x < CB_WARPS; ++x) L += m_w[x];
        sh_L = L;
    }
    __syncthreads();
    if (warp == 0 && live) {
        float4 t = acc_s[0][lane];
#pragma unroll
        for (int x = 1; x < CB_WARPS; ++x) {
            const float4 y = acc_s[x][lane];
            t.x += y.x;
            t.y += y.y;
            t.z += y.z;
            t.w += y.w;
        }
        const float inv = 1.f / sh_L;
        __nv_bfloat16* op = O + wid * D + 4 * lane;
        op[0] = __float2bfloat16_rn(t.x * inv);
        op[1] = __float2bfloat16_rn(t.y * inv);
        op[2] = __float2bfloat16_rn(t.z * inv);
        op[3] = __float2bfloat16_rn(t.w * inv);
    }
    if (threadIdx.x == 0 && lse) lse[wid] = (M + log2f(sh_L)) * 0.69314718055994531f;
}

cudaError_t launch_attn_combine(const float* part, int ns, int64_t rows, int Hq, int d, void* O,
                                float* lse, cudaStream_t st)
{
    if (ns < 1 || ns > CB_MAX_SPLITS) return cudaErrorInvalidValue;
    const unsigned grid = (unsigned)(rows * Hq);
    if (d == 128)
        attn_combine_kernel<128><<<grid, 32 * CB_WARPS, 0, st>>>(part, ns, Hq, (__nv_bfloat16*)O, lse);
    else
        attn_combine_kernel<64><<<grid, 32 * CB_WARPS, 0, st>>>(part, ns, Hq, (__nv_bfloat16*)O, lse);
    note_launch();
    return cudaGetLastError();
}

template <int D, int HG, int STAGES>
static cudaError_t launch_bf16(const void* Q, const void* K, const void* V, int64_t B, int64_t Nq,
                               int64_t T_cap, int Hq, int Hkv, const int32_t* indices,
                               const int32_t* counts, int s_max, float scale, void* O, float* lse,
                               uint32_t* status, SplitKV sk, cudaStream_t st)
{
    using C = AttnCfg<D, HG, STAGES>;
    auto kern = attn_bf16_kernel<D, HG, STAGES>;
    cudaError_t e = ensure_smem_attr((const void*)kern, C::BYTES);
    if (e != cudaSuccess) return e;
    if (sk.ns > 1 && sk.keys_per_split % C::KT != 0) return cudaErrorInvalidValue;
    // the split combine keeps 2 * (query heads of the CTA) * ns + heads floats
    // in the freed ring
    if (sk.ns > 1 && (size_t)(2 * HG * (Hq / Hkv) * sk.ns) * 4 > (size_t)C::BODY)
        return cudaErrorInvalidValue;
    const int64_t ctas = B * Nq * (Hkv / HG) * sk.ns;
    kern<<<(unsigned)ctas, ATT_THREADS, C::BYTES, st>>>(
        (const __nv_bfloat16*)Q, (const __nv_bfloat16*)K, (const __nv_bfloat16*)V, Nq, T_cap, Hq,
        Hkv, Hq / Hkv, indices, counts, s_max, scale * 1.4426950408889634f, (__nv_bfloat16*)O, lse,
        status, sk);
    note_launch();
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
    note_launch();
    return cudaGetLastError();
}

// KV heads per CTA and keys per stage of the bf16 kernel for a given KV head
// count (split sizes must be multiples of the stage).
int attn_head_group(int Hkv) { return (Hkv % 4 == 0) ? 4 : Hkv; }

int attn_stage_keys(int Hkv) { return 16 * (CONS_WARPS / attn_head_group(Hkv)); }

cudaError_t ensure_smem_attr(const void* kernel, int bytes)
{
    constexpr int MAXDEV = 64;
    struct Rec {
        const void* k;
        int dev;
    };
    static Rec done[256];
    static int n_done = 0;
    static std::mutex mu;
    std::lock_guard<std::mutex> lock(mu);
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    for (int i = 0; i < n_done; ++i)
        if (done[i].k == kernel && done[i].dev == dev) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    if (n_done < 256 && dev < MAXDEV) done[n_done++] = Rec{kernel, dev};
    return cudaSuccess;
}

template <int D>
static cudaError_t launch_bf16_d(const void* Q, const void* K, const void* V, int64_t B, int64_t Nq,
                                 int64_t T_cap, int Hq, int Hkv, const int32_t* indices,
                                 const int32_t* counts, int s_max, float scale, void* O,
                                 float* lse, uint32_t* status, SplitKV sk, int hg, cudaStream_t st)
{
    if (hg == 1)
        return launch_bf16<D, 1, 3>(Q, K, V, B, Nq, T_cap, Hq, Hkv, indices, counts, s_max, scale,
                                    O, lse, status, sk, st);
    if (Hkv % 4 == 0)
        return launch_bf16<D, 4, 3>(Q, K, V, B, Nq, T_cap, Hq, Hkv, indices, counts, s_max, scale,
                                    O, lse, status, sk, st);
    if (Hkv == 2)
        return launch_bf16<D, 2, 3>(Q, K, V, B, Nq, T_cap, Hq, Hkv, indices, counts, s_max, scale,
                                    O, lse, status, sk, st);
    if (Hkv == 1)
        return launch_bf16<D, 1, 3>(Q, K, V, B, Nq, T_cap, Hq, Hkv, indices, counts, s_max, scale,
                                    O, lse, status, sk, st);
    return cudaErrorInvalidValue;
}

cudaError_t launch_attn_split(const void* Q, const void* K, const void* V, int64_t B, int64_t Nq,
                              int64_t T_cap, int Hq, int Hkv, int d, const int32_t* indices,
                              const int32_t* counts, int s_max, float scale, void* O, float* lse,
                              uint32_t* status, int ns, int keys_per_split, float* part,
                              uint32_t* counter, int hg, cudaStream_t st)
{
    SplitKV sk{ns, keys_per_split, part, counter};
    if (d == 128)
        return launch_bf16_d<128>(Q, K, V, B, Nq, T_cap, Hq, Hkv, indices, counts, s_max, scale,
                                  O, lse, status, sk, hg, st);
    return launch_bf16_d<64>(Q, K, V, B, Nq, T_cap, Hq, Hkv, indices, counts, s_max, scale, O, lse,
                             status, sk, hg, st);
}

cudaError_t launch_attn_rows(const void* Q, const void* K, const void* V, int64_t B, int64_t Nq,
                             int64_t T_cap, int Hq, int Hkv, int d, const int32_t* indices,
                             const int32_t* counts, int s_max, float scale, void* O,
                             uint32_t* status, const int32_t* row_list, const int32_t* row_count,
                             cudaStream_t st)
{
    if (B * Nq == 0) return cudaSuccess;
    SplitKV sk{1, s_max, nullptr, nullptr, row_list, row_count};
    if (d == 128)
        return launch_bf16_d<128>(Q, K, V, B, Nq, T_cap, Hq, Hkv, indices, counts, s_max, scale,
                                  O, nullptr, status, sk, 0, st);
    return launch_bf16_d<64>(Q, K, V, B, Nq, T_cap, Hq, Hkv, indices, counts, s_max, scale, O,
                             nullptr, status, sk, 0, st);
}

cudaError_t launch_attn_status(const void* Q, const void* K, const void* V, lsa_dtype dt, int64_t B,
                               int64_t Nq, int64_t T_cap, int Hq, int Hkv, int d,
                               const int32_t* indices, const int32_t* counts, int s_max, float scale,
                               void* O, float* lse, uint32_t* status, cudaStream_t st)
{
    if (B * Nq == 0) return cudaSuccess;
    const int hpg = Hq / Hkv;
    if (dt == LSA_BF16)
        return launch_attn_split(Q, K, V, B, Nq, T_cap, Hq, Hkv, d, indices, counts, s_max, scale,
                                 O, lse, status, 1, s_max, nullptr, nullptr, 0, st);
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

cudaError_t set_attn_wait_polls(int64_t polls)
{
    const uint32_t v = (polls < 0 || polls > (int64_t)WAIT_LIMIT) ? WAIT_LIMIT : (uint32_t)polls;
    return cudaMemcpyToSymbol(g_attn_wait, &v, sizeof(v));
}

}  // namespace lsa
