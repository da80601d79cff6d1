// lsa_api.cu -- host side of the liblsa C-ABI: argument checks, index
// storage layout, stream-ordered orchestration of the kernels, status words.
// Every entry point is declared and documented in include/lsa.h.
#include <stdarg.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <math.h>

#include <atomic>
#include <new>

#include <nvtx3/nvToolsExt.h>

#include "hooks.cuh"
#include "lsa_internal.cuh"

using namespace lsa;

namespace {

std::atomic<uint64_t> g_launches{0};

thread_local char g_err[512] = "";

lsa_status fail(lsa_status s, const char* fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof(g_err), fmt, ap);
    va_end(ap);
    return s;
}

lsa_status cuda_fail(cudaError_t e, const char* where)
{
    return fail(LSA_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

inline size_t al256(size_t x) { return (x + 255) & ~(size_t)255; }

// NVTX range around a public entry (visible to nsys / ncu range filters; a
// no-op when no tool is attached).
struct NvtxRange {
    explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
};

// ---- LSA_DEBUG=1 checks (k_debug.cu) ----
const char* dbg_kind_name(uint32_t k)
{
    switch (k) {
    case DBG_OFFSETS: return "CSR offsets of a block out of range or decreasing";
    case DBG_MEMBER: return "a bucket member outside its block";
    case DBG_ORDER: return "bucket members not ascending";
    case DBG_ASSIGN: return "a member whose assignment names another bucket";
    case DBG_OPEN: return "an open-block entry that is no closed bucket";
    case DBG_COUNT: return "a selection count out of range";
    case DBG_INDEX: return "a gather index outside [0, T_cap)";
    case DBG_CAUSAL: return "a selected index after its query's position";
    case DBG_LAYOUT: return "a selection row not laid out as sinks, long-range keys, window";
    default: return "unknown";
    }
}

lsa_status dbg_result(cudaError_t e, const uint32_t h[4], const char* what)
{
    if (e != cudaSuccess) return cuda_fail(e, "debug check");
    if (h[0] == 0u) return LSA_OK;
    return fail(LSA_ERR_INTERNAL, "debug check (%s): %s (sequence/row %u, at %u, value %d)", what,
                dbg_kind_name(h[0]), h[1], h[2], (int)h[3]);
}

lsa_status dbg_index(const IndexView& v, int64_t n_blk, cudaStream_t st, const char* what)
{
    if (!debug_enabled()) return LSA_OK;
    uint32_t h[4];
    const cudaError_t e = debug_check_index(v, n_blk, st, h);
    return dbg_result(e, h, what);
}

lsa_status dbg_gather(const int32_t* indices, const int32_t* counts, int64_t B, int64_t Nq,
                      int s_max, int64_t T_cap, PosSrc pos, lsa_select_params sp, int mode,
                      cudaStream_t st, const char* what)
{
    if (!debug_enabled()) return LSA_OK;
    uint32_t h[4];
    const cudaError_t e = debug_check_gather(indices, counts, B * Nq, s_max, T_cap, pos, Nq,
                                             sp.window, sp.sinks, mode, st, h);
    return dbg_result(e, h, what);
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

lsa_status check_index_params(int64_t B, int64_t T_cap, lsa_index_params ip)
{
    if (B < 1 || B > 65535) return fail(LSA_ERR_INVALID_ARG, "B=%lld outside [1, 65535]", (long long)B);
    if (T_cap < 1 || T_cap > 2147483647LL)
        return fail(LSA_ERR_INVALID_ARG, "T_cap=%lld outside [1, 2^31-1]", (long long)T_cap);
    if (ip.p < 1 || ip.block < 1 || ip.n_buckets < 1 || ip.lloyd_iters < 1)
        return fail(LSA_ERR_INVALID_ARG, "index parameters must be >= 1");
    if (ip.n_buckets > ip.block)
        return fail(LSA_ERR_INVALID_ARG, "n_buckets=%d > block=%d", ip.n_buckets, ip.block);
    if (ip.n_buckets > MAX_K)
        return fail(LSA_ERR_UNSUPPORTED, "n_buckets=%d > %d", ip.n_buckets, MAX_K);
    if (ip.block > 4096) return fail(LSA_ERR_UNSUPPORTED, "block=%d > 4096", ip.block);
    if (ip.lloyd_iters > 1000) return fail(LSA_ERR_INVALID_ARG, "lloyd_iters > 1000");
    if ((int64_t)ip.p * ip.block > T_cap)
        return fail(LSA_ERR_INVALID_ARG, "T_cap=%lld holds no whole block", (long long)T_cap);
    return LSA_OK;
}

struct Layout {
    size_t pooled, unit, cent, cent_rt, offsets, members, assign, open, status, total;
};

Layout layout(int64_t B, int64_t T_cap, lsa_index_params ip, lsa_dtype dt)
{
    const int64_t NP = T_cap / ip.p;
    const int64_t nblk = NP / ip.block;
    const int64_t NBK = nblk * ip.n_buckets;
    const size_t rt = (dt == LSA_BF16) ? 2 : 4;
    Layout L;
    size_t o = 0;
    L.pooled = o;  o += al256((size_t)B * NP * DL * 4);
    L.unit = o;    o += al256((size_t)B * NP * DL * 4);
    L.cent = o;    o += al256((size_t)B * NBK * DL * 4);
    L.cent_rt = o; o += al256((size_t)B * NBK * DL * rt);
    L.offsets = o; o += al256((size_t)B * (NBK + 1) * 4);
    L.members = o; o += al256((size_t)B * NP * 4);
    L.assign = o;  o += al256((size_t)B * NP * 2);
    L.open = o;    o += al256((size_t)B * ip.block * 4);
    L.status = o;  o += al256(8 * 4);
    L.total = o;
    return L;
}

lsa_status check_select(const lsa_index* idx, lsa_select_params sp, int s_max)
{
    if (sp.budget < 0 || sp.window < 0 || sp.sinks < 0)
        return fail(LSA_ERR_INVALID_ARG, "budget/window/sinks must be >= 0");
    if ((int64_t)sp.budget + sp.window + sp.sinks > s_max)
        return fail(LSA_ERR_INVALID_ARG, "s_max=%d < budget+window+sinks=%lld", s_max,
                    (long long)sp.budget + sp.window + sp.sinks);
    if (sp.window < idx->v.p - 1)
        return fail(LSA_ERR_UNSUPPORTED,
                    "window=%d < p-1: keys of an incomplete pooled group would be unreachable",
                    sp.window);
    return LSA_OK;
}

// The SIMT nominator keeps every eligible score in shared memory.
constexpr int64_t SIMT_MAX_BUCKETS = (220 * 1024) / 4;

bool use_tc_path(const lsa_index* idx, int64_t Nq) { return select_uses_tc(idx->v, Nq); }

lsa_status run_select(const lsa_index* idx, const void* lq, PosSrc pos, int64_t Nq,
                      lsa_select_params sp, int32_t* indices, int32_t* counts, int s_max, void* ws,
                      cudaStream_t st, const BucketPlan* plan = nullptr)
{
    const bool tc = use_tc_path(idx, Nq);
    if (!tc && idx->n_blk * idx->v.k > SIMT_MAX_BUCKETS)
        return fail(LSA_ERR_UNSUPPORTED, "%lld buckets exceed the SIMT scorer's %lld",
                    (long long)(idx->n_blk * idx->v.k), (long long)SIMT_MAX_BUCKETS);
    lsa_status s = dbg_index(idx->v, idx->n_blk, st, "index before selection");
    if (s != LSA_OK) return s;
    SelectWs w = select_ws_carve(ws, idx->v, Nq);
    if (plan) w.plan = *plan;
    cudaError_t e = launch_select(idx->v, idx->n_blk, lq, pos, Nq, sp, indices, counts, s_max, w,
                                  tc, st);
    if (e != cudaSuccess) return cuda_fail(e, "select");
    return dbg_gather(indices, counts, idx->v.B, Nq, s_max, idx->v.T_cap, pos, sp, DBG_SELECTION,
                      st, "selection");
}

// Prefill workspace: selection output and scratch, then (bf16 with a
// supported head shape) the bucket-major attention lists with ent_cap
// partial slots of Hq * (d + 4) floats each.
struct PrefillLayout {
    size_t indices, counts, sel, zero, row_n, row_base, gather, ent, ent2, bucket_off, tiles,
        sorted, part, part_ml, recs, total;
    int64_t ent_cap, tile_cap, n_zero;
    bool bucket;
};

PrefillLayout prefill_layout(const lsa_index* idx, int64_t Nq, int Hq, int Hkv, int d,
                             lsa_select_params sp, int64_t ent_cap)
{
    const IndexView& v = idx->v;
    const int64_t s_max = (int64_t)sp.budget + sp.window + sp.sinks;
    const size_t rows = (size_t)v.B * (size_t)Nq;
    PrefillLayout L{};
    size_t o = 0;
    L.indices = o; o += al256(rows * (size_t)s_max * 4);
    L.counts = o;  o += al256(rows * 4);
    L.sel = o;     o += select_ws_bytes(v, Nq);
    // (sinks within the first block: no open-block key is ever below the sinks bound)
    L.bucket = v.dtype == LSA_BF16 && bucket_attn_supported(Hq, Hkv, d) &&
               (int64_t)sp.sinks <= (int64_t)v.p * v.G;
    if (L.bucket) {
        const int64_t nbt = v.B * v.NBK;
        L.ent_cap = ent_cap;
        L.tile_cap = ent_cap / BA_Q + (nbt < ent_cap ? nbt : ent_cap) + 1;
        L.n_zero = nbt + CTR_N;
        L.zero = o;       o += al256((size_t)L.n_zero * 4);
        L.row_n = o;      o += al256(rows * 4);
        L.row_base = o;   o += al256(rows * 4);
        L.gather = o;     o += al256(rows * 4);
        L.ent = o;        o += al256((size_t)ent_cap * 16);
        L.ent2 = o;       o += al256((size_t)ent_cap * 8);
        L.bucket_off = o; o += al256((size_t)nbt * 4);
        L.tiles = o;      o += al256((size_t)L.tile_cap * 8);
        L.sorted = o;     o += al256((size_t)ent_cap * 4);
        L.part = o;       o += al256((size_t)ent_cap * Hq * d * 2);
        L.part_ml = o;    o += al256((size_t)ent_cap * Hq * 8);
        const int64_t n_wt = v.B * ((Nq + BA_Q - 1) / BA_Q);
        L.recs = o;       o += al256((size_t)(n_wt + L.tile_cap) * TILE_REC_BYTES);
    }
    L.total = o;
    return L;
}

// Partial slots per query row that the recommended workspace provides: one
// per expected bucket (budget / mean bucket size) with half again as much
// room, plus the sinks-and-window slot and one spare.  The slots are shared
// by the whole chunk, so only the chunk's mean matters.
int64_t default_ent_cap(const lsa_index* idx, int64_t Nq, lsa_select_params sp)
{
    const IndexView& v = idx->v;
    int64_t bk = (int64_t)v.p * v.G / v.k;
    if (bk < 1) bk = 1;
    int64_t e = (3 * (int64_t)sp.budget + 2 * bk - 1) / (2 * bk) + 2;
    if (e > KC + 1) e = KC + 1;
    return v.B * Nq * e;
}

// Largest slot count whose layout fits in ws_bytes (-1: not even zero slots).
// The layout grows monotonically with the slot count, so a binary search over
// the exact layout finds it (the recommended workspace gives exactly the
// recommended slots).
int64_t ent_cap_for(const lsa_index* idx, int64_t Nq, int Hq, int Hkv, int d, lsa_select_params sp,
                    size_t ws_bytes)
{
    const PrefillLayout L0 = prefill_layout(idx, Nq, Hq, Hkv, d, sp, 0);
    if (ws_bytes < L0.total) return -1;
    if (!L0.bucket) return 0;
    int64_t lo = 0, hi = idx->v.B * Nq * (KC + 1);
    if (prefill_layout(idx, Nq, Hq, Hkv, d, sp, hi).total <= ws_bytes) return hi;
    while (hi - lo > 1) {   // invariant: lo fits, hi does not
        const int64_t mid = lo + (hi - lo) / 2;
        if (prefill_layout(idx, Nq, Hq, Hkv, d, sp, mid).total <= ws_bytes) lo = mid;
        else hi = mid;
    }
    return lo;
}

struct DecodeLayout {
    size_t indices, counts, sel, part, counter, dl_s, dl_g, dl_n, dl_tau, app_score, app_g,
        app_slot, total;
    int ns, kps, n_hg, n_slice;
};


#ifndef LSA_DEC_SPLIT_MULT
#define LSA_DEC_SPLIT_MULT 2
#endif

DecodeLayout decode_layout(const lsa_index* idx, int Hq, int Hkv, int d, lsa_select_params sp)
{
    const IndexView& v = idx->v;
    const int64_t s_max = (int64_t)sp.budget + sp.window + sp.sinks;
    DecodeLayout L;
    // decode attends one query per sequence: each CTA gathers whole head-group
    // rows (1 KB at Hkv=4, d=128: few large bulk copies) over one key split;
    // a separate combine kernel merges the splits
    const int hg = attn_head_group(Hkv);
    L.n_hg = Hkv / hg;
    const int kt = attn_stage_keys(Hkv);
    const int64_t units = v.B * L.n_hg;
    // about LSA_DEC_SPLIT_MULT CTAs per SM over all (sequence, head group, split)
    // triples
    int64_t ns = ((int64_t)sm_count() * LSA_DEC_SPLIT_MULT + units - 1) / units;
    if (ns < 1) ns = 1;
    if (ns > 128) ns = 128;   // the combine takes at most 128 splits
    int64_t kps = (s_max + ns - 1) / ns;
    kps = ((kps + kt - 1) / kt) * kt;
    ns = (s_max + kps - 1) / kps;
    L.ns = (int)ns;
    L.kps = (int)kps;
    size_t o = 0;
    L.indices = o; o += al256((size_t)v.B * s_max * 4);
    L.counts = o;  o += al256((size_t)v.B * 4);
    L.sel = o;     o += select_ws_bytes(v, 1);
    L.part = o;    o += al256((size_t)v.B * ns * Hq * (d + 4) * 4);
    L.counter = o; o += al256((size_t)v.B * L.n_hg * 4);
    // the append and scoring pass: about one CTA per SM over all sequences,
    // with at most 992 buckets per slice and at most 128 slices (the fill
    // merges one candidate list per slice); each slice nominates its m best
    int64_t nsl = ((int64_t)sm_count() + v.B - 1) / v.B;
    const int64_t min_sl = (v.NBK + 991) / 992;
    if (nsl < min_sl) nsl = min_sl;
    if (nsl > DEC_MAX_SLICES) nsl = DEC_MAX_SLICES;
    L.n_slice = (int)nsl;
    // each slice's sorted list of its DEC_M best scores (the fill merges them)
    L.dl_s = o;      o += al256((size_t)v.B * nsl * DEC_M * 4);
    L.dl_g = o;      o += al256((size_t)v.B * nsl * DEC_M * 4);
    L.dl_n = o;      o += al256((size_t)v.B * nsl * 4);
    L.dl_tau = o;    o += al256((size_t)v.B * nsl * 4);
    L.app_score = o; o += al256((size_t)v.B * nsl * 8);
    L.app_g = o;     o += al256((size_t)v.B * nsl * 4);
    L.app_slot = o;  o += al256((size_t)v.B * 4);
    L.total = o;
    return L;
}

lsa_status check_attn_shape(int Hq, int Hkv, int d, lsa_dtype dt)
{
    if (Hkv < 1 || Hq < 1 || Hq % Hkv != 0) return fail(LSA_ERR_INVALID_ARG, "Hq %% Hkv != 0");
    const int hpg = Hq / Hkv;
    if (hpg != 1 && hpg != 2 && hpg != 4 && hpg != 8)
        return fail(LSA_ERR_UNSUPPORTED, "Hq/Hkv=%d not in {1,2,4,8}", hpg);
    if (d != 64 && d != 128) return fail(LSA_ERR_UNSUPPORTED, "d=%d not in {64,128}", d);
    if (dt == LSA_BF16 && !(Hkv == 1 || Hkv == 2 || Hkv % 4 == 0))
        return fail(LSA_ERR_UNSUPPORTED, "Hkv=%d: bf16 kernels need Hkv in {1, 2} or a multiple of 4",
                    Hkv);
    return LSA_OK;
}

}  // namespace

int lsa::sm_count()
{
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && n > 0)
        return n;
    cudaGetLastError();  // clear the error of a host without a device
    return 148;
}

void lsa::note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

extern "C" {

uint64_t lsa_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

const char* lsa_last_error(void) { return g_err; }

const char* lsa_version(void) { return "liblsa 0.1 (D-LSA Flat, sm_100a)"; }

size_t lsa_index_bytes(int64_t B, int64_t T_cap, lsa_index_params ip, lsa_dtype dtype)
{
    if (check_index_params(B, T_cap, ip) != LSA_OK) return 0;
    if (dtype != LSA_F32 && dtype != LSA_BF16) {
        fail(LSA_ERR_INVALID_ARG, "unknown dtype %d", (int)dtype);
        return 0;
    }
    return layout(B, T_cap, ip, dtype).total;
}

lsa_status lsa_index_init(void* buf, size_t bytes, int64_t B, int64_t T_cap, lsa_index_params ip,
                          lsa_dtype dtype, lsa_index** out)
{
    if (!out) return fail(LSA_ERR_INVALID_ARG, "out is NULL");
    *out = nullptr;
    lsa_status s = check_index_params(B, T_cap, ip);
    if (s != LSA_OK) return s;
    if (dtype != LSA_F32 && dtype != LSA_BF16) return fail(LSA_ERR_INVALID_ARG, "unknown dtype");
    if (!buf) return fail(LSA_ERR_INVALID_ARG, "buf is NULL");
    if (((uintptr_t)buf & 255u) != 0) return fail(LSA_ERR_ALIGNMENT, "buf not 256-byte aligned");
    const Layout L = layout(B, T_cap, ip, dtype);
    if (bytes < L.total)
        return fail(LSA_ERR_WORKSPACE, "index buffer %zu < %zu bytes", bytes, L.total);
    lsa_index* h = new (std::nothrow) lsa_index;
    if (!h) return fail(LSA_ERR_INTERNAL, "host allocation failed");
    char* base = (char*)buf;
    IndexView& v = h->v;
    v.B = B;
    v.T_cap = T_cap;
    v.NP = T_cap / ip.p;
    v.nblk_max = (int)(v.NP / ip.block);
    v.NBK = (int64_t)v.nblk_max * ip.n_buckets;
    v.p = ip.p;
    v.G = ip.block;
    v.k = ip.n_buckets;
    v.L = ip.lloyd_iters;
    v.dtype = dtype;
    v.pooled = (float*)(base + L.pooled);
    v.unit = (float*)(base + L.unit);
    v.cent = (float*)(base + L.cent);
    v.cent_rt = (void*)(base + L.cent_rt);
    v.offsets = (int32_t*)(base + L.offsets);
    v.members = (int32_t*)(base + L.members);
    v.assign = (int16_t*)(base + L.assign);
    v.open_bucket = (int32_t*)(base + L.open);
    v.status = (uint32_t*)(base + L.status);
    h->n_blk = 0;
    h->buf = buf;
    h->bytes = bytes;
    h->status_clean = false;
    *out = h;
    return LSA_OK;
}

void lsa_index_release(lsa_index* idx) { delete idx; }

int64_t lsa_index_num_blocks(const lsa_index* idx) { return idx ? idx->n_blk : -1; }

lsa_status lsa_index_extend(lsa_index* idx, const void* latent_K, int64_t T_old, int64_t T_new,
                            void* stream)
{
    NvtxRange nv("lsa_index_extend");
    if (!idx || !latent_K) return fail(LSA_ERR_INVALID_ARG, "NULL index or latent_K");
    if (!aligned16(latent_K)) return fail(LSA_ERR_ALIGNMENT, "latent_K not 16-byte aligned");
    const IndexView& v = idx->v;
    if (T_old < 0 || T_new < T_old || T_new > v.T_cap)
        return fail(LSA_ERR_INVALID_ARG, "need 0 <= T_old <= T_new <= T_cap (%lld, %lld, %lld)",
                    (long long)T_old, (long long)T_new, (long long)v.T_cap);
    const int64_t span = (int64_t)v.p * v.G;
    const int64_t b0 = T_old / span, b1 = T_new / span;
    if (b0 > idx->n_blk)
        return fail(LSA_ERR_INVALID_ARG, "extend from block %lld leaves a gap after %lld blocks",
                    (long long)b0, (long long)idx->n_blk);
    cudaStream_t st = (cudaStream_t)stream;
    cudaError_t e;
    if (!idx->status_clean) {
        e = cudaMemsetAsync(v.status, 0, 8 * sizeof(uint32_t), st);
        if (e != cudaSuccess) return cuda_fail(e, "status clear");
        idx->status_clean = true;
    }
    const int64_t j_end = T_new / v.p;
    e = launch_pool_unit(v, latent_K, b0 * v.G, j_end, st);
    if (e != cudaSuccess) return cuda_fail(e, "pool");
    e = launch_kmeans(v, b0, b1, st);
    if (e != cudaSuccess) return cuda_fail(e, "kmeans");
    if (b1 > b0 || b1 > idx->n_blk) {
        if (b1 > idx->n_blk) idx->n_blk = b1;
        e = launch_open_assign(v, idx->n_blk, j_end, st);
        if (e != cudaSuccess) return cuda_fail(e, "open assign");
    } else if (j_end > idx->n_blk * v.G) {
        e = launch_open_assign(v, idx->n_blk, j_end, st);
        if (e != cudaSuccess) return cuda_fail(e, "open assign");
    }
    return dbg_index(v, idx->n_blk, st, "index after extension");
}

lsa_status lsa_build_index(lsa_index* idx, const void* latent_K, int64_t T, void* stream)
{
    return lsa_index_extend(idx, latent_K, 0, T, stream);
}

lsa_status lsa_index_export(const lsa_index* idx, float* pooled, float* unit, float* cent,
                            void* cent_rt, int32_t* offsets, int32_t* members, int16_t* assign,
                            int32_t* open_bucket, void* stream)
{
    if (!idx) return fail(LSA_ERR_INVALID_ARG, "NULL index");
    const IndexView& v = idx->v;
    cudaStream_t st = (cudaStream_t)stream;
    const size_t rt = (v.dtype == LSA_BF16) ? 2 : 4;
    struct {
        void* dst;
        const void* src;
        size_t n;
    } items[] = {
        {pooled, v.pooled, (size_t)v.B * v.NP * DL * 4},
        {unit, v.unit, (size_t)v.B * v.NP * DL * 4},
        {cent, v.cent, (size_t)v.B * v.NBK * DL * 4},
        {cent_rt, v.cent_rt, (size_t)v.B * v.NBK * DL * rt},
        {offsets, v.offsets, (size_t)v.B * (v.NBK + 1) * 4},
        {members, v.members, (size_t)v.B * v.NP * 4},
        {assign, v.assign, (size_t)v.B * v.NP * 2},
        {open_bucket, v.open_bucket, (size_t)v.B * v.G * 4},
    };
    for (auto& it : items) {
        if (!it.dst) continue;
        cudaError_t e = cudaMemcpyAsync(it.dst, it.src, it.n, cudaMemcpyDeviceToDevice, st);
        if (e != cudaSuccess) return cuda_fail(e, "export");
    }
    return LSA_OK;
}

lsa_status lsa_index_check(lsa_index* idx, int64_t* fallbacks, void* stream)
{
    if (!idx) return fail(LSA_ERR_INVALID_ARG, "NULL index");
    cudaStream_t st = (cudaStream_t)stream;
    uint32_t h[8] = {0};
    cudaError_t e = cudaMemcpyAsync(h, idx->v.status, sizeof(h), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e == cudaSuccess) e = cudaMemsetAsync(idx->v.status, 0, sizeof(h), st);
    if (e != cudaSuccess) return cuda_fail(e, "index check");
    if (fallbacks) *fallbacks = (int64_t)h[1];
    switch (h[0]) {
    case DEV_OK: return LSA_OK;
    case DEV_OPEN_FULL:
        return fail(LSA_ERR_INTERNAL, "decode append found the open block full (sequence %u)", h[2]);
    case DEV_BAD_INDEX:
        return fail(LSA_ERR_INVALID_ARG, "a selected index (%d) was outside [0, T_cap)", (int)h[2]);
    case DEV_TIMEOUT:
        return fail(LSA_ERR_TIMEOUT, "a bounded wait gave up (row %u)", h[2]);
    default: return fail(LSA_ERR_INTERNAL, "device status %u (detail %u)", h[0], h[2]);
    }
}

size_t lsa_select_workspace_bytes(const lsa_index* idx, int64_t Nq)
{
    if (!idx || Nq < 0) return 0;
    return select_ws_bytes(idx->v, Nq);
}

lsa_status lsa_select(const lsa_index* idx, const void* latent_Q, const int32_t* positions,
                      int64_t Nq, lsa_select_params sp, int32_t* indices, int32_t* counts,
                      int s_max, void* workspace, size_t ws_bytes, void* stream)
{
    NvtxRange nv("lsa_select");
    if (!idx || !latent_Q || !positions || !indices || !counts || !workspace)
        return fail(LSA_ERR_INVALID_ARG, "NULL argument");
    if (Nq < 0 || Nq > 2147483647LL) return fail(LSA_ERR_INVALID_ARG, "Nq out of range");
    lsa_status s = check_select(idx, sp, s_max);
    if (s != LSA_OK) return s;
    if (!aligned16(latent_Q) || !aligned16(positions) || !aligned16(indices) ||
        !aligned16(counts) || !aligned16(workspace))
        return fail(LSA_ERR_ALIGNMENT, "device pointers must be 16-byte aligned");
    if (ws_bytes < select_ws_bytes(idx->v, Nq))
        return fail(LSA_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes,
                    select_ws_bytes(idx->v, Nq));
    PosSrc pos{positions, 0};
    return run_select(idx, latent_Q, pos, Nq, sp, indices, counts, s_max, workspace,
                      (cudaStream_t)stream);
}

// ---- D-LSA Tree ----

namespace {
lsa_status check_tree(const lsa_index* idx, int n_super)
{
    if (!idx) return fail(LSA_ERR_INVALID_ARG, "NULL index");
    const int64_t nb = idx->n_blk * idx->v.k;
    if (idx->n_blk < 1) return fail(LSA_ERR_INVALID_ARG, "the index has no closed block");
    if (n_super < 1 || n_super > nb)
        return fail(LSA_ERR_INVALID_ARG, "n_super %d outside [1, %lld]", n_super, (long long)nb);
    if ((int64_t)n_super * 8 > 100 * 1024)
        return fail(LSA_ERR_UNSUPPORTED, "n_super %d above the 12800 super-buckets supported",
                    n_super);
    return LSA_OK;
}
}  // namespace

size_t lsa_tree_bytes(const lsa_index* idx, int n_super)
{
    if (!idx || n_super < 1) return 0;
    return tree_bytes(idx->v, n_super);
}

lsa_status lsa_tree_build(const lsa_index* idx, void* tree, size_t bytes, int n_super,
                          int lloyd_iters, void* stream)
{
    NvtxRange nv("lsa_tree_build");
    lsa_status s = check_tree(idx, n_super);
    if (s != LSA_OK) return s;
    if (!tree) return fail(LSA_ERR_INVALID_ARG, "NULL tree buffer");
    if (lloyd_iters < 1) return fail(LSA_ERR_INVALID_ARG, "lloyd_iters < 1");
    if (((uintptr_t)tree & 255) != 0) return fail(LSA_ERR_ALIGNMENT, "tree buffer not 256-byte aligned");
    if (bytes < tree_bytes(idx->v, n_super))
        return fail(LSA_ERR_WORKSPACE, "tree buffer %zu < %zu bytes", bytes,
                    tree_bytes(idx->v, n_super));
    cudaError_t e = launch_tree_build(idx->v, idx->n_blk, tree, n_super, lloyd_iters,
                                      (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "tree build");
    return LSA_OK;
}

lsa_status lsa_tree_export(const lsa_index* idx, const void* tree, int n_super, float* sup,
                           void* sup_rt, int32_t* offsets, int32_t* members, void* stream)
{
    if (!idx || !tree || n_super < 1) return fail(LSA_ERR_INVALID_ARG, "NULL argument or n_super < 1");
    cudaError_t e = tree_export(idx->v, tree, n_super, sup, sup_rt, offsets, members,
                                (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "tree export");
    return LSA_OK;
}

size_t lsa_tree_select_workspace_bytes(const lsa_index* idx, int64_t Nq, int branches)
{
    if (!idx || Nq < 0 || branches < 1) return 0;
    return tree_select_ws_bytes(idx->v, Nq, branches);
}

lsa_status lsa_tree_select(const lsa_index* idx, const void* tree, int n_super, int branches,
                           const void* latent_Q, const int32_t* positions, int64_t Nq,
                           lsa_select_params sp, int32_t* indices, int32_t* counts, int s_max,
                           void* workspace, size_t ws_bytes, void* stream)
{
    NvtxRange nv("lsa_tree_select");
    lsa_status s = check_tree(idx, n_super);
    if (s != LSA_OK) return s;
    if (!tree || !latent_Q || !positions || !indices || !counts || !workspace)
        return fail(LSA_ERR_INVALID_ARG, "NULL argument");
    if (branches < 1 || branches > 256 || branches > n_super)
        return fail(LSA_ERR_INVALID_ARG, "branches %d outside [1, min(n_super, 256)]", branches);
    if (Nq < 0 || Nq > 2147483647LL) return fail(LSA_ERR_INVALID_ARG, "Nq out of range");
    s = check_select(idx, sp, s_max);
    if (s != LSA_OK) return s;
    if (((uintptr_t)tree & 255) != 0) return fail(LSA_ERR_ALIGNMENT, "tree buffer not 256-byte aligned");
    if (!aligned16(latent_Q) || !aligned16(positions) || !aligned16(indices) ||
        !aligned16(counts) || !aligned16(workspace))
        return fail(LSA_ERR_ALIGNMENT, "device pointers must be 16-byte aligned");
    const size_t need = tree_select_ws_bytes(idx->v, Nq, branches);
    if (ws_bytes < need) return fail(LSA_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, need);
    if (Nq == 0) return LSA_OK;
    const cudaStream_t st = (cudaStream_t)stream;
    s = dbg_index(idx->v, idx->n_blk, st, "index before tree selection");
    if (s != LSA_OK) return s;
    cudaError_t e = launch_tree_select(idx->v, idx->n_blk, tree, n_super, branches, latent_Q,
                                       positions, Nq, sp, indices, counts, s_max, workspace, st);
    if (e != cudaSuccess) return cuda_fail(e, "tree select");
    return dbg_gather(indices, counts, idx->v.B, Nq, s_max, idx->v.T_cap, PosSrc{positions, 0},
                      sp, DBG_SELECTION, st, "tree selection");
}

lsa_status lsa_sparse_attn(const void* Q, const void* K, const void* V, lsa_dtype dtype, int64_t B,
                           int64_t Nq, int64_t T_cap, int Hq, int Hkv, int d,
                           const int32_t* indices, const int32_t* counts, int s_max, float scale,
                           void* O, float* lse, void* stream)
{
    NvtxRange nv("lsa_sparse_attn");
    if (!Q || !K || !V || !indices || !counts || !O)
        return fail(LSA_ERR_INVALID_ARG, "NULL argument");
    if (dtype != LSA_F32 && dtype != LSA_BF16) return fail(LSA_ERR_INVALID_ARG, "unknown dtype");
    if (B < 1 || Nq < 0 || T_cap < 1 || T_cap > 2147483647LL || s_max < 1)
        return fail(LSA_ERR_INVALID_ARG, "bad sizes");
    lsa_status sh = check_attn_shape(Hq, Hkv, d, dtype);
    if (sh != LSA_OK) return sh;
    if (B * Nq * Hkv > 2147483647LL) return fail(LSA_ERR_UNSUPPORTED, "too many (query, head) pairs");
    if (!(scale > 0.f)) return fail(LSA_ERR_INVALID_ARG, "scale must be > 0");
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(indices) ||
        !aligned16(counts) || !aligned16(O) || (lse && !aligned16(lse)))
        return fail(LSA_ERR_ALIGNMENT, "device pointers must be 16-byte aligned");
    lsa_select_params none{0, 0, 0};
    lsa_status s = dbg_gather(indices, counts, B, Nq, s_max, T_cap, PosSrc{nullptr, 0}, none,
                              DBG_BOUNDS, (cudaStream_t)stream, "gather indices");
    if (s != LSA_OK) return s;
    cudaError_t e = launch_attn(Q, K, V, dtype, B, Nq, T_cap, Hq, Hkv, d, indices, counts, s_max,
                                scale, O, lse, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "sparse attention");
    return LSA_OK;
}

lsa_status lsa_sparse_attn_backward(const void* Q, const void* K, const void* V, const void* O,
                                    const float* lse, const void* dO, lsa_dtype dtype, int64_t B,
                                    int64_t Nq, int64_t T_cap, int Hq, int Hkv, int d,
                                    const int32_t* indices, const int32_t* counts, int s_max,
                                    float scale, void* dQ, float* dK, float* dV, void* stream)
{
    NvtxRange nv("lsa_sparse_attn_backward");
    if (!Q || !K || !V || !O || !lse || !dO || !indices || !counts || !dQ || !dK || !dV)
        return fail(LSA_ERR_INVALID_ARG, "NULL argument");
    if (dtype != LSA_F32 && dtype != LSA_BF16) return fail(LSA_ERR_INVALID_ARG, "unknown dtype");
    if (B < 1 || Nq < 0 || T_cap < 1 || T_cap > 2147483647LL || s_max < 1)
        return fail(LSA_ERR_INVALID_ARG, "bad sizes");
    if (!attn_backward_supported(Hq, Hkv, d))
        return fail(LSA_ERR_UNSUPPORTED, "backward needs Hq %% Hkv == 0, Hq/Hkv <= 8, d <= 128");
    if (B * Nq * Hkv > 2147483647LL) return fail(LSA_ERR_UNSUPPORTED, "too many (query, head) pairs");
    if (!(scale > 0.f)) return fail(LSA_ERR_INVALID_ARG, "scale must be > 0");
    const void* ptrs[] = {Q, K, V, O, lse, dO, indices, counts, dQ, dK, dV};
    for (const void* p : ptrs)
        if (!aligned16(p)) return fail(LSA_ERR_ALIGNMENT, "device pointers must be 16-byte aligned");
    lsa_select_params none{0, 0, 0};
    lsa_status s = dbg_gather(indices, counts, B, Nq, s_max, T_cap, PosSrc{nullptr, 0}, none,
                              DBG_BOUNDS, (cudaStream_t)stream, "gather indices");
    if (s != LSA_OK) return s;
    cudaError_t e = launch_attn_backward(Q, K, V, O, lse, dO, dtype, B, Nq, T_cap, Hq, Hkv, d,
                                         indices, counts, s_max, scale, dQ, dK, dV, nullptr,
                                         (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "sparse attention backward");
    return LSA_OK;
}

// ---- brute-force per-key indexer ----------------------------------------------
namespace {

struct PkLayout {
    size_t status, colmax, theta, cnt, over, gmax, cand, total;
};

PkLayout pk_layout(int64_t B, int64_t Nq, int64_t T_cap)
{
    const size_t rows = (size_t)B * Nq;
    const int64_t ng = per_key_groups(T_cap);
    PkLayout L;
    size_t o = 0;
    L.status = o; o += 256;
    L.colmax = o; o += al256((size_t)B * DL * 4);
    L.theta = o;  o += al256(rows * 4);
    L.cnt = o;    o += al256(rows * 4);
    L.over = o;   o += al256(rows * 4);
    L.gmax = o;   o += al256(rows * ng * 2);
    L.cand = o;   o += al256(rows * PK_CAP * 4);
    L.total = o;
    return L;
}

bool pk_sizes_ok(int64_t B, int64_t Nq, int64_t T_cap)
{
    return B >= 1 && Nq >= 0 && T_cap >= 1 && T_cap <= 2147483647LL &&
           B * T_cap <= 2147483647LL && B * Nq <= 2147483647LL;
}

}  // namespace

size_t lsa_select_per_key_workspace_bytes(int64_t B, int64_t Nq, int64_t T_cap)
{
    if (!pk_sizes_ok(B, Nq, T_cap)) return 0;
    return pk_layout(B, Nq, T_cap).total;
}

lsa_status lsa_select_per_key(const void* latent_K, lsa_dtype dtype, int64_t B, int64_t T_cap,
                              int64_t n_keys, const void* latent_Q, const int32_t* positions,
                              int64_t Nq, lsa_select_params sp, int32_t* indices, int32_t* counts,
                              int s_max, void* workspace, size_t ws_bytes, void* stream)
{
    NvtxRange nv("lsa_select_per_key");
    if (!latent_K || !latent_Q || !positions || !indices || !counts || !workspace)
        return fail(LSA_ERR_INVALID_ARG, "NULL argument");
    if (dtype != LSA_F32 && dtype != LSA_BF16) return fail(LSA_ERR_INVALID_ARG, "unknown dtype");
    if (dtype != LSA_BF16)
        return fail(LSA_ERR_UNSUPPORTED, "the per-key indexer scores bf16 latents only");
    if (!pk_sizes_ok(B, Nq, T_cap) || n_keys < 0 || n_keys > T_cap)
        return fail(LSA_ERR_INVALID_ARG, "bad sizes (B*T_cap and B*Nq below 2^31, n_keys <= T_cap)");
    if (sp.budget < 0 || sp.window < 0 || sp.sinks < 0)
        return fail(LSA_ERR_INVALID_ARG, "budget, window and sinks must be >= 0");
    if (sp.budget > PK_MAX_R)
        return fail(LSA_ERR_UNSUPPORTED, "budget %d > %d", sp.budget, PK_MAX_R);
    if ((int64_t)sp.budget + sp.window + sp.sinks > (int64_t)s_max)
        return fail(LSA_ERR_INVALID_ARG, "s_max=%d < budget + window + sinks", s_max);
    if (ws_bytes < lsa_select_per_key_workspace_bytes(B, Nq, T_cap))
        return fail(LSA_ERR_WORKSPACE, "workspace too small");
    if (!aligned16(latent_K) || !aligned16(latent_Q) || !aligned16(positions) ||
        !aligned16(indices) || !aligned16(counts) || !aligned16(workspace))
        return fail(LSA_ERR_ALIGNMENT, "device pointers must be 16-byte aligned");
    const cudaStream_t st = (cudaStream_t)stream;
    const PkLayout L = pk_layout(B, Nq, T_cap);
    char* w = (char*)workspace;
    cudaError_t e = cudaMemsetAsync(w, 0, L.theta, st);          // status words and colmax
    if (e != cudaSuccess) return cuda_fail(e, "per-key indexer");
    if (Nq == 0) return LSA_OK;
    PerKeyArgs a;
    a.lat_k = latent_K;
    a.lat_q = latent_Q;
    a.pos = positions;
    a.B = B;
    a.T_cap = T_cap;
    a.n_keys = n_keys;
    a.Nq = Nq;
    a.R = sp.budget;
    a.W = sp.window;
    a.S = sp.sinks;
    a.indices = indices;
    a.counts = counts;
    a.s_max = s_max;
    PerKeyWs ws;
    ws.status = (uint32_t*)(w + L.status);
    ws.colmax = (uint32_t*)(w + L.colmax);
    ws.theta = (float*)(w + L.theta);
    ws.cnt = (int32_t*)(w + L.cnt);
    ws.over = (int32_t*)(w + L.over);
    ws.gmax = (uint16_t*)(w + L.gmax);
    ws.cand = (int32_t*)(w + L.cand);
    ws.ng = per_key_groups(T_cap);
    e = launch_per_key(a, ws, st);
    if (e != cudaSuccess) return cuda_fail(e, "per-key indexer");
    return dbg_gather(indices, counts, B, Nq, s_max, T_cap, PosSrc{positions, 0}, sp,
                      DBG_SELECTION_SORTED, st, "per-key selection");
}

lsa_status lsa_select_per_key_check(const void* workspace, int64_t* fallbacks, void* stream)
{
    if (!workspace) return fail(LSA_ERR_INVALID_ARG, "NULL workspace");
    cudaStream_t st = (cudaStream_t)stream;
    uint32_t h[8] = {0};
    cudaError_t e = cudaMemcpyAsync(h, workspace, sizeof(h), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "per-key check");
    if (fallbacks) *fallbacks = (int64_t)h[1];
    switch (h[0]) {
    case DEV_OK: return LSA_OK;
    case DEV_BAD_INDEX:
        return fail(LSA_ERR_INVALID_ARG, "a query position (%d) was outside [0, n_keys)", (int)h[2]);
    case DEV_TIMEOUT:
        return fail(LSA_ERR_TIMEOUT, "a bounded wait gave up (site %u)", h[2]);
    default: return fail(LSA_ERR_INTERNAL, "device status %u (detail %u)", h[0], h[2]);
    }
}

size_t lsa_attend_key_range_workspace_bytes(int64_t B, int64_t Nq, int s_max)
{
    if (B < 1 || Nq < 0 || s_max < 1) return 0;
    return al256((size_t)B * Nq * s_max * 4) + al256((size_t)B * Nq * 4);
}

lsa_status lsa_attend_key_range(const void* Q, const void* K_shard, const void* V_shard,
                                lsa_dtype dtype, int64_t B, int64_t Nq, int Hq, int Hkv, int d,
                                const int32_t* indices, const int32_t* counts, int s_max,
                                int64_t key_lo, int64_t key_hi, float scale, void* workspace,
                                size_t ws_bytes, void* O_part, float* lse_part, void* stream)
{
    NvtxRange nv("lsa_attend_key_range");
    if (!Q || !K_shard || !V_shard || !indices || !counts || !O_part || !lse_part || !workspace)
        return fail(LSA_ERR_INVALID_ARG, "NULL argument");
    if (dtype != LSA_F32 && dtype != LSA_BF16) return fail(LSA_ERR_INVALID_ARG, "unknown dtype");
    if (B < 1 || Nq < 0 || s_max < 1 || key_lo < 0 || key_hi <= key_lo ||
        key_hi - key_lo > 2147483647LL)
        return fail(LSA_ERR_INVALID_ARG, "bad sizes or key range");
    lsa_status sh = check_attn_shape(Hq, Hkv, d, dtype);
    if (sh != LSA_OK) return sh;
    if (B * Nq * Hkv > 2147483647LL) return fail(LSA_ERR_UNSUPPORTED, "too many (query, head) pairs");
    if (!(scale > 0.f)) return fail(LSA_ERR_INVALID_ARG, "scale must be > 0");
    if (ws_bytes < lsa_attend_key_range_workspace_bytes(B, Nq, s_max))
        return fail(LSA_ERR_WORKSPACE, "workspace too small");
    if (!aligned16(Q) || !aligned16(K_shard) || !aligned16(V_shard) || !aligned16(indices) ||
        !aligned16(counts) || !aligned16(O_part) || !aligned16(lse_part) || !aligned16(workspace))
        return fail(LSA_ERR_ALIGNMENT, "device pointers must be 16-byte aligned");
    if (Nq == 0) return LSA_OK;
    const cudaStream_t st = (cudaStream_t)stream;
    int32_t* loc_idx = (int32_t*)workspace;
    int32_t* loc_cnt = (int32_t*)((char*)workspace + al256((size_t)B * Nq * s_max * 4));
    cudaError_t e = launch_range_filter(indices, counts, B * Nq, s_max, key_lo, key_hi, loc_idx,
                                        loc_cnt, st);
    if (e == cudaSuccess)
        e = launch_attn(Q, K_shard, V_shard, dtype, B, Nq, key_hi - key_lo, Hq, Hkv, d, loc_idx,
                        loc_cnt, s_max, scale, O_part, lse_part, st);
    if (e == cudaSuccess) e = launch_range_empty(loc_cnt, B * Nq, Hq, d, dtype, O_part, lse_part, st);
    if (e != cudaSuccess) return cuda_fail(e, "key-range attention");
    return LSA_OK;
}

lsa_status lsa_merge_partials(const void* O_parts, const float* lse_parts, lsa_dtype dtype,
                              int n_parts, int64_t rows, int Hq, int d, void* O, float* lse,
                              void* stream)
{
    NvtxRange nv("lsa_merge_partials");
    if (!O_parts || !lse_parts || !O) return fail(LSA_ERR_INVALID_ARG, "NULL argument");
    if (dtype != LSA_F32 && dtype != LSA_BF16) return fail(LSA_ERR_INVALID_ARG, "unknown dtype");
    if (n_parts < 1 || n_parts > 32 || rows < 0 || Hq < 1 || d < 1 || d > 1024)
        return fail(LSA_ERR_INVALID_ARG, "bad sizes (1 <= n_parts <= 32)");
    if (!aligned16(O_parts) || !aligned16(lse_parts) || !aligned16(O) || (lse && !aligned16(lse)))
        return fail(LSA_ERR_ALIGNMENT, "device pointers must be 16-byte aligned");
    cudaError_t e = launch_merge_partials(O_parts, lse_parts, dtype, n_parts, rows, Hq, d, O, lse,
                                          (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "merge of partials");
    return LSA_OK;
}

size_t lsa_prefill_workspace_bytes(const lsa_index* idx, int64_t Nq, int Hq, int Hkv, int d,
                                   lsa_select_params sp)
{
    if (!idx || Nq < 0 || sp.budget < 0 || sp.window < 0 || sp.sinks < 0) return 0;
    if (Hq < 1 || Hkv < 1 || d < 1) return 0;
    return prefill_layout(idx, Nq, Hq, Hkv, d, sp, default_ent_cap(idx, Nq, sp)).total;
}

int64_t lsa_prefill_partial_slots(const lsa_index* idx, int64_t Nq, int Hq, int Hkv, int d,
                                  lsa_select_params sp, size_t ws_bytes)
{
    if (!idx || Nq < 0 || sp.budget < 0 || sp.window < 0 || sp.sinks < 0) return -1;
    if (Hq < 1 || Hkv < 1 || d < 1) return -1;
    return ent_cap_for(idx, Nq, Hq, Hkv, d, sp, ws_bytes);
}

namespace {

// Checks shared by the prefill entries; fills the layout and the plan view.
lsa_status prefill_prepare(const lsa_index* idx, int64_t Nq, int Hq, int Hkv, int d,
                           lsa_select_params sp, void* workspace, size_t ws_bytes,
                           PrefillLayout* L, BucketPlan* P)
{
    if (Nq < 1) return fail(LSA_ERR_INVALID_ARG, "empty chunk");
    const int s_max = sp.budget + sp.window + sp.sinks;
    lsa_status s = check_select(idx, sp, s_max);
    if (s != LSA_OK) return s;
    // attention shape checks up front so that nothing launches on bad input
    s = check_attn_shape(Hq, Hkv, d, idx->v.dtype);
    if (s != LSA_OK) return s;
    const int64_t ent_cap = ent_cap_for(idx, Nq, Hq, Hkv, d, sp, ws_bytes);
    if (ent_cap < 0)
        return fail(LSA_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes,
                    prefill_layout(idx, Nq, Hq, Hkv, d, sp, 0).total);
    if (!aligned16(workspace)) return fail(LSA_ERR_ALIGNMENT, "workspace not 16-byte aligned");
    *L = prefill_layout(idx, Nq, Hq, Hkv, d, sp, ent_cap);
    if (L->bucket && (idx->v.B * Nq * (int64_t)(KC + 1) > 2147483647LL ||
                      idx->v.B * idx->v.NBK > 2147483647LL))
        return fail(LSA_ERR_UNSUPPORTED, "chunk too large for the bucket lists");
    char* base = (char*)workspace;
    *P = BucketPlan{};
    if (L->bucket) {
        P->zero = (int32_t*)(base + L->zero);
        P->n_zero = L->n_zero;
        P->bucket_cnt = P->zero;
        P->ctr = P->zero + idx->v.B * idx->v.NBK;
        P->row_n = (int32_t*)(base + L->row_n);
        P->row_base = (int32_t*)(base + L->row_base);
        P->gather_rows = (int32_t*)(base + L->gather);
        P->ent = (int4*)(base + L->ent);
        P->ent2 = (int2*)(base + L->ent2);
        P->ent_cap = L->ent_cap;
        P->bucket_off = (int32_t*)(base + L->bucket_off);
        P->tiles = (int2*)(base + L->tiles);
        P->tile_cap = L->tile_cap;
        P->sorted = (int32_t*)(base + L->sorted);
        P->part_o = (__nv_bfloat16*)(base + L->part);
        P->part_ml = (float2*)(base + L->part_ml);
        P->recs = (unsigned char*)(base + L->recs);
    }
    return LSA_OK;
}

}  // namespace

namespace {

// Chunk queries [q0, q1) of positions [T_old, T_new): the query at row r sits
// at position T_old + q0 + r.
lsa_status query_range(int64_t T_old, int64_t T_new, int64_t q0, int64_t q1)
{
    if (T_old < 0 || T_new <= T_old) return fail(LSA_ERR_INVALID_ARG, "empty chunk");
    if (q0 < 0 || q1 <= q0 || q1 > T_new - T_old)
        return fail(LSA_ERR_INVALID_ARG, "query range [%lld, %lld) outside the chunk of %lld",
                    (long long)q0, (long long)q1, (long long)(T_new - T_old));
    return LSA_OK;
}

lsa_status select_part(lsa_index* idx, const void* latent_K, const void* latent_Q, int64_t T_old,
                       int64_t T_new, int64_t q0, int64_t q1, int Hq, int Hkv, int d,
                       lsa_select_params sp, void* workspace, size_t ws_bytes, void* stream)
{
    if (!idx || !latent_K || !latent_Q || !workspace)
        return fail(LSA_ERR_INVALID_ARG, "NULL argument");
    lsa_status s = query_range(T_old, T_new, q0, q1);
    if (s != LSA_OK) return s;
    PrefillLayout L;
    BucketPlan P;
    s = prefill_prepare(idx, q1 - q0, Hq, Hkv, d, sp, workspace, ws_bytes, &L, &P);
    if (s != LSA_OK) return s;
    if (!aligned16(latent_Q)) return fail(LSA_ERR_ALIGNMENT, "latent_Q not 16-byte aligned");
    cudaStream_t st = (cudaStream_t)stream;
    s = lsa_index_extend(idx, latent_K, T_old, T_new, stream);
    if (s != LSA_OK) return s;
    char* base = (char*)workspace;
    const int s_max = sp.budget + sp.window + sp.sinks;
    return run_select(idx, latent_Q, PosSrc{nullptr, T_old + q0}, q1 - q0, sp,
                      (int32_t*)(base + L.indices), (int32_t*)(base + L.counts), s_max,
                      base + L.sel, st, L.bucket ? &P : nullptr);
}

lsa_status attend_part(const lsa_index* idx, const void* Q, const void* K, const void* V,
                       int64_t T_old, int64_t T_new, int64_t q0, int64_t q1, int Hq, int Hkv,
                       int d, lsa_select_params sp, void* workspace, size_t ws_bytes, void* O,
                       void* stream)
{
    if (!idx || !Q || !K || !V || !workspace || !O)
        return fail(LSA_ERR_INVALID_ARG, "NULL argument");
    lsa_status s = query_range(T_old, T_new, q0, q1);
    if (s != LSA_OK) return s;
    PrefillLayout L;
    BucketPlan P;
    s = prefill_prepare(idx, q1 - q0, Hq, Hkv, d, sp, workspace, ws_bytes, &L, &P);
    if (s != LSA_OK) return s;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O))
        return fail(LSA_ERR_ALIGNMENT, "Q, K, V and O must be 16-byte aligned");
    cudaStream_t st = (cudaStream_t)stream;
    const int64_t Nq = q1 - q0;
    const int s_max = sp.budget + sp.window + sp.sinks;
    char* base = (char*)workspace;
    const int32_t* indices = (const int32_t*)(base + L.indices);
    const int32_t* counts = (const int32_t*)(base + L.counts);
    const float scale = (float)(1.0 / sqrt((double)d));
    s = dbg_gather(indices, counts, idx->v.B, Nq, s_max, idx->v.T_cap, PosSrc{nullptr, T_old + q0},
                   sp, DBG_SELECTION, st, "chunk selection before attention");
    if (s != LSA_OK) return s;
    cudaError_t e;
    if (L.bucket)
        e = launch_bucket_attn(idx->v, idx->n_blk, P, Q, K, V, Nq, Hq, Hkv, d,
                               PosSrc{nullptr, T_old + q0}, sp.window, sp.sinks, indices, counts,
                               s_max, scale, O, st);
    else
        e = launch_attn_status(Q, K, V, idx->v.dtype, idx->v.B, Nq, idx->v.T_cap, Hq, Hkv, d,
                               indices, counts, s_max, scale, O, nullptr, idx->v.status, st);
    if (e != cudaSuccess) return cuda_fail(e, "sparse attention");
    return LSA_OK;
}

lsa_status chunk_part(lsa_index* idx, const void* latent_K, const void* latent_Q, const void* Q,
                      const void* K, const void* V, int64_t T_old, int64_t T_new, int64_t q0,
                      int64_t q1, int Hq, int Hkv, int d, lsa_select_params sp, void* workspace,
                      size_t ws_bytes, void* O, void* stream)
{
    if (!idx || !latent_K || !latent_Q || !Q || !K || !V || !workspace || !O)
        return fail(LSA_ERR_INVALID_ARG, "NULL argument");
    lsa_status s = query_range(T_old, T_new, q0, q1);
    if (s != LSA_OK) return s;
    PrefillLayout L;
    BucketPlan P;
    // every argument check of both halves before the first launch
    s = prefill_prepare(idx, q1 - q0, Hq, Hkv, d, sp, workspace, ws_bytes, &L, &P);
    if (s != LSA_OK) return s;
    if (!aligned16(latent_Q) || !aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O))
        return fail(LSA_ERR_ALIGNMENT, "device pointers must be 16-byte aligned");
    s = select_part(idx, latent_K, latent_Q, T_old, T_new, q0, q1, Hq, Hkv, d, sp, workspace,
                    ws_bytes, stream);
    if (s != LSA_OK) return s;
    return attend_part(idx, Q, K, V, T_old, T_new, q0, q1, Hq, Hkv, d, sp, workspace, ws_bytes, O,
                       stream);
}

}  // namespace

lsa_status lsa_prefill_select(lsa_index* idx, const void* latent_K, const void* latent_Q,
                              int64_t T_old, int64_t T_new, int Hq, int Hkv, int d,
                              lsa_select_params sp, void* workspace, size_t ws_bytes, void* stream)
{
    NvtxRange nv("lsa_prefill_select");
    return select_part(idx, latent_K, latent_Q, T_old, T_new, 0, T_new - T_old, Hq, Hkv, d, sp,
                       workspace, ws_bytes, stream);
}

lsa_status lsa_prefill_attend(const lsa_index* idx, const void* Q, const void* K, const void* V,
                              int64_t T_old, int64_t T_new, int Hq, int Hkv, int d,
                              lsa_select_params sp, void* workspace, size_t ws_bytes, void* O,
                              void* stream)
{
    NvtxRange nv("lsa_prefill_attend");
    return attend_part(idx, Q, K, V, T_old, T_new, 0, T_new - T_old, Hq, Hkv, d, sp, workspace,
                       ws_bytes, O, stream);
}

lsa_status lsa_prefill_chunk(lsa_index* idx, const void* latent_K, const void* latent_Q,
                             const void* Q, const void* K, const void* V, int64_t T_old,
                             int64_t T_new, int Hq, int Hkv, int d, lsa_select_params sp,
                             void* workspace, size_t ws_bytes, void* O, void* stream)
{
    NvtxRange nv("lsa_prefill_chunk");
    return chunk_part(idx, latent_K, latent_Q, Q, K, V, T_old, T_new, 0, T_new - T_old, Hq, Hkv,
                      d, sp, workspace, ws_bytes, O, stream);
}

lsa_status lsa_prefill_chunk_queries(lsa_index* idx, const void* latent_K, const void* latent_Q,
                                     const void* Q, const void* K, const void* V, int64_t T_old,
                                     int64_t T_new, int64_t q_begin, int64_t q_end, int Hq,
                                     int Hkv, int d, lsa_select_params sp, void* workspace,
                                     size_t ws_bytes, void* O, void* stream)
{
    NvtxRange nv("lsa_prefill_chunk_queries");
    return chunk_part(idx, latent_K, latent_Q, Q, K, V, T_old, T_new, q_begin, q_end, Hq, Hkv, d,
                      sp, workspace, ws_bytes, O, stream);
}

lsa_status lsa_prefill_chunk_host(lsa_index* idx, const void* h_latent_K, const void* h_K,
                                  const void* h_V, const void* h_latent_Q, const void* h_Q,
                                  void* latent_K, void* K, void* V, void* latent_Q, void* Q,
                                  int64_t T_old, int64_t T_new, int Hq, int Hkv, int d,
                                  lsa_select_params sp, void* workspace, size_t ws_bytes,
                                  void* O, void* h_O, void* stream, void* copy_stream)
{
    NvtxRange nv("lsa_prefill_chunk_host");
    if (!idx || !h_latent_K || !h_K || !h_V || !h_latent_Q || !h_Q || !latent_K || !K || !V ||
        !latent_Q || !Q || !O || !h_O)
        return fail(LSA_ERR_INVALID_ARG, "NULL argument");
    if (stream == copy_stream) return fail(LSA_ERR_INVALID_ARG, "copy_stream must differ from stream");
    PrefillLayout L;
    BucketPlan P;
    lsa_status s = prefill_prepare(idx, T_new - T_old, Hq, Hkv, d, sp, workspace, ws_bytes, &L, &P);
    if (s != LSA_OK) return s;
    if (!aligned16(latent_K) || !aligned16(latent_Q) || !aligned16(Q) || !aligned16(K) ||
        !aligned16(V) || !aligned16(O))
        return fail(LSA_ERR_ALIGNMENT, "device pointers must be 16-byte aligned");
    const IndexView& v = idx->v;
    const size_t es = (v.dtype == LSA_BF16) ? 2 : 4;
    const int64_t Nq = T_new - T_old, B = v.B;
    const size_t lat_row = (size_t)DL * es, kv_row = (size_t)Hkv * d * es;
    cudaStream_t st = (cudaStream_t)stream, cs = (cudaStream_t)copy_stream;
    // one pair of events per host thread and device, reused call after call
    constexpr int MAX_DEV = 64;
    static thread_local cudaEvent_t evs[MAX_DEV][2] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "current device");
    if (dev < 0 || dev >= MAX_DEV) return fail(LSA_ERR_UNSUPPORTED, "device %d", dev);
    cudaEvent_t& ev_in = evs[dev][0];
    cudaEvent_t& ev_kvq = evs[dev][1];
    if (!ev_in) e = cudaEventCreateWithFlags(&ev_in, cudaEventDisableTiming);
    if (e == cudaSuccess && !ev_kvq) e = cudaEventCreateWithFlags(&ev_kvq, cudaEventDisableTiming);
    if (e != cudaSuccess) return cuda_fail(e, "event create");
    // the copy stream starts after the work already queued on stream (which
    // may still read the caches and Q)
    e = cudaEventRecord(ev_in, st);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(cs, ev_in, 0);
    // the latent rows first, on stream: the extension and the selection need them
    for (int64_t b = 0; b < B && e == cudaSuccess; ++b)
        e = cudaMemcpyAsync((char*)latent_K + ((size_t)b * v.T_cap + T_old) * lat_row,
                            (const char*)h_latent_K + (size_t)b * Nq * lat_row, Nq * lat_row,
                            cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(latent_Q, h_latent_Q, (size_t)B * Nq * lat_row, cudaMemcpyHostToDevice,
                            st);
    // K, V and Q on the copy stream, under the selection
    for (int64_t b = 0; b < B && e == cudaSuccess; ++b) {
        const size_t dst = ((size_t)b * v.T_cap + T_old) * kv_row, src = (size_t)b * Nq * kv_row;
        e = cudaMemcpyAsync((char*)K + dst, (const char*)h_K + src, Nq * kv_row,
                            cudaMemcpyHostToDevice, cs);
        if (e == cudaSuccess)
            e = cudaMemcpyAsync((char*)V + dst, (const char*)h_V + src, Nq * kv_row,
                                cudaMemcpyHostToDevice, cs);
    }
    const size_t q_bytes = (size_t)B * Nq * Hq * d * es;
    if (e == cudaSuccess) e = cudaMemcpyAsync(Q, h_Q, q_bytes, cudaMemcpyHostToDevice, cs);
    if (e == cudaSuccess) e = cudaEventRecord(ev_kvq, cs);
    if (e != cudaSuccess) return cuda_fail(e, "host-to-device copies");
    s = lsa_prefill_select(idx, latent_K, latent_Q, T_old, T_new, Hq, Hkv, d, sp, workspace,
                           ws_bytes, stream);
    if (s != LSA_OK) return s;
    e = cudaStreamWaitEvent(st, ev_kvq, 0);
    if (e != cudaSuccess) return cuda_fail(e, "copy join");
    s = lsa_prefill_attend(idx, Q, K, V, T_old, T_new, Hq, Hkv, d, sp, workspace, ws_bytes, O,
                           stream);
    if (s != LSA_OK) return s;
    e = cudaMemcpyAsync(h_O, O, q_bytes, cudaMemcpyDeviceToHost, st);
    if (e != cudaSuccess) return cuda_fail(e, "device-to-host copy");
    return LSA_OK;
}

lsa_status lsa_set_wait_limit(int64_t polls)
{
    cudaError_t e = set_score_wait_polls(polls);
    if (e == cudaSuccess) e = set_tile_wait_polls(polls);
    if (e == cudaSuccess) e = set_attn_wait_polls(polls);
    if (e == cudaSuccess) e = set_per_key_wait_polls(polls);
    if (e != cudaSuccess) return cuda_fail(e, "wait limit");
    return LSA_OK;
}

size_t lsa_decode_workspace_bytes(const lsa_index* idx, int Hq, int Hkv, int d,
                                  lsa_select_params sp)
{
    if (!idx || sp.budget < 0 || sp.window < 0 || sp.sinks < 0) return 0;
    if (check_attn_shape(Hq, Hkv, d, idx->v.dtype) != LSA_OK) return 0;
    return decode_layout(idx, Hq, Hkv, d, sp).total;
}

lsa_status lsa_decode_step(lsa_index* idx, void* latent_K, void* K, void* V,
                           const void* new_latent_k, const void* new_k, const void* new_v,
                           const void* latent_q, const void* q, const int32_t* pos, int Hq,
                           int Hkv, int d, lsa_select_params sp, void* workspace, size_t ws_bytes,
                           void* O, void* stream)
{
    NvtxRange nv("lsa_decode_step");
    if (!idx || !latent_K || !K || !V || !new_latent_k || !new_k || !new_v || !latent_q || !q ||
        !pos || !workspace || !O)
        return fail(LSA_ERR_INVALID_ARG, "NULL argument");
    const IndexView& v = idx->v;
    const int s_max = sp.budget + sp.window + sp.sinks;
    lsa_status s = check_select(idx, sp, s_max);
    if (s != LSA_OK) return s;
    s = check_attn_shape(Hq, Hkv, d, v.dtype);
    if (s != LSA_OK) return s;
    if (idx->n_blk < 1 || idx->n_blk * v.G >= v.NP)
        return fail(LSA_ERR_INVALID_ARG,
                    "decode needs at least one closed block and room for an open block");
    const void* ptrs[] = {latent_K, K, V, new_latent_k, new_k, new_v, latent_q, q, pos, workspace, O};
    for (const void* p : ptrs)
        if (!aligned16(p)) return fail(LSA_ERR_ALIGNMENT, "device pointers must be 16-byte aligned");
    const DecodeLayout L = decode_layout(idx, Hq, Hkv, d, sp);
    if (ws_bytes < L.total)
        return fail(LSA_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, L.total);
    cudaStream_t st = (cudaStream_t)stream;
    char* base = (char*)workspace;
    int32_t* indices = (int32_t*)(base + L.indices);
    int32_t* counts = (int32_t*)(base + L.counts);
    SelectWs w = select_ws_carve(base + L.sel, v, 1);
    // the fill merges the slices' lists the prep pass writes, and finishes
    // the prep pass's append
    w.dl_s = (float*)(base + L.dl_s);
    w.dl_g = (int32_t*)(base + L.dl_g);
    w.dl_n = (int32_t*)(base + L.dl_n);
    w.dl_tau = (float*)(base + L.dl_tau);
    w.n_slice = L.n_slice;
    double* app_score = (double*)(base + L.app_score);
    int32_t* app_g = (int32_t*)(base + L.app_g);
    int32_t* app_slot = (int32_t*)(base + L.app_slot);
    w.app_score = app_score;
    w.app_g = app_g;
    w.app_slot = app_slot;
    w.app_n = L.n_slice;
    float* part = (float*)(base + L.part);
    uint32_t* counter = (uint32_t*)(base + L.counter);
    if (!idx->status_clean) {
        cudaError_t e = cudaMemsetAsync(v.status, 0, 8 * sizeof(uint32_t), st);
        if (e != cudaSuccess) return cuda_fail(e, "status clear");
        idx->status_clean = true;
    }
    s = dbg_index(v, idx->n_blk, st, "index before decode step");
    if (s != LSA_OK) return s;
    cudaError_t e = launch_decode_prep(v, idx->n_blk, latent_K, K, V, new_latent_k, new_k, new_v,
                                       latent_q, pos, Hkv, d, sp.window, w, app_score, app_g,
                                       app_slot, L.n_slice, counter, L.n_hg, st);
    if (e != cudaSuccess) return cuda_fail(e, "decode append/nominate");
    e = launch_decode_finish(v, idx->n_blk, latent_q, pos, sp, indices, counts, s_max, w, st);
    if (e != cudaSuccess) return cuda_fail(e, "decode select");
    const float scale = (float)(1.0 / sqrt((double)d));
    if (v.dtype == LSA_BF16)
    {
        e = launch_attn_split(q, K, V, v.B, 1, v.T_cap, Hq, Hkv, d, indices, counts, s_max, scale,
                              O, nullptr, v.status, L.ns, L.kps, part, nullptr, 0, st);
        if (e == cudaSuccess && L.ns > 1)
            e = launch_attn_combine(part, L.ns, v.B, Hq, d, O, nullptr, st);
    }
    else
        e = launch_attn_status(q, K, V, v.dtype, v.B, 1, v.T_cap, Hq, Hkv, d, indices, counts,
                               s_max, scale, O, nullptr, v.status, st);
    if (e != cudaSuccess) return cuda_fail(e, "decode attention");
    return LSA_OK;
}

lsa_status lsa_select_noalloc(const lsa_index* idx, const void* latent_Q,
                              const int32_t* positions, int64_t Nq, lsa_select_params sp,
                              int32_t* indices, int32_t* counts, int s_max, void* stream)
{
    NvtxRange nv("lsa_select_noalloc");
    if (!idx || !latent_Q || !positions || !indices || !counts)
        return fail(LSA_ERR_INVALID_ARG, "NULL argument");
    if (Nq < 0 || Nq > 2147483647LL) return fail(LSA_ERR_INVALID_ARG, "Nq out of range");
    lsa_status s = check_select(idx, sp, s_max);
    if (s != LSA_OK) return s;
    if (!aligned16(latent_Q) || !aligned16(positions) || !aligned16(indices) || !aligned16(counts))
        return fail(LSA_ERR_ALIGNMENT, "device pointers must be 16-byte aligned");
    const size_t need = select_ws_bytes(idx->v, Nq);
    if (need > noalloc_scratch_bytes())
        return fail(LSA_ERR_WORKSPACE,
                    "selection of %lld queries over this index needs %zu bytes of scratch; the "
                    "built-in array holds %zu: use lsa_select with a caller workspace",
                    (long long)Nq, need, noalloc_scratch_bytes());
    const bool tc = use_tc_path(idx, Nq);
    if (!tc && idx->n_blk * idx->v.k > SIMT_MAX_BUCKETS)
        return fail(LSA_ERR_UNSUPPORTED, "%lld buckets exceed the SIMT scorer's %lld",
                    (long long)(idx->n_blk * idx->v.k), (long long)SIMT_MAX_BUCKETS);
    if (Nq == 0) return LSA_OK;
    const cudaStream_t st = (cudaStream_t)stream;
    s = dbg_index(idx->v, idx->n_blk, st, "index before selection");
    if (s != LSA_OK) return s;
    cudaError_t e = noalloc_select(idx->v, idx->n_blk, latent_Q, positions, Nq, sp, indices,
                                   counts, s_max, tc, st);
    if (e != cudaSuccess) return cuda_fail(e, "select (built-in scratch)");
    return dbg_gather(indices, counts, idx->v.B, Nq, s_max, idx->v.T_cap, PosSrc{positions, 0},
                      sp, DBG_SELECTION, st, "selection");
}

}  // extern "C"
