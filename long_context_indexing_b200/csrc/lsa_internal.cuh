// lsa_internal.cuh -- shared declarations of liblsa's CUDA sources.
//
// Index layout in the caller's device buffer (per array, B sequences
// back to back; every array starts on a 256-byte boundary):
//   pooled   f32 [B][NP][64]     x_j, mean of p consecutive latent keys
//   unit     f32 [B][NP][64]     u_j = x_j / ||x_j||
//   cent     f32 [B][NBK][64]    centroids, g = b*k + m
//   cent_rt  T   [B][NBK][64]    retrieval copy (bf16 or f32)
//   offsets  i32 [B][NBK+1]      CSR offsets (global pooled positions)
//   members  i32 [B][NP]         pooled ids, ascending inside a bucket
//   assign   i16 [B][NP]         bucket m inside the block
//   open     i32 [B][G]          bucket of each completed open-block group, -1 if none
//   status   u32 [8]             [0] first error code, [1] fallback count,
//                                [2] error detail
// with NP = T_cap / p pooled groups and NBK = (NP / G) * k buckets.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "lsa.h"

namespace lsa {

constexpr int DL = 64;         // latent dimension (the pages' 64-d index)
constexpr int KC = 64;         // candidate buckets nominated per query
constexpr int MAX_K = 32;      // buckets per block supported by the kernels

// Device-visible view of an index (passed by value to kernels).
struct IndexView {
    int64_t B;
    int64_t T_cap;
    int64_t NP;        // pooled groups per sequence (capacity)
    int64_t NBK;       // buckets per sequence (capacity)
    int p, G, k, L;
    int nblk_max;
    lsa_dtype dtype;
    float* pooled;
    float* unit;
    float* cent;
    void* cent_rt;
    int32_t* offsets;
    int32_t* members;
    int16_t* assign;
    int32_t* open_bucket;
    uint32_t* status;
};

// Where a query's position comes from: an int32 array [B][Nq] or base + i.
struct PosSrc {
    const int32_t* arr;
    int64_t base;
    __host__ __device__ int64_t at(int64_t b, int64_t nq, int64_t i) const
    {
        return arr ? (int64_t)arr[b * nq + i] : base + i;
    }
};

// Status codes written by kernels (first one wins).
enum DevErr : uint32_t {
    DEV_OK = 0,
    DEV_OPEN_FULL = 1,     // decode append found the open block full
    DEV_BAD_INDEX = 2,     // an index outside [0, T_cap) reached a gather
    DEV_FALLBACK_OVF = 3,  // fallback list overflow (cannot happen by sizing)
    DEV_TIMEOUT = 4,       // a bounded wait on a copy gave up
};

__device__ __forceinline__ void dev_error(uint32_t* status, uint32_t code, uint32_t detail)
{
    if (atomicCAS(status, 0u, code) == 0u) status[2] = detail;
}

// Host-side count of kernel launches enqueued by the library (all threads).
void note_launch();

// Streaming multiprocessors of the current device (148 when it cannot be read).
int sm_count();

__device__ __forceinline__ float load_elt(const float* p) { return *p; }
__device__ __forceinline__ float load_elt(const __nv_bfloat16* p) { return __bfloat162float(*p); }

// ---------------------------------------------------------------------------
// Launchers (each enqueues on `st`; returns cudaGetLastError()).
// ---------------------------------------------------------------------------

// Pool + normalise pooled groups [j0, j1) of every sequence.
cudaError_t launch_pool_unit(const IndexView& ix, const void* latent_K, int64_t j0, int64_t j1,
                             cudaStream_t st);

// Spherical k-means of blocks [b0, b1) of every sequence (L Lloyd iterations),
// CSR records and the retrieval copy.  Needs `unit` of those blocks.
cudaError_t launch_kmeans(const IndexView& ix, int64_t b0, int64_t b1, cudaStream_t st);

// Reset the open block (every slot -1) and assign its completed groups
// [n_blk*G, j_end) to their nearest closed centroid.  Needs `unit` rows.
cudaError_t launch_open_assign(const IndexView& ix, int64_t n_blk, int64_t j_end,
                               cudaStream_t st);

// Lists for bucket-major attention, written by the selection fill (bf16
// prefill only; row_n == nullptr turns them off).  Every query row that the
// fill ranks exactly and that finds room gets nt + 1 consecutive partial
// slots: slot base + t for its t-th taken bucket, base + nt for its sinks and
// recent window.  Other rows (exact fallback, no room) are listed in
// gather_rows and attended key by key.
enum PlanCtr : int {
    CTR_RESERVED = 0,   // partial slots handed out (may pass ent_cap)
    CTR_VALID_END = 1,  // end of the slots actually granted
    CTR_GATHER = 2,     // rows in gather_rows
    CTR_WORK = 3,       // work counter of the persistent attention kernel
    CTR_TILES = 4,      // bucket tiles built by the plan kernel
    CTR_N = 8
};
struct BucketPlan {
    int32_t* zero;        // [n_zero] cleared by the scorer: bucket_cnt then ctr
    int64_t n_zero;
    int32_t* bucket_cnt;  // [B*NBK] taken entries per bucket
    int32_t* ctr;         // [CTR_N]
    int32_t* row_n;       // [rows] buckets taken by a listed row, -1 = gather row
    int32_t* row_base;    // [rows] first partial slot of the row
    int32_t* gather_rows; // [rows]
    int4* ent;            // [ent_cap] (row, sequence-level bucket b*NBK+g or -1, lo, hi)
    int2* ent2;           // [ent_cap] (rank of the entry inside its bucket, open keys taken)
    int64_t ent_cap;
    int32_t* bucket_off;  // [B*NBK] first sorted position of each bucket
    int2* tiles;          // [tile_cap] (bucket, tile number inside the bucket)
    int64_t tile_cap;
    int32_t* sorted;      // [ent_cap] partial slots grouped by bucket
    __nv_bfloat16* part_o; // [ent_cap][Hq][d] softmax partials, normalised by their own sum
    float2* part_ml;       // [ent_cap][Hq] (max in log2 units, sum) of each partial
    unsigned char* recs;  // [window tiles + tile_cap] tile descriptions (TILE_REC_BYTES each)
};
constexpr int TILE_REC_BYTES = 448;

// Selection workspace carve-up.  Candidates reach the fill as n_lst lists
// per query row (one per tensor-core split, per decode slice, or one from the
// SIMT nominator): list l of row r holds lst_n[r*n_lst+l] <= lst_cap bucket
// ids, and lst_tau[r*n_lst+l] bounds the approximate score of every eligible
// bucket of the list's range that it does not hold (-inf: it holds them all).
struct SelectWs {
    int32_t* lst_g;      // [B*Nq][n_lst][lst_cap] candidate bucket ids
    int32_t* lst_n;      // [B*Nq][n_lst]
    float* lst_tau;      // [B*Nq][n_lst]
    int n_lst, lst_cap;
    uint16_t* gmax;      // [B*Nq][n_grp] tensor-core path: group maxima (fp16 keys)
    float* theta;        // [B*Nq] tensor-core path: each row's list threshold
    int64_t n_grp;
    // Decode: slice s of sequence b lists its DEC_M best approximate scores,
    // sorted (dl_s, dl_g at [(b * n_slice + s) * DEC_M]), their count dl_n and
    // dl_tau, the slice's next score (-inf when it listed all of them).
    float* dl_s;
    int32_t* dl_g;
    int32_t* dl_n;
    float* dl_tau;
    int n_slice;
    // D-LSA Tree: the rows' chosen branches ([rows][tree_nbr] super-bucket ids)
    // and the tree's CSR ([B][tree_ns + 1] offsets, [B][NBK] members); when
    // set, the exact fallback ranks only the chosen branches' buckets.
    int32_t* tree_br;
    const int32_t* tree_off;
    const int32_t* tree_mem;
    int tree_nbr;
    int64_t tree_ns;
    int32_t* fb_list;    // [B*Nq]      queries that need the exact fallback
    int32_t* fb_count;   // [1]
    double* fb_scores;   // [FB_CTAS][NBK] scratch of the fallback
    BucketPlan plan;     // bucket-major attention lists (all null when unused)
    // Decode append finished by the fill (app_n = 0 when unused): the exact
    // nearest-centroid search of sequence b's completed group ran in app_n
    // slices, each leaving its best (score, bucket); open slot app_slot[b]
    // (-1: no group completed) receives the best of them.
    const double* app_score;   // [B][app_n]
    const int32_t* app_g;      // [B][app_n]
    const int32_t* app_slot;   // [B]
    int app_n;
};
constexpr int FB_CTAS = 148;
constexpr int KCF = 128;          // candidates the fill ranks at most (one per thread)
constexpr int TC_LIST_CAP = KCF;  // candidates per (row, tensor-core split)
constexpr int TC_MAX_SPLITS = 8;
constexpr int TC_TARGET = 48;     // rank of a row's threshold among its group maxima
constexpr int DEC_M = 16;         // best scores a decode slice lists
constexpr int DEC_MAX_SLICES = 128;

// Work split of the tensor-core scorer (k_score_tc.cu).
struct TcSplit {
    int n_split;      // centroid ranges (lists per row)
    int tps;          // centroid tiles of 256 per range
    int gw_log2;      // group width (columns) of the group maxima, 2 .. 6
    int m;            // threshold rank among a row's group maxima
    int64_t n_grp;    // row stride of the group maxima (every width the call may pick)
    int64_t n_qt;     // 128-query tiles per sequence
    int64_t n_items;  // B * n_qt * n_split
};
// n_blk: closed blocks at the time of the call (the group width follows the
// buckets that exist; every other field depends on the index capacity only).
TcSplit tc_split_plan(const IndexView& ix, int64_t Nq, int64_t n_blk);
// The tensor-core scorer serves bf16 indices and at least one 128-query tile.
bool select_uses_tc(const IndexView& ix, int64_t Nq);
size_t select_ws_bytes(const IndexView& ix, int64_t Nq);
SelectWs select_ws_carve(void* ws, const IndexView& ix, int64_t Nq);

cudaError_t launch_select(const IndexView& ix, int64_t n_blk, const void* latent_Q, PosSrc pos,
                          int64_t Nq, lsa_select_params sp, int32_t* indices, int32_t* counts,
                          int s_max, const SelectWs& ws, bool use_tc, cudaStream_t st);

// D-LSA Tree (k_tree.cu): storage bytes, build over the n_blk closed blocks,
// and the arrays the selection reads.
size_t tree_bytes(const IndexView& ix, int64_t NS);
cudaError_t launch_tree_build(const IndexView& ix, int64_t n_blk, void* buf, int64_t NS, int L,
                              cudaStream_t st);
void tree_select_arrays(const IndexView& ix, const void* buf, int64_t NS, const void** sup_rt,
                        const int32_t** off, const int32_t** mem);
cudaError_t tree_export(const IndexView& ix, const void* buf, int64_t NS, float* sup,
                        void* sup_rt, int32_t* off, int32_t* mem, cudaStream_t st);
// Tree selection: workspace bytes and the launch (nominate over the chosen
// branches, exact fill, exact fallback restricted to the branches).
size_t tree_select_ws_bytes(const IndexView& ix, int64_t Nq, int branches);
cudaError_t launch_tree_select(const IndexView& ix, int64_t n_blk, const void* tree_buf,
                               int64_t NS, int branches, const void* latent_Q,
                               const int32_t* positions, int64_t Nq, lsa_select_params sp,
                               int32_t* indices, int32_t* counts, int s_max, void* ws,
                               cudaStream_t st);

// Decode: exact fill + emission from the slices' sorted lists, then the
// exact fallback (one query per sequence).
cudaError_t launch_decode_finish(const IndexView& ix, int64_t n_blk, const void* latent_q,
                                 const int32_t* pos, lsa_select_params sp, int32_t* indices,
                                 int32_t* counts, int s_max, const SelectWs& ws, cudaStream_t st);

// Exact fill + emission + fallback only (candidates already nominated).
cudaError_t launch_select_finish(const IndexView& ix, int64_t n_blk, const void* latent_Q,
                                 PosSrc pos, int64_t Nq, lsa_select_params sp, int32_t* indices,
                                 int32_t* counts, int s_max, const SelectWs& ws, cudaStream_t st);

// Sparse attention (status nullable: receives DEV_BAD_INDEX / DEV_TIMEOUT).
cudaError_t launch_attn_status(const void* Q, const void* K, const void* V, lsa_dtype dt,
                               int64_t B, int64_t Nq, int64_t T_cap, int Hq, int Hkv, int d,
                               const int32_t* indices, const int32_t* counts, int s_max,
                               float scale, void* O, float* lse, uint32_t* status,
                               cudaStream_t st);
// Raises a kernel's dynamic shared-memory limit once per device (so that calls
// made later, for example under stream capture, do not repeat it).
cudaError_t ensure_smem_attr(const void* kernel, int bytes);

// Split-KV bf16 attention: ns splits of keys_per_split keys per (row, head
// group); part [rows][ns][Hq][d+4] and counter [rows * head groups] (zero
// before the launch, left zero after it) are caller scratch.  hg = 1 forces
// one KV head per CTA (smaller partials), 0 picks the default head group.
cudaError_t launch_attn_split(const void* Q, const void* K, const void* V, int64_t B, int64_t Nq,
                              int64_t T_cap, int Hq, int Hkv, int d, const int32_t* indices,
                              const int32_t* counts, int s_max, float scale, void* O, float* lse,
                              uint32_t* status, int ns, int keys_per_split, float* part,
                              uint32_t* counter, int hg, cudaStream_t st);
int attn_stage_keys(int Hkv);
// bf16 attention of the rows row_list[0 .. *row_count) only (grid sized for
// all B * Nq rows; CTAs past the count exit at once).
cudaError_t launch_attn_rows(const void* Q, const void* K, const void* V, int64_t B, int64_t Nq,
                             int64_t T_cap, int Hq, int Hkv, int d, const int32_t* indices,
                             const int32_t* counts, int s_max, float scale, void* O,
                             uint32_t* status, const int32_t* row_list, const int32_t* row_count,
                             cudaStream_t st);
// Merges the ns split partials of every (row, query head) into O (bf16) and lse.
cudaError_t launch_attn_combine(const float* part, int ns, int64_t rows, int Hq, int d, void* O,
                                float* lse, cudaStream_t st);
int attn_head_group(int Hkv);

// Decode: append + approximate scores for one query per sequence, over
// n_slice CTAs per sequence.  ws.dl_* receive every slice's sorted top list
// and bound; app_score / app_g / app_slot the sliced nearest-centroid search.
cudaError_t launch_decode_prep(const IndexView& ix, int64_t n_blk, void* latent_K, void* K,
                               void* V, const void* new_latent_k, const void* new_k,
                               const void* new_v, const void* latent_q, const int32_t* pos,
                               int Hkv, int d, int W, const SelectWs& ws, double* app_score,
                               int32_t* app_g, int32_t* app_slot, int n_slice,
                               uint32_t* attn_counter, int n_counter, cudaStream_t st);

// Selection with scratch in a built-in device array (no caller workspace);
// see k_select_noalloc.cu.
size_t noalloc_scratch_bytes();
cudaError_t noalloc_select(const IndexView& ix, int64_t n_blk, const void* latent_Q,
                           const int32_t* positions, int64_t Nq, lsa_select_params sp,
                           int32_t* indices, int32_t* counts, int s_max, bool use_tc,
                           cudaStream_t st);

// Bucket-major attention of a bf16 prefill chunk (k_attn_bucket.cu): plan,
// scatter, the persistent tile kernel, the per-query kernel for gather rows
// and the merge of every listed row's partials into O.
constexpr int BA_Q = 16;   // queries per bucket or window tile
bool bucket_attn_supported(int Hq, int Hkv, int d);
cudaError_t launch_bucket_attn(const IndexView& ix, int64_t n_blk, const BucketPlan& P,
                               const void* Q, const void* K, const void* V, int64_t Nq, int Hq,
                               int Hkv, int d, PosSrc pos, int W, int S, const int32_t* indices,
                               const int32_t* counts, int s_max, float scale, void* O,
                               cudaStream_t st);

// True when the tensor-core candidate scorer is compiled in.
bool tc_scoring_available();

// Gradients of the sparse attention (k_attn_bwd.cu): dQ written, dK and dV
// (fp32) added to.
bool attn_backward_supported(int Hq, int Hkv, int d);
cudaError_t launch_attn_backward(const void* Q, const void* K, const void* V, const void* O,
                                 const float* lse, const void* dO, lsa_dtype dt, int64_t B,
                                 int64_t Nq, int64_t T_cap, int Hq, int Hkv, int d,
                                 const int32_t* indices, const int32_t* counts, int s_max,
                                 float scale, void* dQ, float* dK, float* dV, uint32_t* status,
                                 cudaStream_t st);

// Context parallel (k_cp.cu): a row's selected positions inside [lo, hi) as
// shard rows; zero output / -inf lse for rows without one; the LSE-weighted
// merge of n_parts partial results [n_parts][rows][Hq][d].
cudaError_t launch_range_filter(const int32_t* indices, const int32_t* counts, int64_t rows,
                                int s_max, int64_t lo, int64_t hi, int32_t* loc_idx,
                                int32_t* loc_cnt, cudaStream_t st);
cudaError_t launch_range_empty(const int32_t* loc_cnt, int64_t rows, int Hq, int d, lsa_dtype dt,
                               void* O, float* lse, cudaStream_t st);
cudaError_t launch_merge_partials(const void* parts, const float* lse_parts, lsa_dtype dt,
                                  int n_parts, int64_t rows, int Hq, int d, void* O, float* lse,
                                  cudaStream_t st);

// Brute-force latent per-key indexer (k_perkey.cu): every long-range key of
// a query scored on the tensor cores, the best R read.
constexpr int PK_CAP = 8192;        // candidate list per query row
constexpr int PK_MAX_R = 4096;      // largest long-range budget
constexpr int PK_NG_MAX = 32768;    // strided key groups per row (at most)
struct PerKeyArgs {
    const void* lat_k;       // bf16 [B][T_cap][64]
    const void* lat_q;       // bf16 [B][Nq][64]
    const int32_t* pos;      // [B][Nq]
    int64_t B, T_cap, n_keys, Nq;
    int R, W, S;
    int32_t* indices;        // [B][Nq][s_max]
    int32_t* counts;         // [B][Nq]
    int s_max;
};
struct PerKeyWs {
    uint32_t* status;        // [8]: code, fallback rows, detail, overflow rows listed
    uint32_t* colmax;        // [B][64] max |latent key| per dimension (fp32 bits)
    float* theta;            // [rows] candidate threshold (-inf: every key, +inf: none)
    int32_t* cnt;            // [rows] keys appended (may pass PK_CAP)
    int32_t* over;           // [rows] rows sent to the exact fallback
    uint16_t* gmax;          // [rows][ng] strided-group maxima (fp16 bits)
    int32_t* cand;           // [rows][PK_CAP] candidate positions
    int64_t ng;              // groups per row (power of two, 256 .. PK_NG_MAX)
};
int64_t per_key_groups(int64_t T_cap);
cudaError_t set_per_key_wait_polls(int64_t polls);
cudaError_t launch_per_key(const PerKeyArgs& a, const PerKeyWs& ws, cudaStream_t st);

// Checks run when LSA_DEBUG=1 (k_debug.cu).  Each synchronises the stream
// (it does nothing while the stream is being captured) and returns in out[4]
// the first violation found: kind (0 = none), sequence or row, place, value.
enum DbgKind : uint32_t {
    DBG_OFFSETS = 1,    // a block's CSR offsets out of its range or decreasing
    DBG_MEMBER = 2,     // a member outside its block
    DBG_ORDER = 3,      // members not ascending inside a bucket
    DBG_ASSIGN = 4,     // a member's assignment names another bucket
    DBG_OPEN = 5,       // an open-block entry that is no closed bucket
    DBG_COUNT = 6,      // a selection count outside [0, s_max]
    DBG_INDEX = 7,      // a selected index outside [0, T_cap)
    DBG_CAUSAL = 8,     // a selected index after the query's position
    DBG_LAYOUT = 9,     // a selection row not laid out as sinks, long-range keys, window
};
// debug_check_gather modes: bounds [0, T_cap) only; a selection row's layout
// (positions from pos, window W, sinks S); layout with ascending long-range keys.
enum DbgGather : int { DBG_BOUNDS = 0, DBG_SELECTION = 1, DBG_SELECTION_SORTED = 2 };
bool debug_enabled();
cudaError_t debug_check_index(const IndexView& ix, int64_t n_blk, cudaStream_t st, uint32_t out[4]);
cudaError_t debug_check_gather(const int32_t* indices, const int32_t* counts, int64_t rows,
                               int s_max, int64_t T_cap, PosSrc pos, int64_t Nq, int W, int S,
                               int mode, cudaStream_t st, uint32_t out[4]);

cudaError_t launch_attn(const void* Q, const void* K, const void* V, lsa_dtype dt, int64_t B,
                        int64_t Nq, int64_t T_cap, int Hq, int Hkv, int d,
                        const int32_t* indices, const int32_t* counts, int s_max, float scale,
                        void* O, float* lse, cudaStream_t st);

}  // namespace lsa

struct lsa_index {
    lsa::IndexView v;
    int64_t n_blk;       // closed blocks (host-side counter)
    void* buf;
    size_t bytes;
    bool status_clean;   // status words cleared on the device
};
