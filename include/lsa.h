/*
 * lsa.h -- C-ABI of liblsa: the D-LSA Flat hot path (content index, bucket
 * retrieval, exact sparse attention) as hand-written CUDA kernels for B200
 * (sm_100a).
 *
 * Method sources (web pages about arXiv 2610.42147):
 *   "Latent Sparse Attention: un indice gerarchico per contesti lunghi",
 *     paragraph on index construction: consecutive keys are pooled in small
 *     groups, the pooled sequence is split into blocks, each block groups
 *     similar representations into buckets that keep a centroid and the
 *     indices of the original keys;
 *     paragraph on retrieval: the query is compared with the centroids to
 *     choose buckets; attention then runs over the selected keys and values;
 *     paragraph on the read budget: a 64-dimensional index; each query reads
 *     4096 long-range keys outside the recent window, the 512 most recent keys
 *     and 4 sink keys (2048 long-range keys for GLM below position 1M).
 *   "Prefrontal's Latent Sparse Attention speeds up one attention layer 72x at
 *     10M tokens; end to end, the gain is 9x", section "What it changes": the
 *     attention kernel itself is unchanged; LSA only decides which keys are
 *     read.  Section "The numbers, and which ones to quote": the timed unit is
 *     the last 32k query chunk of a 10M-token context.
 *
 * Conventions for every call
 *   - Status: every call returns lsa_status; nothing is thrown or aborted
 *     across the ABI.  lsa_last_error() returns a thread-local description of
 *     the last failure on the calling thread.
 *   - Arguments are checked on the host before any launch.  A failed check
 *     launches nothing and returns LSA_ERR_INVALID_ARG (or LSA_ERR_ALIGNMENT /
 *     LSA_ERR_WORKSPACE).
 *   - Memory: every tensor pointer is a DEVICE pointer owned by the caller.
 *     The library never allocates device memory: index storage and scratch
 *     are caller buffers sized by lsa_index_bytes / lsa_*_workspace_bytes.
 *     Device pointers must be 16-byte aligned.
 *   - Streams: `stream` is a cudaStream_t passed as void* (NULL = legacy
 *     default stream).  All work is enqueued asynchronously; outputs are
 *     valid once the stream has been synchronised.  No call synchronises the
 *     stream, so every call can be captured in a CUDA graph (except
 *     lsa_index_check, which reads back a status word).
 *   - Layouts (row-major, innermost last):
 *       latent keys   latent_K [B][T_cap][64]
 *       keys, values  K, V     [B][T_cap][Hkv][d]   (token-major: one key of
 *                                                   all KV heads is contiguous)
 *       latent query  latent_Q [B][Nq][64]
 *       query         Q        [B][Nq][Hq][d]
 *       output        O        [B][Nq][Hq][d]       (same dtype as Q)
 *       selection     indices  [B][Nq][s_max] int32, -1 padded
 *                     counts   [B][Nq] int32
 *     T_cap is the per-sequence capacity given to lsa_index_init; every
 *     per-sequence cache uses it as its sequence stride.
 *   - Dtypes: LSA_F32 or LSA_BF16, uniform for the index and the call.
 *     Positions and indices are int32 (T_cap <= 2^31 - 1); device offsets are
 *     64-bit internally.
 *   - Shapes supported by the kernels: latent dim 64; d in {64, 128};
 *     Hq % Hkv == 0 with Hq / Hkv in {1, 2, 4, 8}.
 */
#ifndef LSA_H
#define LSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    LSA_OK = 0,
    LSA_ERR_INVALID_ARG = 1, /* a size, shape, pointer or parameter is invalid */
    LSA_ERR_ALIGNMENT = 2,   /* a pointer is not 16-byte aligned */
    LSA_ERR_WORKSPACE = 3,   /* a caller buffer is smaller than required */
    LSA_ERR_CUDA = 4,        /* a CUDA runtime call failed (message in lsa_last_error) */
    LSA_ERR_TIMEOUT = 5,     /* a bounded device wait gave up (status word) */
    LSA_ERR_INTERNAL = 6,    /* a device-side consistency check failed (status word) */
    LSA_ERR_UNSUPPORTED = 7  /* valid request outside what the kernels implement */
} lsa_status;

typedef enum { LSA_F32 = 0, LSA_BF16 = 1 } lsa_dtype;

/* Index parameters.  p: keys per pooled group; block: pooled groups per block
 * (G); n_buckets: buckets per block (k); lloyd_iters: Lloyd iterations (L). */
typedef struct {
    int p;
    int block;
    int n_buckets;
    int lloyd_iters;
} lsa_index_params;

/* Read budget.  budget: long-range keys R; window: recent keys W; sinks: S. */
typedef struct {
    int budget;
    int window;
    int sinks;
} lsa_select_params;

/* Opaque host handle over caller-owned index storage. */
typedef struct lsa_index lsa_index;

/* Thread-local text of the last failure on this thread ("" if none). */
const char* lsa_last_error(void);

/* Library version string. */
const char* lsa_version(void);

/* Number of CUDA kernel launches this library has enqueued in the process so
 * far (all threads, all devices).  Host-side counter, never synchronises. */
uint64_t lsa_kernel_launches(void);

/* ---------------------------------------------------------------------------
 * Content index  ("un indice gerarchico", paragraph on index construction)
 *
 * Per sequence: pooled groups j = 0 .. T/p - 1 (keys jp .. jp+p-1, mean of
 * their latent keys, summed left to right in binary32 then divided by p);
 * unit vectors u_j = x_j / ||x_j|| (norm from a binary64 sum of squares);
 * block b = pooled groups [bG, (b+1)G); inside each block spherical k-means
 * into k buckets: c_m initialised to u[bG + floor(m*G/k)], then L times
 * {assign each u to the bucket of largest <u, c_m> (exact products summed in
 * binary64 in ascending dimension; ties to the lowest m); c_m = normalised
 * binary64 sum of its members in ascending order, an empty bucket keeps its
 * centroid}.  Bucket records: global bucket g = b*k + m, CSR offsets and
 * members (pooled ids, ascending).  Retrieval copy of the centroids: bf16
 * (round to nearest even) for LSA_BF16 indices, fp32 otherwise.
 * Completed pooled groups after the last whole block ("open block") are
 * assigned to the bucket of their nearest closed centroid (decode append).
 * ------------------------------------------------------------------------- */

/* Bytes of device storage for an index of B sequences with capacity T_cap
 * keys each.  Returns 0 on invalid arguments (see lsa_last_error). */
size_t lsa_index_bytes(int64_t B, int64_t T_cap, lsa_index_params ip, lsa_dtype dtype);

/* Creates a host handle over `buf` (device, >= lsa_index_bytes, 256-byte
 * aligned) and records the parameters.  The index starts empty (0 blocks);
 * storage is not touched until the first build/extend.  *out must be released
 * with lsa_index_release; the device buffer stays owned by the caller. */
lsa_status lsa_index_init(void* buf, size_t bytes, int64_t B, int64_t T_cap, lsa_index_params ip,
                          lsa_dtype dtype, lsa_index** out);

/* Frees the host handle only. */
void lsa_index_release(lsa_index* idx);

/* Builds the index over keys [0, T) of every sequence: same as
 * lsa_index_extend(idx, latent_K, 0, T, stream). */
lsa_status lsa_build_index(lsa_index* idx, const void* latent_K, int64_t T, void* stream);

/* (Re)clusters every whole block overlapping [T_old, T_new) (blocks
 * floor(T_old/(pG)) .. floor(T_new/(pG)) - 1), then resets the open block and
 * assigns its completed pooled groups below T_new.  Requires
 * floor(T_old/(pG)) <= current block count (no gap) and T_new <= T_cap.
 * Rebuilding a block from the same keys reproduces it bit for bit. */
lsa_status lsa_index_extend(lsa_index* idx, const void* latent_K, int64_t T_old, int64_t T_new,
                            void* stream);

/* Number of closed blocks currently indexed (host-side counter). */
int64_t lsa_index_num_blocks(const lsa_index* idx);

/* Copies the index state to caller DEVICE buffers (any may be NULL):
 * pooled/unit [B][T_cap/p][64] f32, cent [B][nblk_max*k][64] f32,
 * cent_rt [B][nblk_max*k][64] (dtype of the index), offsets
 * [B][nblk_max*k + 1] i32, members [B][T_cap/p] i32, assign [B][T_cap/p] i16,
 * open_bucket [B][G] i32 (-1 = not assigned). */
lsa_status lsa_index_export(const lsa_index* idx, float* pooled, float* unit, float* cent,
                            void* cent_rt, int32_t* offsets, int32_t* members, int16_t* assign,
                            int32_t* open_bucket, void* stream);

/* Reads and clears the index's device status word (synchronises `stream`).
 * Returns LSA_OK, or the error recorded by a kernel since the last check
 * (for example LSA_ERR_INTERNAL when a decode step found its open block full);
 * *fallbacks (nullable) receives the number of queries that took the exact
 * selection fallback since the last check. */
lsa_status lsa_index_check(lsa_index* idx, int64_t* fallbacks, void* stream);

/* ---------------------------------------------------------------------------
 * Retrieval  ("un indice gerarchico", paragraphs on retrieval and on the
 * read budget)
 *
 * Query at position pos with latent q: s_g = <q, c~_g> over every closed
 * bucket; buckets ranked by (s desc, g asc); key t of bucket g is available
 * iff S <= t <= pos - W; long-range keys are filled greedily up to R: whole
 * buckets' available keys while they fit, then the first `rem` available keys
 * of the next bucket in ascending position.  Emitted row: sinks
 * [0, min(S, pos+1)), long-range keys in take order, window
 * [max(pos-W+1, min(S,pos+1)), pos]; the rest -1.  The scores are those of
 * exact products summed in binary64, so the selection is reproducible bit
 * for bit (approximate tensor-core scores only nominate candidates; a query
 * whose candidates cannot prove the exact ranking takes an exact fallback).
 * ------------------------------------------------------------------------- */

/* Workspace bytes for lsa_select on Nq queries per sequence. */
size_t lsa_select_workspace_bytes(const lsa_index* idx, int64_t Nq);

/* latent_Q [B][Nq][64] (index dtype), positions [B][Nq] int32 device (each
 * 0 <= pos < T_cap; keys below pos-W+1 must be indexed or in the open lists),
 * indices [B][Nq][s_max] with s_max >= budget+window+sinks, counts [B][Nq]. */
lsa_status lsa_select(const lsa_index* idx, const void* latent_Q, const int32_t* positions,
                      int64_t Nq, lsa_select_params sp, int32_t* indices, int32_t* counts,
                      int s_max, void* workspace, size_t ws_bytes, void* stream);

/* Same as lsa_select, for callers that cannot allocate device memory (a
 * plug-in whose host hands it only input and output buffers, a serving loop
 * whose device memory was divided up at start-up, a program with no device
 * allocator): no workspace argument and no allocation.  The pages describe no
 * such call; it exists for those callers.  Its scratch is one built-in 8 MiB
 * device array that every GPU loading the library keeps until the process
 * exits.  A call is refused (LSA_ERR_WORKSPACE, nothing launched) exactly
 * when lsa_select_workspace_bytes(idx, Nq) exceeds 8 MiB; that size counts
 * every query row of every sequence (B * Nq rows) and grows with the number
 * of buckets per sequence, so ask lsa_select_workspace_bytes rather than
 * estimate it.  The first call on each device looks up the array's device
 * address (cudaGetSymbolAddress) and keeps it for the process; make that
 * first call before any stream capture, and do not call this entry again on
 * a device after cudaDeviceReset (the kept address would be stale).  All
 * calls share the array: calls that overlap on the GPU (other streams, other
 * threads) race and must be serialised by the caller.  Results are identical
 * to lsa_select's. */
lsa_status lsa_select_noalloc(const lsa_index* idx, const void* latent_Q,
                              const int32_t* positions, int64_t Nq, lsa_select_params sp,
                              int32_t* indices, int32_t* counts, int s_max, void* stream);

/* ---------------------------------------------------------------------------
 * D-LSA Tree ("Prefrontal's ...", section "What it changes": clusters are
 * grouped into a hierarchy; a query scores a few clusters at each level, walks
 * down the tree and only then fetches keys.  "Latent Sparse Attention: un
 * indice gerarchico per contesti lunghi", paragraph on Flat vs Tree: the tree
 * computes less, a wrong branch can leave useful keys out.)
 *
 * This library's two-level reading: level 2 clusters every sequence's closed
 * buckets' fp32 centroids into n_super super-buckets exactly as a block's unit
 * vectors are clustered (init c2_h = c[floor(h * NB / n_super)], lloyd_iters
 * Lloyd iterations, exact binary64 scores, ties to the lowest id, an empty
 * super-bucket keeps its centroid); each super-bucket lists its bucket ids in
 * ascending order, and its retrieval copy is bf16 for bf16 indices.  A query
 * scores every super-centroid exactly, walks the `branches` best (score desc,
 * lowest id on ties) and ranks and fills only their buckets, as lsa_select
 * ranks and fills all of them (same budget, sinks, window, emitted order).
 * With branches = n_super the selection is lsa_select's.
 * ------------------------------------------------------------------------- */

/* Bytes of device storage for a tree of n_super super-buckets over idx (0 on
 * bad arguments). */
size_t lsa_tree_bytes(const lsa_index* idx, int n_super);

/* Builds the tree over the index's current closed blocks into `tree`
 * (device, 256-byte aligned, >= lsa_tree_bytes).  Requires at least one
 * closed block and 1 <= n_super <= closed buckets (and <= 12800).  Rebuild it
 * after lsa_index_extend: buckets added later belong to no branch. */
lsa_status lsa_tree_build(const lsa_index* idx, void* tree, size_t bytes, int n_super,
                          int lloyd_iters, void* stream);

/* Copies the tree to caller DEVICE buffers (any may be NULL): sup
 * [B][n_super][64] f32 super-centroids, sup_rt [B][n_super][64] retrieval
 * copy (index dtype), offsets [B][n_super + 1] i32 and members [B][NBK] i32
 * (bucket ids of super-bucket h at offsets[h] .. offsets[h+1]), NBK being the
 * index's bucket capacity per sequence. */
lsa_status lsa_tree_export(const lsa_index* idx, const void* tree, int n_super, float* sup,
                           void* sup_rt, int32_t* offsets, int32_t* members, void* stream);

/* Workspace bytes for lsa_tree_select on Nq queries per sequence. */
size_t lsa_tree_select_workspace_bytes(const lsa_index* idx, int64_t Nq, int branches);

/* Tree selection: the arguments of lsa_select plus the tree (built with the
 * same n_super) and 1 <= branches <= min(n_super, 256).  The candidates of a
 * query are the chosen branches' buckets; the exact ranking is proved as in
 * lsa_select, and a query whose proof fails (or whose branches hold more
 * buckets than the nominator's shared memory) takes an exact fallback over
 * its chosen branches, counted by lsa_index_check. */
lsa_status lsa_tree_select(const lsa_index* idx, const void* tree, int n_super, int branches,
                           const void* latent_Q, const int32_t* positions, int64_t Nq,
                           lsa_select_params sp, int32_t* indices, int32_t* counts, int s_max,
                           void* workspace, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Brute-force latent per-key indexer: the baseline that LSA's bucket
 * retrieval replaces ("Prefrontal's ...", section "What it changes": the
 * indexer that scores every earlier key for every query, quadratic in the
 * context and most of a layer's prefill time at 10M tokens; "Latent Sparse
 * Attention: un indice gerarchico per contesti lunghi", paragraph on the read
 * budget).  No index is involved: every long-range key of a query is scored.
 *
 * For query i of sequence b at p = positions[b][i] (0 <= p < n_keys): the
 * keys t in [sinks, p - window] are ranked by <latent_Q[b][i], latent_K[b][t]>
 * (the exact products summed in binary64 in ascending dimension), highest
 * first, ties to the lower position, and the `budget` first are taken.  The
 * row is emitted as lsa_select emits it: sinks 0 .. min(sinks, p+1)-1, the
 * taken keys in ascending position, the window max(p-window+1, n_sinks) .. p,
 * -1 padded to s_max; counts[b][i] is its length.  A position outside
 * [0, n_keys) gives an empty row (count 0) and LSA_ERR_INVALID_ARG from
 * lsa_select_per_key_check.
 *
 * Scores come from the tensor cores (bf16 in, fp32 accumulated); the exact
 * ranking is then proved: a threshold that at least `budget` keys reach,
 * lowered by twice a bound on the fp32 error, keeps every key of the exact
 * top set among the candidates, which are ranked by exact binary64 scores.
 * A query with more than 8192 candidates (scores tied over that many keys)
 * ranks every eligible key exactly instead (counted by the check).
 * ------------------------------------------------------------------------- */

/* Workspace bytes for lsa_select_per_key (0 on bad sizes).  About
 * B*Nq*(2*min(32768, max(256, T_cap rounded up to a power of two)) + 32 KiB + 12) bytes:
 * 3.1 GB for 32,768 queries of one 10M-key sequence. */
size_t lsa_select_per_key_workspace_bytes(int64_t B, int64_t Nq, int64_t T_cap);

/* latent_K [B][T_cap][64] and latent_Q [B][Nq][64] of dtype LSA_BF16 (LSA_F32
 * returns LSA_ERR_UNSUPPORTED); keys 0 .. n_keys-1 of each sequence are read
 * (n_keys <= T_cap); positions [B][Nq] int32; sp.budget <= 4096; indices
 * [B][Nq][s_max] with s_max >= budget + window + sinks; counts [B][Nq].
 * B*T_cap and B*Nq must stay below 2^31.  The workspace holds the call's
 * status until the next call on it. */
lsa_status lsa_select_per_key(const void* latent_K, lsa_dtype dtype, int64_t B, int64_t T_cap,
                              int64_t n_keys, const void* latent_Q, const int32_t* positions,
                              int64_t Nq, lsa_select_params sp, int32_t* indices, int32_t* counts,
                              int s_max, void* workspace, size_t ws_bytes, void* stream);

/* Synchronises `stream` and reads the status the last lsa_select_per_key on
 * this workspace left: LSA_ERR_TIMEOUT (a bounded wait gave up; the outputs
 * are undefined), LSA_ERR_INVALID_ARG (a position outside [0, n_keys)), else
 * LSA_OK.  fallbacks (nullable) receives the queries ranked over every
 * eligible key. */
lsa_status lsa_select_per_key_check(const void* workspace, int64_t* fallbacks, void* stream);

/* ---------------------------------------------------------------------------
 * Exact sparse attention ("Prefrontal's ...", section "What it changes")
 *
 * For query (b, i) and head h with KV head kh = h / (Hq/Hkv):
 *   o = softmax_t(scale * <Q_h, K_{t,kh}>) V_{t,kh}
 * over t = indices[b][i][0 .. counts[b][i]).  fp32 softmax and accumulation;
 * bf16 inputs use tensor-core MMA.  lse (nullable) [B][Nq][Hq] f32 receives
 * max + ln(sum) of the scaled logits.  counts must be >= 1 and every listed
 * index in [0, T_cap).
 * ------------------------------------------------------------------------- */
lsa_status lsa_sparse_attn(const void* Q, const void* K, const void* V, lsa_dtype dtype,
                           int64_t B, int64_t Nq, int64_t T_cap, int Hq, int Hkv, int d,
                           const int32_t* indices, const int32_t* counts, int s_max, float scale,
                           void* O, float* lse, void* stream);

/* Gradients of lsa_sparse_attn over the same stored selection ("Latent Sparse
 * Attention: un indice gerarchico per contesti lunghi", paragraph on N-LSA's
 * memory: the selected indices are kept for the backward pass).  Inputs: the
 * forward's Q, K, V, indices, counts, scale, its output O and lse (as
 * lsa_sparse_attn returns them), and the upstream gradient dO [B][Nq][Hq][d]
 * (dtype).  With p_t = exp(scale <q, k_t> - lse):
 *   D = <dO, O>, dS_t = p_t (<dO, v_t> - D),
 *   dQ = scale sum_t dS_t k_t          -> dQ [B][Nq][Hq][d] (dtype), written;
 *   dK_t += scale dS_t q, dV_t += p_t dO -> dK, dV [B][T_cap][Hkv][d] f32,
 *   ADDED to (zero them first; keys read by several queries receive several
 *   additions in no fixed order).
 * Hq/Hkv <= 8, d <= 128; listed indices outside [0, T_cap) are skipped.
 * Caller-owned device memory, 16-byte aligned; asynchronous on `stream`. */
lsa_status lsa_sparse_attn_backward(const void* Q, const void* K, const void* V, const void* O,
                                    const float* lse, const void* dO, lsa_dtype dtype, int64_t B,
                                    int64_t Nq, int64_t T_cap, int Hq, int Hkv, int d,
                                    const int32_t* indices, const int32_t* counts, int s_max,
                                    float scale, void* dQ, float* dK, float* dV, void* stream);

/* ---------------------------------------------------------------------------
 * KV cache in shards of whole blocks ("Latent Sparse Attention: un indice
 * gerarchico per contesti lunghi", paragraph on memory: with context
 * parallelism every rank keeps its share of the KV cache and a full copy of
 * the bucket index, so every rank makes the same selection)
 * ------------------------------------------------------------------------- */

/* Workspace bytes for lsa_attend_key_range (0 on bad sizes). */
size_t lsa_attend_key_range_workspace_bytes(int64_t B, int64_t Nq, int s_max);

/* Attention of every query over the keys of its selection that lie in
 * [key_lo, key_hi), read from a shard of the caches:
 *   K_shard, V_shard [B][key_hi - key_lo][Hkv][d] hold rows key_lo .. key_hi-1
 *   of the full caches; indices / counts / s_max are the selection in global
 *   positions (as lsa_select writes it);
 *   O_part [B][Nq][Hq][d] (dtype) receives the softmax over those keys alone,
 *   lse_part [B][Nq][Hq] f32 their max + ln(sum) of the scaled logits; a
 *   (query, head) without a key in the range gets O = 0 and lse = -inf.
 * The partial results of shards that cover every selected key merge into
 * lsa_sparse_attn's result with lsa_merge_partials.  Caller-owned device
 * memory; workspace of lsa_attend_key_range_workspace_bytes(B, Nq, s_max);
 * all pointers 16-byte aligned; asynchronous on `stream`. */
lsa_status lsa_attend_key_range(const void* Q, const void* K_shard, const void* V_shard,
                                lsa_dtype dtype, int64_t B, int64_t Nq, int Hq, int Hkv, int d,
                                const int32_t* indices, const int32_t* counts, int s_max,
                                int64_t key_lo, int64_t key_hi, float scale, void* workspace,
                                size_t ws_bytes, void* O_part, float* lse_part, void* stream);

/* LSE-weighted merge of n_parts (1 .. 32) partial attention results:
 *   O_parts [n_parts][rows][Hq][d] (dtype), lse_parts [n_parts][rows][Hq] f32;
 *   O[r][h] = sum_p exp(lse_p - L) O_p[r][h] with L = ln sum_p exp(lse_p)
 *   (parts with lse = -inf weigh 0; a row no part covers gets 0), lse
 *   (nullable) [rows][Hq] receives L.  Asynchronous on `stream`. */
lsa_status lsa_merge_partials(const void* O_parts, const float* lse_parts, lsa_dtype dtype,
                              int n_parts, int64_t rows, int Hq, int d, void* O, float* lse,
                              void* stream);

/* ---------------------------------------------------------------------------
 * Fused entries
 * ------------------------------------------------------------------------- */

/* Recommended workspace bytes for lsa_prefill_chunk with Nq = T_new - T_old
 * queries of Hq query heads, Hkv KV heads and head size d (0 on bad
 * arguments).  For a bf16 index it includes the bucket-major attention lists
 * with room for the chunk's expected softmax partials: about
 * 1.5 * budget / (p * block / n_buckets) + 2 slots of Hq * (d + 4) floats per
 * query (14.4 GB for 32768 queries, Hq = 32, d = 128, budget 4096, 256-key
 * buckets).  A smaller workspace also works; see lsa_prefill_partial_slots. */
size_t lsa_prefill_workspace_bytes(const lsa_index* idx, int64_t Nq, int Hq, int Hkv, int d,
                                   lsa_select_params sp);

/* Softmax partial slots that a workspace of ws_bytes gives lsa_prefill_chunk
 * (this library's own quantity; the pages have no counterpart): -1 when
 * ws_bytes is below the minimum, 0 for the fp32 path or a minimal bf16
 * workspace.  Each query row of a bf16 chunk needs (buckets it took + 1) slots;
 * rows that find no free slot are attended key by key instead, which gives
 * the same result up to fp32 summation order, only slower. */
int64_t lsa_prefill_partial_slots(const lsa_index* idx, int64_t Nq, int Hq, int Hkv, int d,
                                  lsa_select_params sp, size_t ws_bytes);

/* One prefill chunk ("Prefrontal's ...", section "The numbers, and which ones
 * to quote": prefilling the last query chunk of a long context).  Queries are
 * the positions [T_old, T_new) of every sequence.  Steps: lsa_index_extend
 * over [T_old, T_new), selection for every chunk query, sparse attention with
 * scale 1/sqrt(d).  latent_Q [B][Nq][64], Q and O [B][Nq][Hq][d]; the caches
 * already hold keys [0, T_new).  The selection is written to the workspace
 * (read it back as indices [B][Nq][s_max] int32 at offset 0 and counts
 * [B][Nq] int32 at the next 256-byte boundary).
 * bf16 attention runs bucket-major ("Latent Sparse Attention: un indice
 * gerarchico per contesti lunghi", paragraph on retrieval: the selected keys
 * are whole buckets plus sinks and window): the key rows of every bucket that
 * chunk queries took are read once per KV head for up to 16 of those queries,
 * each query's softmax partials (one per bucket, one for sinks and window)
 * are merged in fp32.  Rows listed as exact-selection fallbacks, or that find
 * no partial slot, are attended key by key from their index list.
 * ws_bytes may be anything from the minimum (lsa_prefill_partial_slots >= 0)
 * up; less than that returns LSA_ERR_WORKSPACE. */
lsa_status lsa_prefill_chunk(lsa_index* idx, const void* latent_K, const void* latent_Q,
                             const void* Q, const void* K, const void* V, int64_t T_old,
                             int64_t T_new, int Hq, int Hkv, int d, lsa_select_params sp,
                             void* workspace, size_t ws_bytes, void* O, void* stream);

/* lsa_prefill_chunk for a contiguous range of the chunk's queries: rows
 * q_begin .. q_end - 1 of the chunk, at positions T_old + q_begin ..
 * T_old + q_end - 1 (this library's own entry, for splitting one chunk's
 * queries over GPUs; the pages' serving layout splits the KV cache instead,
 * "Latent Sparse Attention: un indice gerarchico per contesti lunghi",
 * paragraph on memory).  The index is extended over the whole [T_old, T_new)
 * exactly as lsa_prefill_chunk does -- the extension is deterministic, so
 * every caller that runs it on the same keys holds the same index -- and only
 * the range's queries are selected and attended.  latent_Q [B][n][64], Q and
 * O [B][n][Hq][d] with n = q_end - q_begin; the workspace is sized by
 * lsa_prefill_workspace_bytes(idx, n, ...).  Each query's selection is the
 * one lsa_prefill_chunk gives it over the whole chunk, bit for bit; its output
 * equals that one up to the order of the softmax sums (a tile of sinks and
 * windows spans a run of consecutive queries, and a range boundary can cut a
 * run).
 * Requires 0 <= q_begin < q_end <= T_new - T_old; fails like
 * lsa_prefill_chunk otherwise. */
lsa_status lsa_prefill_chunk_queries(lsa_index* idx, const void* latent_K, const void* latent_Q,
                                     const void* Q, const void* K, const void* V, int64_t T_old,
                                     int64_t T_new, int64_t q_begin, int64_t q_end, int Hq,
                                     int Hkv, int d, lsa_select_params sp, void* workspace,
                                     size_t ws_bytes, void* O, void* stream);

/* The two halves of lsa_prefill_chunk, for callers that overlap or time them
 * separately (this library's split; the pages describe the chunk as one
 * step).  lsa_prefill_select extends the index over [T_old, T_new) and
 * selects for every chunk query, leaving the selection and (bf16) the bucket
 * lists in the workspace.  lsa_prefill_attend then attends from that
 * workspace into O; it must get the same T_old, T_new, Hq, Hkv, d, sp,
 * workspace and ws_bytes, and the caches must hold keys [0, T_new).  It
 * changes only the attention part of the workspace, so it may be repeated.
 * Both check every argument before any launch and fail like
 * lsa_prefill_chunk. */
lsa_status lsa_prefill_select(lsa_index* idx, const void* latent_K, const void* latent_Q,
                              int64_t T_old, int64_t T_new, int Hq, int Hkv, int d,
                              lsa_select_params sp, void* workspace, size_t ws_bytes,
                              void* stream);
lsa_status lsa_prefill_attend(const lsa_index* idx, const void* Q, const void* K, const void* V,
                              int64_t T_old, int64_t T_new, int Hq, int Hkv, int d,
                              lsa_select_params sp, void* workspace, size_t ws_bytes, void* O,
                              void* stream);

/* lsa_prefill_chunk with the chunk's inputs and its output in host memory
 * (this library's own entry; the pages serve from device caches).  The
 * chunk's new rows h_latent_K [B][Nq][64] and h_K, h_V [B][Nq][Hkv][d] are
 * copied into the device caches latent_K, K, V at rows [T_old, T_new) of every
 * sequence, h_latent_Q [B][Nq][64] into latent_Q and h_Q [B][Nq][Hq][d] into Q
 * (all in the index's dtype); after the chunk, O [B][Nq][Hq][d] is copied to
 * h_O.  The latent rows travel first on `stream`; K, V and Q travel on
 * `copy_stream` while the index extension and the selection run on `stream`,
 * and the attention waits for them, so those copies overlap the selection.
 * Host buffers should be page-locked (pageable memory works but does not
 * overlap).  copy_stream must differ from stream; an event orders it after the
 * work queued on stream before the call.  Every check of lsa_prefill_chunk is
 * made before the first copy; a failure after that is LSA_ERR_CUDA.  On return
 * the work is queued: h_O is valid once `stream` has synchronised. */
lsa_status lsa_prefill_chunk_host(lsa_index* idx, const void* h_latent_K, const void* h_K,
                                  const void* h_V, const void* h_latent_Q, const void* h_Q,
                                  void* latent_K, void* K, void* V, void* latent_Q, void* Q,
                                  int64_t T_old, int64_t T_new, int Hq, int Hkv, int d,
                                  lsa_select_params sp, void* workspace, size_t ws_bytes,
                                  void* O, void* h_O, void* stream, void* copy_stream);

/* Test hook (this library's own; not part of the method): the number of
 * polls each bounded wait makes before it gives up, in every kernel that waits
 * on a copy or on another warp: the tensor-core centroid scorer (bf16
 * selection with Nq >= 128), the tensor-core attention tiles of bf16 prefill
 * chunks, the per-query bf16 attention kernel (decode steps, prefill rows
 * attended key by key, lsa_sparse_attn) and the per-key indexer's scoring
 * passes.  A wait that gives up records LSA_ERR_TIMEOUT in the index status
 * word for lsa_index_check (in the workspace for lsa_select_per_key_check;
 * lsa_sparse_attn has no status word), and the kernel still leaves cleanly: its
 * copies and MMAs in flight are waited for with the default limit, so the
 * context stays usable; the outputs of such a launch are undefined.  polls < 0
 * restores the defaults (about 4 million polls for the tensor-core kernels, 16
 * million for the per-query kernel); 0 makes every such wait give up at once.
 * Synchronous; applies to later launches on the current device. */
lsa_status lsa_set_wait_limit(int64_t polls);

/* Workspace bytes for lsa_decode_step (depends on the device's SM count). */
size_t lsa_decode_workspace_bytes(const lsa_index* idx, int Hq, int Hkv, int d,
                                  lsa_select_params sp);

/* One decode step for every sequence ("Latent Sparse Attention: Towards
 * Subquadratic Ultra-Long Context Attention", section "Full text": LSA also
 * speeds up decode; the index maintenance below is this library's reading).
 * Sequence b's new token sits at position pos[b] (device int32 [B]; keys
 * [0, pos[b]) already in the caches, pos[b] in the open block that follows
 * the index's closed blocks).  Steps, all on `stream`:
 *   1. write new_latent_k [B][64], new_k / new_v [B][Hkv][d] to position
 *      pos[b] of latent_K, K, V ([B][T_cap][...]);
 *   2. if (pos[b]+1) % p == 0, pool and normalise the completed group and
 *      append it to the bucket of its nearest closed centroid (exact binary64
 *      score, lowest bucket id on ties); an open block that is already full
 *      records LSA_ERR_INTERNAL in the status word (lsa_index_check) and the
 *      group is not appended;
 *   3. select for latent_q [B][64] at pos[b] exactly as lsa_select does;
 *   4. exact attention of q [B][Hq][d] over the selection into O [B][Hq][d]
 *      (split over keys, partials combined in fp32), scale 1/sqrt(d).
 * The selection of step 3 never depends on the append of step 2 (a group
 * that completes at pos lies inside the recent window), so the two run
 * concurrently.  Graph-capturable: no synchronisation, no allocation.
 * When the sequences' open block is full (the step that wrote its last key,
 * pos[b] + 1 a multiple of p * block for every b), the caller closes it with
 * lsa_index_extend(idx, latent_K, pos + 1 - p * block, pos + 1): the block is
 * clustered into buckets like any other and decoding continues into an empty
 * open block after it. */
lsa_status lsa_decode_step(lsa_index* idx, void* latent_K, void* K, void* V,
                           const void* new_latent_k, const void* new_k, const void* new_v,
                           const void* latent_q, const void* q, const int32_t* pos, int Hq,
                           int Hkv, int d, lsa_select_params sp, void* workspace, size_t ws_bytes,
                           void* O, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* LSA_H */
