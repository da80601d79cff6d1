/*
 * lsa_oracle.c -- plain, slow CPU restatement of D-LSA Flat (content index,
 * bucket retrieval, exact sparse attention).
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header, table or helper with the CUDA path and includes nothing from it.
 *
 * Sources (web pages about arXiv 2610.42147, "Latent Sparse Attention:
 * Towards Subquadratic Ultra-Long Context Attention"):
 *   [P1]  "Latent Sparse Attention: Towards Subquadratic Ultra-Long Context
 *         Attention" (arXiv abstract mirror), section "Full text".
 *   [P4]  "Prefrontal's Latent Sparse Attention speeds up one attention layer
 *         72x at 10M tokens; end to end, the gain is 9x", section
 *         "What it changes".
 *   [P5]  "Latent Sparse Attention: un indice gerarchico per contesti lunghi",
 *         paragraph on index construction (pooling of consecutive keys,
 *         blocks, buckets with a centroid and original key indices),
 *         paragraph on retrieval (query vs centroids; attention over the
 *         selected keys; the KV cache keeps the original keys), paragraph on
 *         the read budget (64-d index, 4096 long-range keys outside the
 *         recent window, 512 recent keys, 4 sink keys at the start).
 *
 * Where the pages are silent the readings below are the ones listed in the
 * project design notes; each is marked READING.
 *
 * Arithmetic conventions (fixed so that a careful GPU implementation can
 * reproduce every integer decision bit for bit):
 *   - compiled with -ffp-contract=off and without -ffast-math, so every
 *     "a*b + c" below is a rounded product followed by a rounded sum;
 *   - sums run in ascending index order, exactly as written;
 *   - a product of two binary32 values is exact in binary64, so the fp64
 *     dot products of fp32 data below are the exact products summed in order.
 *
 * Parity pins: every function here is pinned by a CPU test against closed
 * forms, hand-built cases or brute force (tests/test_oracle_*.py).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_OK 0
#define ORC_EINVAL 1
#define ORC_ENOMEM 2

/* ------------------------------------------------------------------------ */
/* Small helpers                                                             */
/* ------------------------------------------------------------------------ */

/* binary32 -> bfloat16 -> binary32 with round-to-nearest-even on the upper
 * 16 bits (the definition of bf16 RNE).  Inputs here are finite. */
static float orc_round_bf16(float x)
{
    uint32_t u;
    memcpy(&u, &x, 4);
    if ((u & 0x7f800000u) == 0x7f800000u) return x; /* inf / nan: unchanged */
    uint32_t lsb = (u >> 16) & 1u;
    u = u + 0x7fffu + lsb;
    u &= 0xffff0000u;
    memcpy(&x, &u, 4);
    return x;
}

/* Exact products of binary32 values summed in binary64, ascending i. */
static double orc_dot(const float* a, const float* b, int n)
{
    double s = 0.0;
    for (int i = 0; i < n; ++i) s = s + (double)a[i] * (double)b[i];
    return s;
}

int orc_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void orc_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* ------------------------------------------------------------------------ */
/* Index: pooling [P5 index paragraph]                                        */
/* ------------------------------------------------------------------------ */

/* x_j = mean of the p consecutive latent keys jp .. jp+p-1.
 * READING: the p rows are summed left to right in binary32 and the sum is
 * divided by p in binary32.  lat is [n_groups*p][dl], pooled is [n_groups][dl]. */
void orc_pool(const float* lat, int64_t n_groups, int dl, int p, float* pooled)
{
    for (int64_t j = 0; j < n_groups; ++j) {
        const float* row = lat + (j * p) * (int64_t)dl;
        for (int i = 0; i < dl; ++i) {
            float s = row[i];
            for (int r = 1; r < p; ++r) s = s + row[(int64_t)r * dl + i];
            pooled[j * dl + i] = s / (float)p;
        }
    }
}

/* Unit vector of a pooled key (spherical k-means clusters directions).
 * READING: norm = sqrt(sum x_i^2) with the sum in binary64, ascending i;
 * u_i = binary32(x_i / norm); the zero vector maps to the zero vector. */
void orc_unit(const float* x, int64_t n, int dl, float* u)
{
    for (int64_t j = 0; j < n; ++j) {
        const float* xj = x + j * dl;
        float* uj = u + j * dl;
        double ss = orc_dot(xj, xj, dl);
        double nrm = sqrt(ss);
        for (int i = 0; i < dl; ++i)
            uj[i] = (nrm == 0.0) ? 0.0f : (float)((double)xj[i] / nrm);
    }
}

/* ------------------------------------------------------------------------ */
/* Index: spherical k-means inside one block [P5 index paragraph]            */
/* ------------------------------------------------------------------------ */

/* Clusters the G unit vectors of one block into k buckets.
 *   init   : c_m = u[floor(m*G/k)]  (evenly spaced pooled keys of the block)
 *   repeat L times:
 *     assign : a_j = argmax_m <u_j, c_m>, exact ties to the lowest m
 *     update : v_m = sum over a_j == m of u_j (binary64, ascending j);
 *              c_m = binary32(v_m / ||v_m||); an empty bucket or a zero sum
 *              keeps its previous centroid (READING).
 * The result is the iteration-L assignment together with the iteration-L
 * centroids (READING), so a non-empty centroid is exactly the normalised mean
 * of its members.  margin[j] (nullable) = (s1 - s2) / |s1| of the final
 * assignment, s1 >= s2 the two best scores (infinity when k == 1). */
int orc_kmeans_block(const float* u, int G, int dl, int k, int L,
                     float* cent, int16_t* assign, double* margin)
{
    if (G <= 0 || k <= 0 || k > G || L < 1 || dl <= 0) return ORC_EINVAL;
    double* v = (double*)malloc(sizeof(double) * (size_t)dl);
    if (!v) return ORC_ENOMEM;

    for (int m = 0; m < k; ++m) {
        int64_t src = ((int64_t)m * G) / k;
        memcpy(cent + (int64_t)m * dl, u + src * dl, sizeof(float) * (size_t)dl);
    }

    for (int it = 0; it < L; ++it) {
        for (int j = 0; j < G; ++j) {
            const float* uj = u + (int64_t)j * dl;
            double best = -INFINITY, second = -INFINITY;
            int bm = 0;
            for (int m = 0; m < k; ++m) {
                double s = orc_dot(uj, cent + (int64_t)m * dl, dl);
                if (s > best) {
                    second = best;
                    best = s;
                    bm = m;
                } else if (s > second) {
                    second = s;
                }
            }
            assign[j] = (int16_t)bm;
            if (margin) {
                if (k == 1) margin[j] = INFINITY;
                else if (fabs(best) > 0.0) margin[j] = (best - second) / fabs(best);
                else margin[j] = (best - second > 0.0) ? INFINITY : 0.0;
            }
        }
        for (int m = 0; m < k; ++m) {
            int cnt = 0;
            for (int i = 0; i < dl; ++i) v[i] = 0.0;
            for (int j = 0; j < G; ++j) {
                if (assign[j] != m) continue;
                const float* uj = u + (int64_t)j * dl;
                for (int i = 0; i < dl; ++i) v[i] = v[i] + (double)uj[i];
                ++cnt;
            }
            if (cnt == 0) continue;
            double ss = 0.0;
            for (int i = 0; i < dl; ++i) ss = ss + v[i] * v[i];
            double nrm = sqrt(ss);
            if (nrm == 0.0) continue;
            float* cm = cent + (int64_t)m * dl;
            for (int i = 0; i < dl; ++i) cm[i] = (float)(v[i] / nrm);
        }
    }
    free(v);
    return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* Index: whole blocks of one sequence                                       */
/* ------------------------------------------------------------------------ */

/* Builds blocks [b0, b1) of one sequence.  Block b covers pooled ids
 * [bG, (b+1)G), i.e. keys [bGp, (b+1)Gp).  Arrays are sized for the whole
 * sequence and indexed globally:
 *   lat      [T][dl]                    fp32 latent keys (bf16 data widened)
 *   pooled   [n_pooled][dl]             x_j                 (written for the blocks)
 *   unit     [n_pooled][dl]             u_j
 *   cent     [n_blocks*k][dl]           fp32 centroids c_g, g = b*k + m
 *   cent_rt  [n_blocks*k][dl]           retrieval copy: bf16-rounded c when
 *                                       rt_bf16 != 0, else c (READING)
 *   offsets  [n_blocks*k + 1]           CSR offsets, offsets[b*k] = b*G
 *   members  [n_pooled]                 pooled ids, ascending inside a bucket
 *   assign   [n_pooled]                 bucket m (0..k-1) inside the block
 *   margin   [n_pooled] (nullable)      final-assignment margins
 * Blocks are independent and run in parallel. */
int orc_build_blocks(const float* lat, int dl, int p, int G, int k, int L, int rt_bf16,
                     int64_t b0, int64_t b1,
                     float* pooled, float* unit, float* cent, float* cent_rt,
                     int32_t* offsets, int32_t* members, int16_t* assign, double* margin)
{
    if (p <= 0 || G <= 0 || k <= 0 || k > G || L < 1 || b0 < 0 || b1 < b0) return ORC_EINVAL;
    int err = ORC_OK;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t b = b0; b < b1; ++b) {
        int64_t j0 = b * G;
        orc_pool(lat + j0 * p * dl, G, dl, p, pooled + j0 * dl);
        orc_unit(pooled + j0 * dl, G, dl, unit + j0 * dl);
        int e = orc_kmeans_block(unit + j0 * dl, G, dl, k, L, cent + b * k * dl,
                                 assign + j0, margin ? margin + j0 : NULL);
        if (e != ORC_OK) {
#pragma omp atomic write
            err = e;
            continue;
        }
        for (int64_t x = b * k * dl; x < (b + 1) * k * dl; ++x)
            cent_rt[x] = rt_bf16 ? orc_round_bf16(cent[x]) : cent[x];
        /* CSR: stable counting sort of the block's pooled ids by bucket. */
        int64_t pos = j0;
        for (int m = 0; m < k; ++m) {
            offsets[b * k + m] = (int32_t)pos;
            for (int j = 0; j < G; ++j)
                if (assign[j0 + j] == m) members[pos++] = (int32_t)(j0 + j);
        }
        offsets[(b + 1) * k] = (int32_t)((b + 1) * G);
    }
    return err;
}

/* Nearest closed-block centroid for one unit vector: argmax over the fp32
 * centroids c_g, g < n_buckets, exact ties to the lowest g (READING for the
 * decode-time append of a completed pooled group). */
static int32_t orc_nearest(const float* uj, const float* cent, int64_t n_buckets, int dl)
{
    double best = -INFINITY;
    int32_t bg = 0;
    for (int64_t g = 0; g < n_buckets; ++g) {
        double s = orc_dot(uj, cent + g * dl, dl);
        if (s > best) {
            best = s;
            bg = (int32_t)g;
        }
    }
    return bg;
}

/* Open-block maintenance (decode-time append, READING).  Pooled groups
 * [n_blocks*G, j_end) lie after the last closed block; each one that is not
 * yet assigned (open_bucket == -1) is pooled, normalised and assigned to its
 * nearest closed-block centroid.  open_bucket is [G], indexed by
 * j - n_blocks*G.  pooled / unit rows of those groups are written. */
int orc_open_assign(const float* lat, int dl, int p, int G, int k, int64_t n_blocks,
                    int64_t j_end, const float* cent, float* pooled, float* unit,
                    int32_t* open_bucket)
{
    int64_t j0 = n_blocks * G;
    if (j_end < j0 || j_end > j0 + G || n_blocks < 1) return ORC_EINVAL;
    for (int64_t j = j0; j < j_end; ++j) {
        if (open_bucket[j - j0] >= 0) continue;
        orc_pool(lat + j * p * dl, 1, dl, p, pooled + j * dl);
        orc_unit(pooled + j * dl, 1, dl, unit + j * dl);
        open_bucket[j - j0] = orc_nearest(unit + j * dl, cent, n_blocks * k, dl);
    }
    return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* Retrieval [P5 retrieval and read-budget paragraphs; P4 "What it changes"] */
/* ------------------------------------------------------------------------ */

typedef struct {
    double s;
    int32_t g;
} orc_rank;

static int orc_rank_cmp(const void* a, const void* b)
{
    const orc_rank* x = (const orc_rank*)a;
    const orc_rank* y = (const orc_rank*)b;
    if (x->s > y->s) return -1; /* score descending */
    if (x->s < y->s) return 1;
    return (x->g < y->g) ? -1 : (x->g > y->g); /* ties: lowest bucket id */
}

/* Number of available keys of bucket g for a query at pos, and (when out is
 * non-null) the first `limit` of them in ascending position.
 * Available = keys t of the bucket's pooled members with S <= t <= pos - W
 * (long-range keys lie outside the recent window and the sinks; READING for
 * the key-level causal mask).  Members: the closed CSR list of g, then the
 * open-block groups assigned to g (all of which come after every closed key). */
static int64_t orc_avail(int32_t g, int64_t pos, int p, int W, int S,
                         const int32_t* offsets, const int32_t* members,
                         const int32_t* open_bucket, int64_t open_j0, int n_open,
                         int32_t* out, int64_t limit)
{
    int64_t hi = pos - W; /* last admissible key, may be negative */
    int64_t n = 0;
    for (int32_t x = offsets[g]; x < offsets[g + 1]; ++x) {
        int64_t j = members[x];
        for (int r = 0; r < p; ++r) {
            int64_t t = j * p + r;
            if (t < S || t > hi) continue;
            if (out && n < limit) out[n] = (int32_t)t;
            ++n;
        }
    }
    for (int o = 0; o < n_open; ++o) {
        if (!open_bucket || open_bucket[o] != g) continue;
        int64_t j = open_j0 + o;
        for (int r = 0; r < p; ++r) {
            int64_t t = j * p + r;
            if (t < S || t > hi) continue;
            if (out && n < limit) out[n] = (int32_t)t;
            ++n;
        }
    }
    return n;
}

/* One query.  Scores s_g = <q, c~_g> (exact products, binary64 sum); buckets
 * ranked by (s desc, g asc); greedy fill of the long-range budget R: whole
 * buckets while they fit, the first bucket that does not fit is truncated to
 * its first rem keys in ascending position, then stop.
 * Emitted (READING): sinks [0, min(S, pos+1)) ascending, then the long-range
 * keys in take order, then the window [max(pos-W+1, min(S,pos+1)), pos]
 * ascending; the rest of out[0..s_max) is -1.
 * margin (nullable): how far the ranking is from changing the selected SET.
 * Only buckets with at least one available key matter.  If the fill stopped
 * inside the ranked list at bucket c (the last one it touched), the set
 * changes only if c swaps with its predecessor or with its successor among
 * available buckets, so margin = min((s_{c-1} - s_c) / |s_{c-1}|,
 * (s_c - s_{c+1}) / |s_c|) over the pairs that exist; if every available key
 * was taken (or R == 0) no reordering changes the set and margin = infinity.
 * n_lr (nullable): number of long-range keys taken. */
static double orc_rel_gap(double hi, double lo)
{
    double gap = hi - lo;
    if (fabs(hi) > 0.0) return gap / fabs(hi);
    return (gap > 0.0) ? INFINITY : 0.0;
}

static int orc_select_one(const float* q, int dl, int64_t pos, int64_t n_buckets,
                          const float* cent_rt, const int32_t* offsets, const int32_t* members,
                          const int32_t* open_bucket, int64_t open_j0, int n_open,
                          int p, int R, int W, int S, int s_max,
                          orc_rank* rk, int32_t* out, int32_t* count, double* margin,
                          int32_t* n_lr)
{
    for (int64_t g = 0; g < n_buckets; ++g) {
        rk[g].s = orc_dot(q, cent_rt + g * dl, dl);
        rk[g].g = (int32_t)g;
    }
    qsort(rk, (size_t)n_buckets, sizeof(orc_rank), orc_rank_cmp);

    int64_t n = 0;
    int64_t s_end = (S < pos + 1) ? S : pos + 1;
    for (int64_t t = 0; t < s_end; ++t) out[n++] = (int32_t)t;

    int64_t rem = R;
    double mg = INFINITY;
    double s_before = 0.0, s_cut = 0.0; /* scores of the last two available buckets */
    int n_avail_seen = 0;
    int64_t taken_lr = 0;
    int64_t r = 0;
    if (rem > 0) {
        for (; r < n_buckets; ++r) {
            int32_t g = rk[r].g;
            int64_t a = orc_avail(g, pos, p, W, S, offsets, members, open_bucket, open_j0,
                                  n_open, NULL, 0);
            if (a == 0) continue;
            s_before = s_cut;
            s_cut = rk[r].s;
            ++n_avail_seen;
            int64_t take = (a <= rem) ? a : rem;
            orc_avail(g, pos, p, W, S, offsets, members, open_bucket, open_j0, n_open, out + n,
                      take);
            n += take;
            taken_lr += take;
            rem -= take;
            if (rem == 0) break;
        }
        if (rem == 0) {
            /* The fill stopped at rank r: look at its neighbours. */
            if (n_avail_seen >= 2) {
                double m1 = orc_rel_gap(s_before, s_cut);
                if (m1 < mg) mg = m1;
            }
            for (int64_t r2 = r + 1; r2 < n_buckets; ++r2) {
                int64_t a = orc_avail(rk[r2].g, pos, p, W, S, offsets, members, open_bucket,
                                      open_j0, n_open, NULL, 0);
                if (a == 0) continue;
                double m2 = orc_rel_gap(s_cut, rk[r2].s);
                if (m2 < mg) mg = m2;
                break;
            }
        }
    }
    int64_t w0 = pos - W + 1;
    if (w0 < s_end) w0 = s_end;
    for (int64_t t = w0; t <= pos; ++t) out[n++] = (int32_t)t;
    if (n > s_max) return ORC_EINVAL;
    for (int64_t x = n; x < s_max; ++x) out[x] = -1;
    *count = (int32_t)n;
    if (margin) *margin = mg;
    if (n_lr) *n_lr = (int32_t)taken_lr;
    return ORC_OK;
}

/* Selection for nq queries of one sequence.
 *   q        [nq][dl]   latent queries (fp32; bf16 data widened)
 *   pos      [nq]       absolute positions (the query's own key is at pos)
 *   cent_rt  [n_buckets][dl], offsets [n_buckets+1], members: the index
 *   open_bucket [n_open] (nullable) bucket of each open-block pooled group,
 *            -1 when unassigned; open_j0 = first pooled id of the open block
 *   out      [nq][s_max], count [nq], margin [nq] (nullable), n_lr [nq] (nullable) */
int orc_select(const float* q, int dl, const int64_t* pos, int64_t nq, int64_t n_buckets,
               const float* cent_rt, const int32_t* offsets, const int32_t* members,
               const int32_t* open_bucket, int64_t open_j0, int n_open,
               int p, int R, int W, int S, int s_max,
               int32_t* out, int32_t* count, double* margin, int32_t* n_lr)
{
    if (R < 0 || W < 0 || S < 0 || p <= 0 || s_max < 1 || n_buckets < 0) return ORC_EINVAL;
    int err = ORC_OK;
#pragma omp parallel
    {
        orc_rank* rk = (orc_rank*)malloc(sizeof(orc_rank) * (size_t)(n_buckets > 0 ? n_buckets : 1));
        if (!rk) {
#pragma omp atomic write
            err = ORC_ENOMEM;
        }
#pragma omp for schedule(dynamic, 1)
        for (int64_t i = 0; i < nq; ++i) {
            if (!rk) continue;
            int e = orc_select_one(q + i * dl, dl, pos[i], n_buckets, cent_rt, offsets, members,
                                   open_bucket, open_j0, n_open, p, R, W, S, s_max, rk,
                                   out + i * s_max, count + i, margin ? margin + i : NULL,
                                   n_lr ? n_lr + i : NULL);
            if (e != ORC_OK) {
#pragma omp atomic write
                err = e;
            }
        }
        free(rk);
    }
    return err;
}

/* ------------------------------------------------------------------------ */
/* D-LSA Tree retrieval [P4 "What it changes": clusters are grouped into a   */
/* hierarchy, a query scores a few clusters at each level and walks down;    */
/* P5 paragraph on Flat vs Tree: a tree search computes less, but a wrong    */
/* branch can leave useful keys out]                                          */
/* ------------------------------------------------------------------------ */

/* One query of a two-level tree (READING for the tree's shape: level 2 holds
 * n_super super-buckets, each a CSR list of bucket ids in ascending order).
 * The query scores every super-centroid's retrieval copy (exact products,
 * binary64 sum), walks down the `branches` best (score desc, id asc), and
 * the buckets of those branches are ranked and filled exactly as Flat ranks
 * and fills all buckets (orc_select_one): (s desc, g asc), whole buckets
 * while they fit, the next truncated in ascending position, sinks and window.
 * Buckets outside the chosen branches are never read. */
static int orc_tree_select_one(const float* q, int dl, int64_t pos, int64_t n_buckets,
                               const float* cent_rt, const int32_t* offsets,
                               const int32_t* members, const int32_t* open_bucket,
                               int64_t open_j0, int n_open, int64_t n_super,
                               const float* sup_rt, const int32_t* sup_off,
                               const int32_t* sup_mem, int branches, int p, int R, int W, int S,
                               int s_max, orc_rank* rk, orc_rank* rs, int32_t* out,
                               int32_t* count)
{
    for (int64_t h = 0; h < n_super; ++h) {
        rs[h].s = orc_dot(q, sup_rt + h * dl, dl);
        rs[h].g = (int32_t)h;
    }
    qsort(rs, (size_t)n_super, sizeof(orc_rank), orc_rank_cmp);
    int64_t nu = 0; /* the chosen branches' buckets */
    int64_t nb_take = (branches < n_super) ? branches : n_super;
    for (int64_t r = 0; r < nb_take; ++r) {
        int32_t h = rs[r].g;
        for (int32_t x = sup_off[h]; x < sup_off[h + 1]; ++x) {
            int32_t g = sup_mem[x];
            if (g < 0 || g >= n_buckets) continue;
            rk[nu].s = orc_dot(q, cent_rt + (int64_t)g * dl, dl);
            rk[nu].g = g;
            ++nu;
        }
    }
    qsort(rk, (size_t)nu, sizeof(orc_rank), orc_rank_cmp);

    int64_t n = 0;
    int64_t s_end = (S < pos + 1) ? S : pos + 1;
    for (int64_t t = 0; t < s_end; ++t) out[n++] = (int32_t)t;
    int64_t rem = R;
    for (int64_t r = 0; r < nu && rem > 0; ++r) {
        int32_t g = rk[r].g;
        int64_t a = orc_avail(g, pos, p, W, S, offsets, members, open_bucket, open_j0, n_open,
                              NULL, 0);
        if (a == 0) continue;
        int64_t take = (a <= rem) ? a : rem;
        orc_avail(g, pos, p, W, S, offsets, members, open_bucket, open_j0, n_open, out + n, take);
        n += take;
        rem -= take;
    }
    int64_t w0 = pos - W + 1;
    if (w0 < s_end) w0 = s_end;
    for (int64_t t = w0; t <= pos; ++t) out[n++] = (int32_t)t;
    if (n > s_max) return ORC_EINVAL;
    for (int64_t x = n; x < s_max; ++x) out[x] = -1;
    *count = (int32_t)n;
    return ORC_OK;
}

/* Tree selection for nq queries of one sequence: the arguments of orc_select
 * plus the tree (n_super, sup_rt [n_super][dl], sup_off [n_super+1], sup_mem
 * [sup_off[n_super]]) and the number of branches walked. */
int orc_tree_select(const float* q, int dl, const int64_t* pos, int64_t nq, int64_t n_buckets,
                    const float* cent_rt, const int32_t* offsets, const int32_t* members,
                    const int32_t* open_bucket, int64_t open_j0, int n_open, int64_t n_super,
                    const float* sup_rt, const int32_t* sup_off, const int32_t* sup_mem,
                    int branches, int p, int R, int W, int S, int s_max, int32_t* out,
                    int32_t* count)
{
    if (R < 0 || W < 0 || S < 0 || p <= 0 || s_max < 1 || n_buckets < 0 || n_super < 0 ||
        branches < 0)
        return ORC_EINVAL;
    int err = ORC_OK;
    int64_t n_mem = n_super > 0 ? sup_off[n_super] : 0;
#pragma omp parallel
    {
        orc_rank* rk = (orc_rank*)malloc(sizeof(orc_rank) * (size_t)(n_mem > 0 ? n_mem : 1));
        orc_rank* rs = (orc_rank*)malloc(sizeof(orc_rank) * (size_t)(n_super > 0 ? n_super : 1));
        if (!rk || !rs) {
#pragma omp atomic write
            err = ORC_ENOMEM;
        }
#pragma omp for schedule(dynamic, 1)
        for (int64_t i = 0; i < nq; ++i) {
            if (!rk || !rs) continue;
            int e = orc_tree_select_one(q + i * dl, dl, pos[i], n_buckets, cent_rt, offsets,
                                        members, open_bucket, open_j0, n_open, n_super, sup_rt,
                                        sup_off, sup_mem, branches, p, R, W, S, s_max, rk, rs,
                                        out + i * s_max, count + i);
            if (e != ORC_OK) {
#pragma omp atomic write
                err = e;
            }
        }
        free(rk);
        free(rs);
    }
    return err;
}

/* ------------------------------------------------------------------------ */
/* Exact attention over the selected keys [P4 "What it changes": the        */
/* attention kernel is unchanged; P5 retrieval paragraph]                     */
/* ------------------------------------------------------------------------ */

/* For each query i and head h (KV head kh = h / (Hq/Hkv), READING):
 *   z_t = scale * <Q_h, K_{t,kh}>            (binary64)
 *   o_h = sum_t exp(z_t - max z) V_{t,kh} / sum_t exp(z_t - max z)
 *   lse_h = max z + log(sum_t exp(z_t - max z))
 * over the t = idx[i][0 .. count[i]).  Output rounded to binary32.
 *   Q [nq][Hq][d], K/V [T][Hkv][d], idx [nq][s_max], O [nq][Hq][d],
 *   lse [nq][Hq] (nullable). */
int orc_attend(const float* Q, const float* K, const float* V, int64_t T, int64_t nq,
               int Hq, int Hkv, int d, const int32_t* idx, const int32_t* count, int s_max,
               double scale, float* O, float* lse)
{
    if (Hkv <= 0 || Hq % Hkv != 0 || d <= 0 || s_max < 1) return ORC_EINVAL;
    int err = ORC_OK;
    int grp = Hq / Hkv;
#pragma omp parallel
    {
        double* z = (double*)malloc(sizeof(double) * (size_t)s_max);
        double* acc = (double*)malloc(sizeof(double) * (size_t)d);
        if (!z || !acc) {
#pragma omp atomic write
            err = ORC_ENOMEM;
        }
#pragma omp for schedule(dynamic, 1)
        for (int64_t i = 0; i < nq; ++i) {
            if (!z || !acc) continue;
            const int32_t* ix = idx + i * s_max;
            int n = count[i];
            int bad = (n < 1 || n > s_max);
            for (int x = 0; x < n && !bad; ++x)
                if (ix[x] < 0 || ix[x] >= T) bad = 1;
            if (bad) {
#pragma omp atomic write
                err = ORC_EINVAL;
                continue;
            }
            for (int h = 0; h < Hq; ++h) {
                int kh = h / grp;
                const float* qh = Q + (i * Hq + h) * (int64_t)d;
                double mx = -INFINITY;
                for (int x = 0; x < n; ++x) {
                    const float* kt = K + ((int64_t)ix[x] * Hkv + kh) * d;
                    z[x] = scale * orc_dot(qh, kt, d);
                    if (z[x] > mx) mx = z[x];
                }
                double den = 0.0;
                for (int c = 0; c < d; ++c) acc[c] = 0.0;
                for (int x = 0; x < n; ++x) {
                    double w = exp(z[x] - mx);
                    den = den + w;
                    const float* vt = V + ((int64_t)ix[x] * Hkv + kh) * d;
                    for (int c = 0; c < d; ++c) acc[c] = acc[c] + w * (double)vt[c];
                }
                float* oh = O + (i * Hq + h) * (int64_t)d;
                for (int c = 0; c < d; ++c) oh[c] = (float)(acc[c] / den);
                if (lse) lse[i * Hq + h] = (float)(mx + log(den));
            }
        }
        free(z);
        free(acc);
    }
    return err;
}

/* Gradients of orc_attend's outputs for an upstream gradient dO ("Latent Sparse
 * Attention: un indice gerarchico per contesti lunghi", paragraph on N-LSA's
 * memory: the selected indices are kept for the backward pass; the attention
 * itself is unchanged, so its gradients are those of softmax attention over
 * the selected keys).  Per query i and head h, with z_t = scale <q, k_t> over
 * the selected t, p_t = exp(z_t - max) / sum:
 *   dV_t += p_t dO,   dP_t = <dO, v_t>,   D = sum_t p_t dP_t,
 *   dS_t = p_t (dP_t - D),   dQ = scale sum_t dS_t k_t,   dK_t += scale dS_t q.
 * Binary64 throughout, in the order written (queries, heads, keys ascending);
 * dQ rounded to binary32; dK, dV summed in binary64 over every query and head,
 * then rounded.  Serial. */
int orc_attend_backward(const float* Q, const float* K, const float* V, const float* dO,
                        int64_t T, int64_t nq, int Hq, int Hkv, int d, const int32_t* idx,
                        const int32_t* count, int s_max, double scale, float* dQ, float* dK,
                        float* dV)
{
    if (Hkv <= 0 || Hq % Hkv != 0 || d <= 0 || s_max < 1) return ORC_EINVAL;
    const int grp = Hq / Hkv;
    double* z = (double*)malloc(sizeof(double) * (size_t)s_max);
    double* pp = (double*)malloc(sizeof(double) * (size_t)s_max);
    double* dq = (double*)malloc(sizeof(double) * (size_t)d);
    double* gk = (double*)calloc((size_t)T * Hkv * d, sizeof(double));
    double* gv = (double*)calloc((size_t)T * Hkv * d, sizeof(double));
    int err = (!z || !pp || !dq || !gk || !gv) ? ORC_ENOMEM : ORC_OK;
    for (int64_t i = 0; i < nq && err == ORC_OK; ++i) {
        const int32_t* ix = idx + i * s_max;
        const int n = count[i];
        if (n < 1 || n > s_max) {
            err = ORC_EINVAL;
            break;
        }
        for (int x = 0; x < n; ++x)
            if (ix[x] < 0 || ix[x] >= T) err = ORC_EINVAL;
        if (err != ORC_OK) break;
        for (int h = 0; h < Hq; ++h) {
            const int kh = h / grp;
            const float* qh = Q + (i * Hq + h) * (int64_t)d;
            const float* gh = dO + (i * Hq + h) * (int64_t)d;
            double mx = -INFINITY;
            for (int x = 0; x < n; ++x) {
                z[x] = scale * orc_dot(qh, K + ((int64_t)ix[x] * Hkv + kh) * d, d);
                if (z[x] > mx) mx = z[x];
            }
            double den = 0.0;
            for (int x = 0; x < n; ++x) {
                pp[x] = exp(z[x] - mx);
                den = den + pp[x];
            }
            for (int x = 0; x < n; ++x) pp[x] = pp[x] / den;
            // dP_t, kept in z; D
            double D = 0.0;
            for (int x = 0; x < n; ++x) {
                z[x] = orc_dot(gh, V + ((int64_t)ix[x] * Hkv + kh) * d, d);
                D = D + pp[x] * z[x];
            }
            for (int c = 0; c < d; ++c) dq[c] = 0.0;
            for (int x = 0; x < n; ++x) {
                const double ds = pp[x] * (z[x] - D);
                const int64_t row = ((int64_t)ix[x] * Hkv + kh) * d;
                for (int c = 0; c < d; ++c) {
                    dq[c] = dq[c] + ds * (double)K[row + c];
                    gk[row + c] = gk[row + c] + scale * ds * (double)qh[c];
                    gv[row + c] = gv[row + c] + pp[x] * (double)gh[c];
                }
            }
            float* oq = dQ + (i * Hq + h) * (int64_t)d;
            for (int c = 0; c < d; ++c) oq[c] = (float)(scale * dq[c]);
        }
    }
    if (err == ORC_OK)
        for (int64_t x = 0; x < T * Hkv * d; ++x) {
            dK[x] = (float)gk[x];
            dV[x] = (float)gv[x];
        }
    free(z);
    free(pp);
    free(dq);
    free(gk);
    free(gv);
    return err;
}
