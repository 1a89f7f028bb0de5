/*
 * CPU oracle for the Latent Sparse Attention (LSA) indexer and the sparse
 * attention it feeds.  TEST INFRASTRUCTURE ONLY: the tests, the smoke check
 * and the benchmark's CPU-baseline leg call it; the library never does.
 * It shares no code, header or table with the CUDA path.
 *
 * Plain, slow and literal on purpose: each function follows one passage of
 * the LSA pages (cited as page title + section) in their order, with no
 * blocking or fusion.  Build: gcc -O2 -fopenmp -ffp-contract=off.
 *
 * Sources (web pages about "Latent Sparse Attention: Towards Subquadratic
 * Ultra-Long Context Attention", arXiv 2610.42147):
 *   [EXPL]  learnaivisually "Latent Sparse Attention at 10M tokens":
 *           "How the hierarchy is built", "What one query actually does".
 *   [BLOG]  sotaaz "Latent Sparse Attention: 72x in One Layer": "The same
 *           steps in general" (five steps and the short read_list function),
 *           "One real query, start to finish".
 *   [FORUM] zhichai "LSA: A Card-Catalog Approach": "Key points" (64-dim
 *           latent, L2-norm, pool 4, 512-key blocks, Ward, <=16 keys,
 *           Flat vs Tree).
 *
 * Readings taken where the pages are silent, labelled R1.. in this file:
 *   R1  64-term sums of squares use one fixed order: t_l = f(x_l) + f(x_{l+32})
 *       for l < 32, then t_l += t_{l+s} for s = 16, 8, 4, 2, 1; result t_0.
 *       No fused multiply-add anywhere on the build path.
 *   R2  window = [max(0, p - window), p] (513 keys with the query itself),
 *       as the blog's read_list writes it.
 *   R3  sink = {0 .. min(sink, p+1) - 1} (clipped to causal keys).
 *   R5  a query at p sees the buckets of blocks b < floor(p / 512).
 *   R6  buckets rank by (score desc, id asc); members ascend; Ward ties
 *       go to the lowest (i, j).
 *   R7  tree: pair nodes greedily by Ward cost inside consecutive runs of
 *       128 nodes, an odd leftover is promoted alone, until one root.
 *   R8  tree search: level-synchronous beam, candidates = children of kept
 *       nodes + visible nodes whose parent is not visible; keep
 *       max(W, ceil(P / 2^level)).
 *   R9  scores are taken on bf16 (round-to-nearest-even) copies of the
 *       normalised query and centroid.
 *   R10 the pooled key is the sum (not the mean) of 4 normalised keys.
 *   Zero-length key: its normalised form is the zero vector.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <float.h>

#define DIM 64
#define BLOCK_KEYS 512
#define N_POOL 4
#define ITEMS 128        /* pooled items per block = 512 / 4 */
#define TREE_RUN 128     /* nodes paired together at one tree level */

/* ---------- scalar helpers ---------- */

/* bf16 round to nearest even, from the IEEE definition of the format. */
uint16_t orc_f32_to_bf16(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x40u);
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7fffu + lsb;
    return (uint16_t)(u >> 16);
}

float orc_bf16_to_f32(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* R1: sum over 64 terms t_in[0..63] in the fixed pairwise order. */
static float r1_sum(const float *t_in)
{
    float t[32];
    for (int l = 0; l < 32; ++l) t[l] = t_in[l] + t_in[l + 32];
    for (int s = 16; s >= 1; s >>= 1)
        for (int l = 0; l < s; ++l) t[l] = t[l] + t[l + s];
    return t[0];
}

/* Sum of squares of a 64-vector in R1 order. */
float orc_sumsq(const float *x)
{
    float sq[DIM];
    for (int d = 0; d < DIM; ++d) sq[d] = x[d] * x[d];
    return r1_sum(sq);
}

/* Squared distance |a - b|^2 in R1 order. */
float orc_sqdist(const float *a, const float *b)
{
    float sq[DIM];
    for (int d = 0; d < DIM; ++d) {
        float e = a[d] - b[d];
        sq[d] = e * e;
    }
    return r1_sum(sq);
}

/* Length-normalise: out = x / sqrt(sum x^2) ([EXPL] "How the hierarchy is
 * built" and [FORUM] "Key points": keys are scaled to unit length).  Zero
 * vector -> zero. */
void orc_normalize(const float *x, float *out)
{
    float n = sqrtf(orc_sumsq(x));
    for (int d = 0; d < DIM; ++d) out[d] = (n > 0.0f) ? x[d] / n : 0.0f;
}

/* ---------- step a1: normalise and pool ---------- */

/* [EXPL] "How the hierarchy is built": every n_pool = 4 consecutive
 * normalised keys are summed into one pooled key.  keys: [4*n_items, 64],
 * pooled: [n_items, 64]. */
void orc_pool_norm(const float *keys, int64_t n_items, float *pooled)
{
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < n_items; ++j) {
        float nk[N_POOL][DIM];
        for (int e = 0; e < N_POOL; ++e) orc_normalize(keys + (4 * j + e) * DIM, nk[e]);
        for (int d = 0; d < DIM; ++d)
            pooled[j * DIM + d] = ((nk[0][d] + nk[1][d]) + nk[2][d]) + nk[3][d];
    }
}

/* ---------- step a2: Ward clustering of one block ---------- */

/* [EXPL] "How the hierarchy is built": a full block's pooled keys are
 * clustered bottom-up by Ward's criterion down to a fixed bucket count;
 * [BLOG] step 2: buckets average 8 keys and hold no more than 16; Ward 1963
 * for the criterion.
 *
 * items: [m, 64] pooled keys (unit weight each).  Merge cost of clusters A, B:
 *   D(A,B) = n_A n_B / (n_A + n_B) * |mu_A - mu_B|^2   (increase of the SSE),
 * kept current with the Lance-Williams recurrence for Ward:
 *   D(k, A+B) = ((n_A+n_k) D(k,A) + (n_B+n_k) D(k,B) - n_k D(A,B)) / (n_A+n_B+n_k).
 * Repeatedly merge the eligible pair (n_A + n_B <= cap) of least cost, ties to
 * the lowest (i, j), keeping the lower id, until n_target clusters remain.
 * root[i] <- id of the surviving cluster holding item i.
 * trace_i/j/d (nullable, one entry per merge) record each merge.
 * Returns the number of merges made. */
int orc_ward(const float *items, int m, int cap, int n_target, int32_t *root,
             int32_t *trace_i, int32_t *trace_j, float *trace_d)
{
    float *D = (float *)malloc(sizeof(float) * (size_t)m * (size_t)m);
    int *n = (int *)malloc(sizeof(int) * (size_t)m);
    char *live = (char *)malloc((size_t)m);
    for (int i = 0; i < m; ++i) { n[i] = 1; live[i] = 1; root[i] = i; }
    for (int i = 0; i < m; ++i) {
        D[(size_t)i * m + i] = 0.0f;
        for (int j = i + 1; j < m; ++j) {
            float v = 0.5f * orc_sqdist(items + (size_t)i * DIM, items + (size_t)j * DIM);
            D[(size_t)i * m + j] = v;
            D[(size_t)j * m + i] = v;
        }
    }
    int clusters = m, merges = 0;
    while (clusters > n_target) {
        float best = INFINITY;
        int bi = -1, bj = -1;
        for (int i = 0; i < m; ++i) {
            if (!live[i]) continue;
            for (int j = i + 1; j < m; ++j) {
                if (!live[j] || n[i] + n[j] > cap) continue;
                if (D[(size_t)i * m + j] < best) { best = D[(size_t)i * m + j]; bi = i; bj = j; }
            }
        }
        if (bi < 0) break;
        float dij = D[(size_t)bi * m + bj];
        for (int k = 0; k < m; ++k) {
            if (!live[k] || k == bi || k == bj) continue;
            float a = (float)(n[bi] + n[k]) * D[(size_t)k * m + bi];
            float b = (float)(n[bj] + n[k]) * D[(size_t)k * m + bj];
            float c = (float)n[k] * dij;
            float v = ((a + b) - c) / (float)(n[bi] + n[bj] + n[k]);
            D[(size_t)k * m + bi] = v;
            D[(size_t)bi * m + k] = v;
        }
        n[bi] += n[bj];
        live[bj] = 0;
        for (int t = 0; t < m; ++t)
            if (root[t] == bj) root[t] = bi;
        if (trace_i) { trace_i[merges] = bi; trace_j[merges] = bj; trace_d[merges] = dij; }
        ++merges;
        --clusters;
    }
    free(D); free(n); free(live);
    return merges;
}

/* Build the bucket cache for all complete blocks of keys[0..T).
 * Outputs (per block b, bucket r in 0..63, global id g = 64 b + r):
 *   pooled [T/4, 64]; item_bucket [nblk, 128] (u8, bucket of each item);
 *   members [nb, 16] ascending key positions, -1 padded; count [nb] keys;
 *   centroid [nb, 64] = normalise(sum of member pooled keys, ascending items);
 *   centroid_bf16 [nb, 64].  Buckets of a block are ordered by their lowest
 *   item.  Returns the number of complete blocks, or -1 if a block could not
 *   reach n_buckets (impossible for finite inputs, kept as a check). */
int64_t orc_build_cache(const float *keys, int64_t T, int cap_items, int n_buckets,
                        float *pooled, uint8_t *item_bucket, int32_t *members, int32_t *count,
                        float *centroid, uint16_t *centroid_bf16)
{
    int64_t n_items = T / N_POOL;
    int64_t nblk = T / BLOCK_KEYS;
    orc_pool_norm(keys, n_items, pooled);
    int failed = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : failed)
    for (int64_t b = 0; b < nblk; ++b) {
        const float *y = pooled + b * ITEMS * DIM;
        int32_t root[ITEMS];
        int merges = orc_ward(y, ITEMS, cap_items, n_buckets, root, NULL, NULL, NULL);
        if (merges != ITEMS - n_buckets) { failed = 1; continue; }
        int rank_of[ITEMS];
        int r = 0;
        for (int i = 0; i < ITEMS; ++i) rank_of[i] = (root[i] == i) ? r++ : -1;
        for (int i = 0; i < ITEMS; ++i) item_bucket[b * ITEMS + i] = (uint8_t)rank_of[root[i]];
        for (int i = 0; i < ITEMS; ++i) {
            if (root[i] != i) continue;
            int64_t g = b * n_buckets + rank_of[i];
            int32_t *mem = members + g * 16;
            int cnt = 0;
            float sum[DIM];
            for (int d = 0; d < DIM; ++d) sum[d] = 0.0f;
            for (int t = 0; t < ITEMS; ++t) {
                if (root[t] != i) continue;
                for (int e = 0; e < N_POOL; ++e) mem[cnt++] = (int32_t)(b * BLOCK_KEYS + N_POOL * t + e);
                for (int d = 0; d < DIM; ++d) sum[d] = sum[d] + y[t * DIM + d];
            }
            count[g] = cnt;
            for (int s = cnt; s < 16; ++s) mem[s] = -1;
            orc_normalize(sum, centroid + g * DIM);
            for (int d = 0; d < DIM; ++d) centroid_bf16[g * DIM + d] = orc_f32_to_bf16(centroid[g * DIM + d]);
        }
    }
    return failed ? -1 : nblk;
}

/* ---------- step a3: the tree of merged buckets ---------- */

/* Greedy Ward pairing of one run of m nodes ([EXPL] "How the hierarchy is
 * built", tree variant: the buckets are merged again, level after level;
 * [FORUM] "Key points": a binary tree over the buckets).  mu: [m, 64] node means, w: [m] weights (pooled items).
 * D(A,B) = (w_A w_B / (w_A + w_B)) |mu_A - mu_B|^2; repeatedly pair the two
 * unpaired nodes of least cost (ties to the lowest (i, j)).  partner[i] <- the
 * node paired with i, or -1 if i stays alone. */
void orc_pair_run(const float *mu, const int32_t *w, int m, int32_t *partner)
{
    float *D = (float *)malloc(sizeof(float) * (size_t)m * (size_t)m + 1);
    for (int i = 0; i < m; ++i) {
        partner[i] = -1;
        for (int j = i + 1; j < m; ++j) {
            float f = ((float)w[i] * (float)w[j]) / (float)(w[i] + w[j]);
            D[(size_t)i * m + j] = f * orc_sqdist(mu + (size_t)i * DIM, mu + (size_t)j * DIM);
        }
    }
    for (;;) {
        float best = INFINITY;
        int bi = -1, bj = -1;
        for (int i = 0; i < m; ++i) {
            if (partner[i] >= 0) continue;
            for (int j = i + 1; j < m; ++j) {
                if (partner[j] >= 0) continue;
                if (D[(size_t)i * m + j] < best) { best = D[(size_t)i * m + j]; bi = i; bj = j; }
            }
        }
        if (bi < 0) break;
        partner[bi] = bj;
        partner[bj] = bi;
    }
    /* Only non-finite costs can leave more than one node unpaired; pair the
     * rest in index order so every run still yields ceil(m/2) nodes. */
    int open = -1, left = 0;
    for (int i = 0; i < m; ++i) left += (partner[i] < 0);
    for (int i = 0; i < m && left > 1; ++i) {
        if (partner[i] >= 0) continue;
        if (open < 0) {
            open = i;
        } else {
            partner[open] = i;
            partner[i] = open;
            open = -1;
            left -= 2;
        }
    }
    free(D);
}

/* Number of levels (level 0 = buckets, top level = one root) and the node
 * count of each level: n_0 = nb, n_l = ceil(n_{l-1} / 2). */
int orc_tree_levels(int64_t nb, int64_t *level_size, int max_levels)
{
    int L = 0;
    int64_t n = nb;
    level_size[L++] = n;
    while (n > 1 && L < max_levels) {
        n = (n + 1) / 2;
        level_size[L++] = n;
    }
    return L;
}

/* Build every level above the buckets.  Nodes are addressed by global id
 * (level offsets are the prefix sums of level sizes).  Per node: child
 * [n,2] (-1 = none), parent [n] (-1 at the top), weight [n] (pooled items),
 * min_block/max_block [n], sum [n,64] (sum of the pooled keys of its leaves:
 * a leaf's sum runs over its member items in ascending order, a parent's
 * sum is child0 + child1), centroid [n,64] = normalise(sum), centroid_bf16.
 * At each level, consecutive runs of 128 nodes are paired (R7); the new
 * nodes are ordered by their lower child. */
int orc_build_tree(const float *pooled, const int32_t *members, const int32_t *count, int64_t nblk,
                   int n_buckets, int32_t *child, int32_t *parent, int32_t *weight,
                   int32_t *min_block, int32_t *max_block, float *sum, float *centroid,
                   uint16_t *centroid_bf16, int64_t *level_size, int max_levels)
{
    int64_t nb = nblk * n_buckets;
    int L = orc_tree_levels(nb, level_size, max_levels);
    /* level 0 */
#pragma omp parallel for schedule(static)
    for (int64_t g = 0; g < nb; ++g) {
        float *s = sum + g * DIM;
        for (int d = 0; d < DIM; ++d) s[d] = 0.0f;
        for (int e = 0; e < count[g]; e += N_POOL) {
            int64_t item = members[g * 16 + e] / N_POOL;
            for (int d = 0; d < DIM; ++d) s[d] = s[d] + pooled[item * DIM + d];
        }
        weight[g] = count[g] / N_POOL;
        min_block[g] = max_block[g] = (int32_t)(g / n_buckets);
        child[2 * g] = child[2 * g + 1] = -1;
        parent[g] = -1;
        orc_normalize(s, centroid + g * DIM);
        for (int d = 0; d < DIM; ++d) centroid_bf16[g * DIM + d] = orc_f32_to_bf16(centroid[g * DIM + d]);
    }
    int64_t off_prev = 0, off = nb;
    for (int l = 1; l < L; ++l) {
        int64_t n_prev = level_size[l - 1];
        int64_t n_runs = (n_prev + TREE_RUN - 1) / TREE_RUN;
#pragma omp parallel for schedule(dynamic, 1)
        for (int64_t r = 0; r < n_runs; ++r) {
            int64_t first = r * TREE_RUN;
            int m = (int)((n_prev - first) < TREE_RUN ? (n_prev - first) : TREE_RUN);
            float mu[TREE_RUN * DIM];
            int32_t w[TREE_RUN], partner[TREE_RUN];
            for (int i = 0; i < m; ++i) {
                int64_t v = off_prev + first + i;
                w[i] = weight[v];
                for (int d = 0; d < DIM; ++d) mu[i * DIM + d] = sum[v * DIM + d] / (float)w[i];
            }
            orc_pair_run(mu, w, m, partner);
            /* new nodes: one per pair (at its lower member) or lone node */
            int64_t out = off + first / 2; /* full runs of 128 give 64 nodes */
            for (int i = 0; i < m; ++i) {
                if (partner[i] >= 0 && partner[i] < i) continue;
                int64_t a = off_prev + first + i;
                int64_t b = partner[i] >= 0 ? off_prev + first + partner[i] : -1;
                child[2 * out] = (int32_t)(a - off_prev);
                child[2 * out + 1] = b >= 0 ? (int32_t)(b - off_prev) : -1;
                parent[a] = (int32_t)(out - off);
                weight[out] = weight[a] + (b >= 0 ? weight[b] : 0);
                min_block[out] = min_block[a];
                max_block[out] = max_block[a];
                if (b >= 0 && min_block[b] < min_block[out]) min_block[out] = min_block[b];
                if (b >= 0 && max_block[b] > max_block[out]) max_block[out] = max_block[b];
                for (int d = 0; d < DIM; ++d)
                    sum[out * DIM + d] = b >= 0 ? sum[a * DIM + d] + sum[b * DIM + d] : sum[a * DIM + d];
                if (b >= 0) parent[b] = (int32_t)(out - off);
                parent[out] = -1;
                orc_normalize(sum + out * DIM, centroid + out * DIM);
                for (int d = 0; d < DIM; ++d)
                    centroid_bf16[out * DIM + d] = orc_f32_to_bf16(centroid[out * DIM + d]);
                ++out;
            }
        }
        off_prev = off;
        off += level_size[l];
    }
    return L;
}

/* ---------- steps a4-a7: one query ---------- */

/* [EXPL] "What one query actually does": the query is scaled to unit
 * length first; R9: bf16 copy of the normalised query. */
void orc_qnorm(const float *q, int64_t nq, uint16_t *qhat)
{
    for (int64_t i = 0; i < nq; ++i) {
        float n[DIM];
        orc_normalize(q + i * DIM, n);
        for (int d = 0; d < DIM; ++d) qhat[i * DIM + d] = orc_f32_to_bf16(n[d]);
    }
}

/* Score of one centroid: dot product of the bf16 operands, summed exactly in
 * fp64 and rounded once to fp32. */
float orc_score(const uint16_t *qhat, const uint16_t *cbf)
{
    double s = 0.0;
    for (int d = 0; d < DIM; ++d) s += (double)orc_bf16_to_f32(qhat[d]) * (double)orc_bf16_to_f32(cbf[d]);
    return (float)s;
}

typedef struct { float s; int32_t id; } scored_t;

static int cmp_rank(const void *a, const void *b)
{
    const scored_t *x = (const scored_t *)a, *y = (const scored_t *)b;
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
    return (x->id > y->id) - (x->id < y->id);
}

/* Flat search ([EXPL] "What one query actually does": every centroid of the
 * earlier blocks is scored and the best buckets are kept; [FORUM] "Key
 * points", Flat vs Tree): score every bucket of blocks 0..H-1, rank by
 * (score desc, id asc).  Writes all 64*H ranked ids/scores; returns their number. */
int64_t orc_flat_rank(const uint16_t *qhat, int64_t H, int n_buckets, const uint16_t *cbf,
                      int32_t *ids, float *scores)
{
    int64_t n = H * n_buckets;
    scored_t *v = (scored_t *)malloc(sizeof(scored_t) * (size_t)(n > 0 ? n : 1));
    for (int64_t b = 0; b < n; ++b) { v[b].s = orc_score(qhat, cbf + b * DIM); v[b].id = (int32_t)b; }
    qsort(v, (size_t)n, sizeof(scored_t), cmp_rank);
    for (int64_t i = 0; i < n; ++i) { ids[i] = v[i].id; if (scores) scores[i] = v[i].s; }
    free(v);
    return n;
}

/* Tree search (R8; [EXPL] "What one query actually does" and the
 * search-style table: each level opens only the children of the nodes kept at
 * the level above; [FORUM] "Key points": a beam per level).  A node is visible iff all its
 * blocks are < H.  Candidates at level l = children of the nodes kept at
 * level l+1, plus visible level-l nodes whose parent is not visible (or that
 * have no parent).  Keep the best max(W, ceil(P / 2^l)) by (score desc, id
 * asc).  The buckets kept at level 0 are returned ranked (local ids).
 * kept_per_level (NULL, or n_levels entries) receives how many nodes each
 * level kept, a trace for tests; it changes nothing in the search. */
int64_t orc_tree_rank(const uint16_t *qhat, int64_t H, const int32_t *child, const int32_t *parent,
                      const int32_t *max_block, const uint16_t *cbf, const int64_t *level_size,
                      int n_levels, int W, int64_t P, int32_t *ids, float *scores, int64_t *kept_per_level)
{
    int64_t *off = (int64_t *)malloc(sizeof(int64_t) * (size_t)(n_levels + 1));
    off[0] = 0;
    for (int l = 0; l < n_levels; ++l) off[l + 1] = off[l] + level_size[l];
    int64_t cap = 16;
    for (int l = 0; l < n_levels; ++l) cap += level_size[l];
    scored_t *cand = (scored_t *)malloc(sizeof(scored_t) * (size_t)cap);
    int32_t *kept = (int32_t *)malloc(sizeof(int32_t) * (size_t)cap);
    int64_t n_kept = 0;
    for (int l = n_levels - 1; l >= 0; --l) {
        int64_t nc = 0;
        for (int64_t i = 0; i < n_kept; ++i) {
            int64_t v = off[l + 1] + kept[i];
            for (int c = 0; c < 2; ++c)
                if (child[2 * v + c] >= 0) cand[nc++].id = child[2 * v + c];
        }
        for (int64_t u = 0; u < level_size[l]; ++u) {
            int64_t v = off[l] + u;
            if (max_block[v] >= H) continue;
            int top = (l == n_levels - 1);
            if (!top && max_block[off[l + 1] + parent[v]] < H) continue;
            cand[nc++].id = (int32_t)u;
        }
        for (int64_t i = 0; i < nc; ++i) cand[i].s = orc_score(qhat, cbf + (off[l] + cand[i].id) * DIM);
        qsort(cand, (size_t)nc, sizeof(scored_t), cmp_rank);
        int64_t B = (P + ((int64_t)1 << l) - 1) >> l;
        if (B < W) B = W;
        n_kept = nc < B ? nc : B;
        if (kept_per_level) kept_per_level[l] = n_kept;
        for (int64_t i = 0; i < n_kept; ++i) kept[i] = cand[i].id;
        if (l == 0)
            for (int64_t i = 0; i < n_kept; ++i) { ids[i] = cand[i].id; if (scores) scores[i] = cand[i].s; }
    }
    free(off); free(cand); free(kept);
    return n_kept;
}

static int cmp_i32(const void *a, const void *b)
{
    int32_t x = *(const int32_t *)a, y = *(const int32_t *)b;
    return (x > y) - (x < y);
}

/* Open the ranked buckets best first and add sink + window ([BLOG] steps 4-5
 * and read_list; [EXPL] "What one query actually does": buckets turn into
 * key positions in rank order until k long-range keys are in, and the sink
 * and the recent window are always added).
 * near = {0..min(sink,p+1)-1} U [max(0,p-window), p]; members already in
 * near are skipped and the next one takes their place; stop at k far keys.
 * out[0..len) = sorted(near U far), out[len..Lmax) = -1.  Returns len. */
int orc_expand(const int32_t *ranked, int64_t n_ranked, const int32_t *members, const int32_t *count,
               int64_t p, int k, int sink, int window, int32_t *out, int Lmax)
{
    int64_t w0 = p - window > 0 ? p - window : 0;
    int64_t s_end = sink < p + 1 ? sink : p + 1;
    int32_t *all = (int32_t *)malloc(sizeof(int32_t) * (size_t)(k + sink + window + 2));
    int n = 0, nfar = 0;
    for (int64_t r = 0; r < n_ranked && nfar < k; ++r) {
        const int32_t *mem = members + (int64_t)ranked[r] * 16;
        for (int e = 0; e < count[ranked[r]] && nfar < k; ++e) {
            int64_t m = mem[e];
            if (m < s_end || (m >= w0 && m <= p)) continue;
            all[n++] = (int32_t)m;
            ++nfar;
        }
    }
    for (int64_t t = 0; t < s_end; ++t)
        if (t < w0) all[n++] = (int32_t)t;
    for (int64_t t = w0; t <= p; ++t) all[n++] = (int32_t)t;
    qsort(all, (size_t)n, sizeof(int32_t), cmp_i32);
    for (int i = 0; i < Lmax; ++i) out[i] = i < n ? all[i] : -1;
    free(all);
    return n;
}

/* The whole indexer for nq queries at positions pos[] against a cache of
 * nblk complete blocks.  mode 0 = Flat, 1 = Tree (tree arrays non-null).
 * Horizon H(p) = min(floor(p / 512), nblk).  lists [nq, Lmax], lens [nq]. */
int orc_index(const float *qidx, const int64_t *pos, int64_t nq, int64_t nblk, int n_buckets,
              const int32_t *members, const int32_t *count, const uint16_t *centroid_bf16,
              int mode, const int32_t *child, const int32_t *parent, const int32_t *max_block,
              const uint16_t *tree_cbf, const int64_t *level_size, int n_levels,
              int k, int sink, int window, int beam, int32_t *lists, int32_t *lens, int Lmax)
{
    int64_t P = (k + sink + window + N_POOL - 1) / N_POOL;
    int64_t nb = nblk * n_buckets;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int64_t i = 0; i < nq; ++i) {
        uint16_t qh[DIM];
        orc_qnorm(qidx + i * DIM, 1, qh);
        int64_t H = pos[i] / BLOCK_KEYS;
        if (H > nblk) H = nblk;
        int32_t *ids = (int32_t *)malloc(sizeof(int32_t) * (size_t)(nb > 0 ? nb : 1));
        int64_t nr;
        if (mode == 0)
            nr = orc_flat_rank(qh, H, n_buckets, centroid_bf16, ids, NULL);
        else
            nr = orc_tree_rank(qh, H, child, parent, max_block, tree_cbf, level_size, n_levels,
                               beam, P, ids, NULL, NULL);
        if (nr < 0) bad = 1;
        lens[i] = orc_expand(ids, nr, members, count, pos[i], k, sink, window, lists + i * Lmax, Lmax);
        free(ids);
    }
    return bad ? -1 : 0;
}

/* Multi-head Flat search (zhichai forum post, "Key points": N-LSA selects
 * buckets by the best score across heads).  Every query carries n_heads
 * 64-dim index queries; a bucket's score is the largest of its n_heads
 * scores (each the exact fp64 sum rounded once to fp32, as orc_score), and
 * buckets rank by (that score desc, id asc).  Then the same expansion.
 * qidx [nq, n_heads, 64]. */
int orc_index_heads(const float *qidx, const int64_t *pos, int64_t nq, int n_heads, int64_t nblk, int n_buckets,
                    const int32_t *members, const int32_t *count, const uint16_t *centroid_bf16, int k, int sink,
                    int window, int32_t *lists, int32_t *lens, int Lmax)
{
    int64_t nb = nblk * n_buckets;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int64_t i = 0; i < nq; ++i) {
        uint16_t *qh = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)n_heads * DIM);
        for (int h = 0; h < n_heads; ++h) orc_qnorm(qidx + (i * n_heads + h) * DIM, 1, qh + h * DIM);
        int64_t H = pos[i] / BLOCK_KEYS;
        if (H > nblk) H = nblk;
        int64_t n = H * n_buckets;
        scored_t *v = (scored_t *)malloc(sizeof(scored_t) * (size_t)(n > 0 ? n : 1));
        int32_t *ids = (int32_t *)malloc(sizeof(int32_t) * (size_t)(nb > 0 ? nb : 1));
        for (int64_t b = 0; b < n; ++b) {
            float best = orc_score(qh, centroid_bf16 + b * DIM);
            for (int h = 1; h < n_heads; ++h) {
                float s = orc_score(qh + h * DIM, centroid_bf16 + b * DIM);
                if (s > best) best = s;
            }
            v[b].s = best;
            v[b].id = (int32_t)b;
        }
        qsort(v, (size_t)n, sizeof(scored_t), cmp_rank);
        for (int64_t j = 0; j < n; ++j) ids[j] = v[j].id;
        lens[i] = orc_expand(ids, n, members, count, pos[i], k, sink, window, lists + i * Lmax, Lmax);
        free(v); free(ids); free(qh);
    }
    return bad ? -1 : 0;
}

/* ---------- step a8: exact softmax attention over each list ---------- */

/* [EXPL] "What one query actually does": plain softmax attention over the
 * sink, the chosen keys and the window; one list per query serves all its
 * heads.  Q [nq,Hq,dh], K/V [Tk,Hkv,dh]
 * as bf16 bits; query head h reads KV head floor(h*Hkv/Hq).  Computed in fp64:
 * O = sum_j softmax_j(scale * q.k_j) v_j; lse = max + log(sum exp).  O, lse
 * are rounded to fp32 at the end. */
void orc_attention(const uint16_t *Q, const uint16_t *K, const uint16_t *V, int64_t nq, int Hq,
                   int Hkv, int dh, const int32_t *lists, const int32_t *lens, int Lmax, float scale,
                   float *O, float *lse)
{
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t i = 0; i < nq; ++i) {
        int len = lens[i];
        double *s = (double *)malloc(sizeof(double) * (size_t)(len > 0 ? len : 1));
        double *acc = (double *)malloc(sizeof(double) * (size_t)dh);
        for (int h = 0; h < Hq; ++h) {
            int g = (int)(((int64_t)h * Hkv) / Hq);
            const uint16_t *q = Q + (i * Hq + h) * (int64_t)dh;
            double mx = -INFINITY;
            for (int j = 0; j < len; ++j) {
                const uint16_t *kk = K + ((int64_t)lists[i * Lmax + j] * Hkv + g) * dh;
                double dot = 0.0;
                for (int d = 0; d < dh; ++d) dot += (double)orc_bf16_to_f32(q[d]) * (double)orc_bf16_to_f32(kk[d]);
                s[j] = dot * (double)scale;
                if (s[j] > mx) mx = s[j];
            }
            double l = 0.0;
            for (int d = 0; d < dh; ++d) acc[d] = 0.0;
            for (int j = 0; j < len; ++j) {
                double e = exp(s[j] - mx);
                l += e;
                const uint16_t *vv = V + ((int64_t)lists[i * Lmax + j] * Hkv + g) * dh;
                for (int d = 0; d < dh; ++d) acc[d] += e * (double)orc_bf16_to_f32(vv[d]);
            }
            float *o = O + (i * Hq + h) * (int64_t)dh;
            for (int d = 0; d < dh; ++d) o[d] = (float)(acc[d] / l);
            if (lse) lse[i * Hq + h] = (float)(mx + log(l));
        }
        free(s); free(acc);
    }
}
