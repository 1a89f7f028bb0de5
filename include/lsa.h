/*
 * lsa.h -- C ABI of the B200 (sm_100a) implementation of Latent Sparse
 * Attention's hot path for one layer: the indexer (normalise + pool, Ward
 * bucket cache, Flat or Tree search, best-first expansion + sink + window)
 * and the exact GQA sparse attention over the resulting index lists.
 *
 * Method sources (web pages on "Latent Sparse Attention: Towards
 * Subquadratic Ultra-Long Context Attention", arXiv 2610.42147):
 *   [EXPL]  learnaivisually explainer: "How the hierarchy is built",
 *           "What one query actually does", "Search style" table.
 *   [BLOG]  sotaaz blog: "The same steps in general" (five steps and the
 *           read_list function), "One real query, start to finish".
 *   [FORUM] zhichai forum post: "Key points" (64-dim latent, L2 norm,
 *           pool 4, 512-key blocks, Ward, <= 16 keys, Flat vs Tree).
 *
 * Conventions for every call below.
 *   - Pointers to tensors are DEVICE pointers owned by the caller; the
 *     library never allocates, frees or keeps them.  Scratch space is a
 *     caller-provided device workspace sized by the *_workspace_bytes
 *     queries.  lsa_cache / lsa_tree are host structs of device pointers.
 *   - Every tensor is dense and row-major.  bf16 tensors are passed as
 *     uint16_t bit patterns.  Device pointers must be 16-byte aligned.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Calls only enqueue work: they return before it runs, and
 *     outputs are valid once the stream reaches that point.
 *   - Return value: LSA_OK (0) or a negative LSA_ERR_* code; nothing is
 *     enqueued when an argument check fails.  lsa_last_error_string()
 *     describes the last failure on the calling thread.  The library never
 *     aborts the process and its kernels never trap.
 *   - Only the pages' configuration is built: 64-dim index vectors,
 *     n_pool = 4, 512-key blocks, 64 buckets per block, at most 4 pooled
 *     items (16 keys) per bucket, attention head_dim 128.  Other values in
 *     lsa_params are rejected with LSA_ERR_ARG.
 */
#ifndef LSA_H
#define LSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define LSA_DIM 64           /* index key / query width           ([FORUM] Key points) */
#define LSA_BLOCK 512        /* keys per cluster block            ([FORUM] Key points) */
#define LSA_N_POOL 4         /* keys summed into one pooled key   ([EXPL] hierarchy)   */
#define LSA_ITEMS 128        /* pooled items per block = 512 / 4                       */
#define LSA_BUCKETS 64       /* buckets per block (~8 keys each)  ([BLOG] step 2)      */
#define LSA_SLOTS 16         /* member slots per bucket (<= 16 keys, [BLOG] step 2)    */
#define LSA_HEAD_DIM 128     /* attention head width handled by lsa_sparse_attention   */
#define LSA_MAX_LEVELS 40    /* tree levels (ceil(log2(buckets)) + 1 <= 40)            */
#define LSA_MAX_INDEX_HEADS 16 /* index queries per token in multi-head Flat search     */

enum {
    LSA_OK = 0,
    LSA_ERR_ARG = -1,       /* null/misaligned pointer, bad parameter value */
    LSA_ERR_SHAPE = -2,     /* sizes inconsistent with each other or with a buffer */
    LSA_ERR_CUDA = -3,      /* a CUDA launch or query failed */
    LSA_ERR_TIMEOUT = -4,   /* a bounded device-side wait gave up (reserved) */
    LSA_ERR_WORKSPACE = -5  /* workspace missing or smaller than required */
};

enum { LSA_MODE_FLAT = 0, LSA_MODE_TREE = 1 };

/* Parameters of the method.  lsa_default_params() fills the pages' values:
 * n_pool 4, block 512, n_buckets 64, cap_items 4, sink 4, window 512 ([BLOG]
 * step 5: four sink keys and the newest 512 keys are always read), k 4096
 * ([BLOG] step 4: the long-range key budget given for the Qwen model),
 * beam 32, mode Flat.
 * cand_cap: per-query candidate slots of the Flat search (0 = automatic).
 * A smaller value only routes more queries through the exact fallback
 * selection; results do not change.
 * index_heads: index queries per token, 1..LSA_MAX_INDEX_HEADS (default 1).
 * With more than one, Flat search ranks a bucket by the largest of its
 * per-head scores (zhichai forum post, "Key points": N-LSA's bucket
 * selection); qidx is then [nq, index_heads, 64].  Tree mode takes 1 only. */
typedef struct lsa_params {
    int32_t n_pool;
    int32_t block;
    int32_t n_buckets;
    int32_t cap_items;
    int32_t sink;
    int32_t window;
    int32_t k;
    int32_t beam;
    int32_t mode;
    int32_t cand_cap;
    int32_t index_heads;
} lsa_params;

/* Bucket cache ([EXPL] "How the hierarchy is built": a bucket keeps a
 * centroid and the positions of its keys, and a clustered block is never
 * touched again).  Bucket g = 64*b + r is the r-th bucket of block b, buckets of a
 * block ordered by their lowest pooled item.
 *   pooled        fp32 [capacity/4, 64]   sum of 4 normalised keys per item
 *   item_bucket   u8   [capacity/512, 128] bucket (0..63) of each pooled item
 *   members       i32  [nb, 16]  ascending key positions, -1 padded
 *   count         i32  [nb]      keys in the bucket (4..16)
 *   centroid      fp32 [nb, 64]  normalised sum of member pooled keys
 *   centroid_bf16 u16  [nb, 64]  bf16 (round to nearest even) of centroid
 * where nb = 64 * (capacity / 512).  n_blocks = complete blocks clustered so
 * far; lsa_build_cache raises it.  Fill the struct with lsa_cache_bind. */
typedef struct lsa_cache {
    int64_t capacity;
    int64_t n_blocks;
    float *pooled;
    uint8_t *item_bucket;
    int32_t *members;
    int32_t *count;
    float *centroid;
    uint16_t *centroid_bf16;
} lsa_cache;

/* Tree of merged buckets ([EXPL] "How the hierarchy is built": the tree
 * variant merges buckets again, level after level; [FORUM] "Key points": a
 * binary tree over the buckets).  Level 0 = the buckets; level l has ceil(n_{l-1}/2)
 * nodes; the top level holds the root.  Node arrays are indexed by global
 * id = level_offset[l] + local id; child/parent hold LOCAL ids of the level
 * below/above.
 *   child [n,2] (-1 = none), parent [n] (-1 at the top), weight [n] (pooled
 *   items below), min_block / max_block [n], sum fp32 [n,64] (sum of the
 *   leaves' pooled keys), centroid fp32 [n,64] = normalise(sum),
 *   centroid_bf16 [n,64].
 * Fill with lsa_tree_bind, which lays the levels out for its capacity
 * (level_offset fixed, level_size growing with the cache), so that a tree can
 * grow in place; lsa_build_tree / lsa_update_tree set n_blocks. */
typedef struct lsa_tree {
    int64_t n_blocks;
    int32_t n_levels;
    int32_t cap_blocks; /* capacity the buffer was bound for; level_offset is laid out for it */
    int64_t level_size[LSA_MAX_LEVELS];
    int64_t level_offset[LSA_MAX_LEVELS + 1];
    int32_t *child;
    int32_t *parent;
    int32_t *weight;
    int32_t *min_block;
    int32_t *max_block;
    float *sum;
    float *centroid;
    uint16_t *centroid_bf16;
} lsa_tree;

/* ---- parameters, sizes and buffer binding (host only, no GPU work) ---- */

void lsa_default_params(lsa_params *p);
const char *lsa_last_error_string(void);

/* Number of kernels this library has enqueued (all threads, all devices)
 * since it was loaded: instrumentation for benchmarks and tests. */
int64_t lsa_launch_count(void);

/* Device-side failure detection.  Every wait inside a kernel (the mbarrier
 * phases of the tensor-core score kernel's copy ring and accumulators) gives
 * up after a bounded number of tries instead of spinning forever; one that
 * gives up sets an error word on the device, and the kernel leaves its loops,
 * waits (bounded) for the copies it issued, frees its tensor memory and
 * exits, so the context stays usable.  lsa_check_device_errors() waits for
 * the current device to go idle, reads and clears that word: 0 = no wait ran
 * out, 1 = one did (outputs of that call are invalid and
 * lsa_last_error_string() says so), < 0 = CUDA error.
 * The debug build of the library (liblsa_debug.so, built with
 * -DLSA_BOUNDS_CHECKS=1) also checks, before use, the gather indices that
 * kernels read from memory -- the list entries the attention gathers K/V rows
 * with, the bucket ids and member positions the expansion reads, the child
 * ids the tree search follows -- and every list length; a failed check skips
 * the access (it never traps) and adds a code to the word:
 * 2 = an index-list entry outside [0, Tk) or not increasing, or a list length
 * above Lmax; 4 = a bucket id the query cannot see or a member position past
 * the cache; 8 = a tree-node id outside its level.  The release build
 * compiles these checks out.
 * lsa_debug_wait_test(1) is a test hook: in the next lsa_index_* call in
 * Flat mode every score CTA skips its query-tile copy, so the barrier that
 * waits for it never completes, and waits are cut to a short limit; the error
 * path then runs without hanging or faulting the GPU.
 * lsa_debug_wait_test(0) restores the normal limit. */
int lsa_check_device_errors(void);
void lsa_debug_wait_test(int32_t enable);

/* Test hook of lsa_sparse_attention: range_rows > 0 makes every batch with a
 * large enough workspace (sized after the hook is set) take the
 * position-range phases with ranges of range_rows positions, so that small
 * inputs exercise that path; range_rows < 0 turns the phases off; 0
 * restores the automatic choice. */
void lsa_debug_attention_ranges(int64_t range_rows);

/* Tuning and test hook of Flat search.  A single-head Flat query that sees
 * at least stride x 4096 buckets takes its threshold tau from every
 * stride-th tile of 128 centroids (stride 16 and margin 0.9 by default):
 * tau is set so that about margin x P of the visible buckets lie above it.
 * Every bucket at or above tau is still ranked, so the result is the exact
 * one; a query whose buckets above tau hold fewer than k far keys is redone
 * by the exact selection.  stride <= 1 turns the sampling off (the exact
 * histogram of all buckets); a small margin (e.g. 0.01) makes the exact
 * redo happen, which tests exercise. */
void lsa_debug_score_sample(int32_t stride, float margin);

/* Per-kernel timing, a profiling aid.  While enabled (lsa_kernel_timing(1)),
 * every kernel the library launches is bracketed by two CUDA events recorded
 * on the stream it is launched on, tagged with the kernel's name (the
 * tensor-core score passes as "k_score_tc:threshold" and
 * "k_score_tc:filter"); nothing else changes.  lsa_kernel_timing_read waits
 * for the recorded events, sums milliseconds and launches per kernel name
 * since the last read, writes up to max_kernels of them (names as
 * NUL-terminated strings of name_len bytes each, in first-launch order) and
 * forgets the records.  Returns the number of distinct kernels (which may
 * exceed max_kernels), or LSA_ERR_CUDA.  Not thread-safe: enable, call and
 * read from one host thread; do not enable it around a stream capture. */
void lsa_kernel_timing(int32_t enable);
int lsa_kernel_timing_read(char *names, int32_t name_len, double *ms, int64_t *launches, int32_t max_kernels);


/* Longest index list: sink + window + 1 (the query itself) + k. */
int32_t lsa_list_budget(const lsa_params *p);

/* Buckets that always hold k far keys: ceil((k + sink + window) / 4)
 * (every bucket has >= 4 keys; at most sink + window clustered keys are
 * skipped as near).  The Flat search keeps exactly this many. */
int32_t lsa_top_buckets(const lsa_params *p);

/* Bytes of one device buffer holding a cache for `capacity` tokens, and the
 * call that carves such a buffer (256-byte aligned) into an lsa_cache. */
int64_t lsa_cache_bytes(int64_t capacity);
int lsa_cache_bind(void *base, int64_t bytes, int64_t capacity, lsa_cache *out);

/* Same for the tree over n_blocks complete blocks (all levels, level 0 too). */
int64_t lsa_tree_bytes(int64_t n_blocks);
int lsa_tree_bind(void *base, int64_t bytes, int64_t n_blocks, lsa_tree *out);

/* Workspace of lsa_index_prefill / lsa_index_decode for nq queries against a
 * cache of n_blocks blocks, and of lsa_sparse_attention for nq queries over
 * Tk keys (Tk = 0: size without the position-range phases). */
int64_t lsa_index_workspace_bytes(int64_t nq, int64_t n_blocks, const lsa_params *p);
int64_t lsa_attention_workspace_bytes(int64_t nq, int32_t Hq, int32_t head_dim, int32_t Lmax, int64_t Tk);

/* ---- the five calls of the hot path ---- */

/* Step 1, "Shrink" ([BLOG] "The same steps in general", step 1; [FORUM] "Key
 * points"): a linear map of each position's key to a 64-dim vector used only
 * to choose keys (trained per layer in D-LSA; a principal-component map is
 * reported to do about as well).  x_t = W v_t for every row
 * t_begin <= t < t_end of V, fp32 accumulation on the tensor cores.
 * V bf16 [>= t_end, D] (a position's row, e.g. its key over all KV heads,
 * D = Hkv x 128); W bf16 [64, D]; D a multiple of 64, <= 16384; V and W
 * 16-byte aligned.
 * keys (nullable) fp32 [>= t_end, 64]: x_t written at row t.
 * pooled (nullable) fp32 [>= t_end / 4, 64]: item j = sum of the normalised
 * x_4j .. x_4j+3, normalised and summed in the order lsa_build_cache uses,
 * for every item whose four rows lie in the range (t_begin % 4 == 0 then);
 * pass cache->pooled and then lsa_build_cache with keys = NULL to cluster
 * the completed blocks.  At least one of keys, pooled must be non-NULL. */
int lsa_shrink(const uint16_t *V, int64_t D, const uint16_t *W, int64_t t_begin, int64_t t_end, float *keys,
               float *pooled, void *stream);

/* Steps 1-2 of the indexer ([EXPL] "How the hierarchy is built"; [FORUM]
 * Key points; [BLOG] step 2).
 * keys: fp32 [>= t_end, 64], the index keys of positions 0..t_end-1.
 * Pools every item j with t_begin/4 <= j < t_end/4 (integer division):
 * n_t = x_t / |x_t|, y_j = n_4j + n_4j+1 + n_4j+2 + n_4j+3 (a zero key
 * normalises to zero).  Then clusters every block b with
 * t_begin/512 <= b < t_end/512 by Ward's method: 128 unit-weight pooled
 * items, cost D(A,B) = n_A n_B/(n_A+n_B) |mu_A - mu_B|^2, cheapest eligible
 * pair (n_A + n_B <= 4 items) merged first, ties to the lowest (i, j), until
 * 64 buckets remain.  All fp32 arithmetic of this call follows one fixed
 * order, so results are bit-for-bit reproducible.
 * Re-running over a range rewrites identical values.  Requires
 * t_end <= cache->capacity.  Sets cache->n_blocks = max(n_blocks, t_end/512).
 * keys = NULL skips the pooling: the range's items are already in
 * cache->pooled (written by lsa_shrink), and only the blocks are clustered. */
int lsa_build_cache(const float *keys, int64_t t_begin, int64_t t_end, lsa_cache *cache,
                    const lsa_params *p, void *stream);

/* Tree above the buckets of cache->n_blocks blocks ([EXPL] "How the
 * hierarchy is built", tree variant).  At every level,
 * consecutive runs of 128 nodes are paired greedily by Ward cost
 * (weights = pooled items, mu = sum / weight), ties to the lowest (i, j); an
 * odd leftover is promoted alone; new nodes are ordered by their lower
 * child; repeat until one root.  tree must be bound for >= cache->n_blocks. */
int lsa_build_tree(const lsa_cache *cache, lsa_tree *tree, const lsa_params *p, void *stream);

/* Grow a tree built over tree->n_blocks blocks to cache->n_blocks blocks
 * (decode: a block completes every 512 tokens; [EXPL] "How the hierarchy is
 * built": the clusters are made as the context grows).  The pairing of a run
 * of 128 nodes depends on that run alone, and every run but a level's last is
 * full, so new leaves change only the runs from the first new node on at
 * each level: those are paired again and everything else is kept.  The
 * result is bit-identical to lsa_build_tree over the same cache.  A tree
 * with n_blocks == 0 is built whole; cache->n_blocks < tree->n_blocks, or
 * more blocks than the tree was bound for, returns LSA_ERR_SHAPE. */
int lsa_update_tree(const lsa_cache *cache, lsa_tree *tree, const lsa_params *p, void *stream);

/* Steps 3-5 for nq queries ([EXPL] "What one query actually does"; [BLOG]
 * steps 3-5 and read_list).
 * qidx fp32 [nq, 64] index queries ([nq, p->index_heads, 64] with several
 * index heads); pos i64 [nq] their positions.  Query i
 * sees the buckets of blocks b < H = min(pos/512, cache->n_blocks).
 *   Flat (p->mode == LSA_MODE_FLAT, tree may be NULL): score every visible
 *   bucket, s = <bf16(q/|q|), centroid_bf16> with fp32 accumulation, rank by
 *   (score desc, bucket id asc).  Supports caches of up to 65535 blocks
 *   (33.5M tokens) and k + sink + window < 32768; larger requests return
 *   LSA_ERR_SHAPE.  With index_heads > 1 every head is normalised and scored
 *   on its own and a bucket ranks by its largest head score.
 *   Tree: level-synchronous beam search from the root: candidates at level l
 *   are the children of the nodes kept at level l+1 plus the visible
 *   level-l nodes whose parent is not visible; keep the best
 *   max(beam, ceil(lsa_top_buckets / 2^l)).
 * Then open the ranked buckets best first, skipping members in
 * near = {0..min(sink, p+1)-1} U [max(0, p-window), p], until k far keys.
 * lists i32 [nq, Lmax]: ascending positions of near U far, -1 padded;
 * lens i32 [nq].  Lmax must be >= lsa_list_budget(p).
 * ws: >= lsa_index_workspace_bytes(nq, cache->n_blocks, p) bytes. */
int lsa_index_prefill(const float *qidx, const int64_t *pos, int64_t nq, const lsa_cache *cache,
                      const lsa_tree *tree, int32_t *lists, int32_t *lens, int32_t Lmax,
                      const lsa_params *p, void *ws, int64_t ws_bytes, void *stream);

/* The same computation for a few new tokens (decode, batch nq, positions at
 * or past the clustered context).  Identical results to lsa_index_prefill;
 * the launch shape spreads each query's buckets over the whole GPU. */
int lsa_index_decode(const float *qidx, const int64_t *pos, int64_t nq, const lsa_cache *cache,
                     const lsa_tree *tree, int32_t *lists, int32_t *lens, int32_t Lmax,
                     const lsa_params *p, void *ws, int64_t ws_bytes, void *stream);

/* Exact softmax attention over each query's list, shared by all its heads
 * ([EXPL] "What one query actually does": one list per query serves every
 * head of that query, and plain softmax attention runs over it).
 * Q bf16 [nq, Hq, 128]; K, V bf16 [Tk, Hkv, 128]; query head h reads KV head
 * h / (Hq / Hkv) (Hq a multiple of Hkv, Hq / Hkv <= 16).  lists/lens as
 * written by lsa_index_*: each list strictly increasing, every listed
 * position < Tk.  Rows of K and V that no list holds may hold anything
 * (an unwritten cache tail, NaN included): the results depend on listed
 * rows only.
 * O[i,h] = sum_j softmax_j(scale * Q[i,h] . K[j]) V[j] over j in list(i),
 * fp32 softmax and accumulation; O bf16 [nq, Hq, 128]; lse fp32 [nq, Hq]
 * (natural-log log-sum-exp of the scaled scores; may be NULL).
 * ws: >= lsa_attention_workspace_bytes(nq, Hq, 128, Lmax, Tk) bytes.  It
 * holds the partial results when few queries split their lists over many
 * warps (decode), or, for batches of at least 64 queries whose KV head fits
 * in three quarters of L2 (Tk x 512 B), the near-set results of tiles of
 * consecutive queries: the run of consecutive positions that ends a list and
 * the run 0, 1, .. that starts it are read once per tile and merged with the
 * rest of each list by log-sum-exp.  For batches of at least 512 queries
 * whose KV head does not fit in L2, and lists long enough for at least 256
 * entries per range (Lmax >= 256 x ranges), it holds one running result per
 * (query, head) and the keys are taken in position ranges of about half of
 * L2 per head, one kernel launch per (KV head, range), so that the rows of a
 * range stay in L2 while every query reads them.  With a smaller workspace (or
 * none) fewer splits, no tiles or no ranges are used; results are the same
 * up to fp32 summation order. */
int lsa_sparse_attention(const uint16_t *Q, const uint16_t *K, const uint16_t *V, int64_t nq,
                         int32_t Hq, int32_t Hkv, int32_t head_dim, int64_t Tk, const int32_t *lists,
                         const int32_t *lens, int32_t Lmax, float scale, uint16_t *O, float *lse,
                         void *ws, int64_t ws_bytes, void *stream);

/* ---- decode indexing without a caller workspace ---- */

/* Size of the fixed device scratch array behind lsa_index_decode_static. */
#define LSA_STATIC_SCRATCH_BYTES (16u << 20)

/* lsa_index_decode for callers that cannot allocate device memory (an engine
 * that has reserved all device memory up front and gives its plugins no
 * allocator, a host program that only holds pointers handed to it, a decode
 * loop that must never stall on a cudaMalloc/cudaFree).  The LSA pages have
 * no counterpart: this is a deployment convenience, not part of the method.
 *
 * Same arguments, results and errors as lsa_index_decode, without ws and
 * ws_bytes: the scratch is one file-scope device array of
 * LSA_STATIC_SCRATCH_BYTES (16 MiB) that every GPU loading the library holds
 * until the process exits.  The call allocates nothing.  Requests needing more
 * than that (lsa_index_workspace_bytes(nq, cache->n_blocks, p) > 16 MiB) are
 * rejected with LSA_ERR_WORKSPACE and a message saying so; nothing is
 * enqueued then.  At k = 4096 this admits up to 201 Flat queries over 1M
 * tokens; over 10M tokens it admits 1-3 or 17-201 queries (batches of 16 or
 * fewer keep every bucket score, 5 MB per query at 10M).
 *
 * The first call on a device looks up the array's device address (with that
 * device current) and keeps it.  Under CUDA's default lazy module loading the
 * array, and the code of the kernels a call launches, are set up on a device
 * the first time they are used there, so the first call on each device may
 * allocate device memory and synchronise: make one call with the sizes you
 * will use (a call with nq = 0 only sets up the array) before reserving the
 * rest of device memory and before any stream capture, or run with
 * CUDA_MODULE_LOADING=EAGER.  The kept address assumes the device is not
 * reset while the library is in use.  Parameters are checked before the size
 * (bad ones give LSA_ERR_ARG).  All calls share the one array and it keeps the previous call's
 * contents (every value the kernels read is written earlier in the same
 * call); calls whose GPU work overlaps in time -- on different streams, or
 * from several host threads -- race on it and must be serialised by the
 * caller. */
int lsa_index_decode_static(const float *qidx, const int64_t *pos, int64_t nq, const lsa_cache *cache,
                            const lsa_tree *tree, int32_t *lists, int32_t *lens, int32_t Lmax,
                            const lsa_params *p, void *stream);

/* ---- context parallelism: the token range split over ranks ----
 * The pages' end-to-end runs split the KV cache by token range over 8 GPUs
 * ([FORUM] "Reported numbers"; [BLOG] "Why 72x in one layer becomes 9x").
 * Rank s holds complete blocks [b_first_s, b_first_s + n_s) of the bucket
 * cache (a cache built from the keys of positions 512 b_first_s onwards,
 * member positions relative to that) and the K/V rows of its token range;
 * queries are replicated.  A bucket among the global top P is among the top
 * P of the rank that owns it, so each rank sends a set holding its own top P
 * (lsa_index_shard_local), the sets are all-gathered in rank order, and every
 * rank computes the same global top P and list (lsa_index_shard_merge),
 * identical to lsa_index_prefill on the whole cache (Flat, up to ties in the
 * last bit of a score at the cut).  Each rank attends over its own entries
 * (lsa_shard_local_lists, then lsa_sparse_attention with lse) and the parts
 * are combined (lsa_attention_combine).  Flat search only; 1..16 ranks.
 *
 * Exchange block of one rank for nq queries, lsa_shard_exchange_bytes(nq, p)
 * bytes, 256-byte aligned: int32 cnt[nq] padded to 256 bytes, then
 * {float score; int32 global bucket} [nq][lsa_shard_slots(p)]. */
int32_t lsa_shard_slots(const lsa_params *p);
int64_t lsa_shard_exchange_bytes(int64_t nq, const lsa_params *p);
int64_t lsa_shard_local_workspace_bytes(int64_t nq, int64_t n_blocks, const lsa_params *p);
int64_t lsa_shard_merge_workspace_bytes(int64_t nq, const lsa_params *p);

/* This rank's candidate set for each query into its exchange block `xchg`:
 * the Flat passes over `cache` (this rank's blocks, the first being global
 * block b_first; a query at position p sees the rank's blocks below p/512),
 * each query's set holding its top P local buckets with their scores, bucket
 * ids made global (+ 64 b_first).  qidx [nq, index_heads, 64] and pos [nq]
 * as lsa_index_prefill.  ws: lsa_shard_local_workspace_bytes. */
int lsa_index_shard_local(const float *qidx, const int64_t *pos, int64_t nq, const lsa_cache *cache, int64_t b_first,
                          void *xchg, const lsa_params *p, void *ws, int64_t ws_bytes, void *stream);

/* The global lists from n_shards (1..32) exchange blocks stored back to back
 * (xchg_all; one per shard, in any order -- a rank holding several chunks of
 * the context gives one block per chunk): per query the union's top P by
 * (score desc, bucket id asc), expanded as lsa_index_prefill does, over the
 * replicated member table
 * and counts of all n_blocks blocks (members [n_blocks*64, 16] global
 * positions, 16-byte aligned, count [n_blocks*64]; see
 * lsa_shard_publish_members).  Lists as lsa_index_prefill.
 * ws: lsa_shard_merge_workspace_bytes. */
int lsa_index_shard_merge(const void *xchg_all, int32_t n_shards, const int64_t *pos, int64_t nq,
                          const int32_t *members, const int32_t *count, int64_t n_blocks, int32_t *lists,
                          int32_t *lens, int32_t Lmax, const lsa_params *p, void *ws, int64_t ws_bytes, void *stream);

/* This rank's slice of the global member table: members_out [64 n, 16]
 * (n = cache->n_blocks) gets the cache's member positions moved by
 * 512 b_first (-1 pads kept), count_out [64 n] its counts.  With slices of
 * equal size and rank s's first block at s times that size, an all-gather
 * of the slices in rank order is the global table (68 bytes per bucket,
 * 8.5 bytes per token). */
int lsa_shard_publish_members(const lsa_cache *cache, int64_t b_first, int32_t *members_out, int32_t *count_out,
                              void *stream);

/* The entries of each list inside [t_begin, t_end), in order, minus t_begin
 * (this rank's K/V rows); out_lists [nq, Lmax] (entries past out_lens[i]
 * are left unwritten), out_lens [nq]. */
int lsa_shard_local_lists(const int32_t *lists, const int32_t *lens, int64_t nq, int32_t Lmax, int64_t t_begin,
                          int64_t t_end, int32_t *out_lists, int32_t *out_lens, void *stream);

/* Combine n_parts attention outputs of the same queries over disjoint key
 * sets: O_parts bf16 [n_parts, nq, Hq, 128] (each normalised over its own
 * keys), lse_parts fp32 [n_parts, nq, Hq] (-inf for no keys);
 * O = sum_s e^(lse_s - M) O_s / sum_s e^(lse_s - M), lse = M + log(sum). */
int lsa_attention_combine(const uint16_t *O_parts, const float *lse_parts, int32_t n_parts, int64_t nq, int32_t Hq,
                          int32_t head_dim, uint16_t *O, float *lse, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* LSA_H */
