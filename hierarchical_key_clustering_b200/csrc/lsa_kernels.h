// Internal launch interface between the C ABI (lsa_api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace lsa {

// Kernels enqueued since load (see lsa_launch_count in lsa.h).
void count_launches(int n);

// Per-kernel timing (lsa_kernel_timing in lsa.h): while it is on, every
// launch site brackets its kernel with two events on the launch's stream,
// tagged with the kernel's name.  kt_begin returns the record's handle (-1
// when timing is off); kt_end records the closing event.
int kt_begin(const char *name, cudaStream_t st);
void kt_end(int handle, cudaStream_t st);

struct TreeDev {
    int32_t *child;
    int32_t *parent;
    int32_t *weight;
    int32_t *min_block;
    int32_t *max_block;
    float *sum;
    float *centroid;
    uint16_t *centroid_bf16;
};

// Read-only view of the tree used by the beam search.
struct TreeView {
    const int32_t *child;
    const int32_t *parent;
    const int32_t *max_block;
    const uint16_t *centroid_bf16;
    int32_t n_levels;
    int64_t level_size[40];
    int64_t level_offset[41];
};

// Per-call index workspace (device pointers carved by the C ABI).
// Candidates are entries of up to 4 buckets: cand_g holds the first bucket
// id, cand4 the scores of buckets cand_g .. cand_g + 3; a score of -inf marks
// a bucket that is not a candidate.  The expansion keeps the scores >= tau.
struct IndexWs {
    uint16_t *qhat;     // [nq, 64] bf16 normalised queries
    int32_t *horizon;   // [nq] visible blocks
    float *tau;         // [nq] Flat threshold (-inf: keep every listed score)
    int32_t *cnt;       // [nq] candidate entries appended (may exceed cap)
    uint32_t *ghist;    // [nq, HIST_BINS] group-maximum histograms (split ranges)
    float *cand4;       // [nq, cap, 4] candidate scores
    int32_t *cand_g;    // [nq, cap] first bucket of each entry
    float *scores;      // [nq, score_stride] stored scores (small batches only)
    int64_t score_stride;
    int32_t cap;        // entries per query
};
// Histogram of group maxima used to set the Flat threshold: HIST_BINS linear
// bins over [HIST_LO, -HIST_LO] (scores of unit bf16 vectors lie inside).
constexpr int HIST_BINS = 256;
constexpr float HIST_LO = -1.0625f;
constexpr float HIST_BIN_W = 2.0f * -HIST_LO / HIST_BINS;  // 17/2048: every bin edge is an exact float
#ifdef __CUDACC__
__device__ __forceinline__ float hist_edge(int bin)
{
    return HIST_LO + (float)bin * HIST_BIN_W;
}
// Bin of a group maximum m, rounded so that its lower edge is <= m: the bin
// coordinate (m - HIST_LO) / HIST_BIN_W is computed with one fused multiply-add
// and lowered by 1e-4 of a bin, more than that multiply-add's total rounding
// error (< 4e-5 of a bin for |m| <= 1.0625), so its floor never exceeds the
// exact one.  A maximum within 1e-4 of a bin above an edge may land one bin
// low, which only lowers tau.
__device__ __forceinline__ int hist_bin(float m)
{
    const float c = fmaf(m, 1.0f / HIST_BIN_W, -HIST_LO / HIST_BIN_W - 1e-4f);
    return min(max(__float2int_rd(c), 0), HIST_BINS - 1);
}
#endif

// Batches up to this many queries take the small-batch (decode) path:
// streaming thread-per-bucket scoring on the CUDA cores, scores stored for
// the filter pass.
constexpr int SMALL_NQ = 16;

// Launch `kern` on `st`; with pdl the launch may begin before the previous
// kernel of the stream finishes (the kernel waits for it with pdl_wait before
// reading anything it wrote).  Used on the small-batch (decode) path, where a
// token's kernels are short and launch latency adds up.
template <typename... KArgs, typename... Args>
cudaError_t launch_k(bool pdl, void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                     Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = pdl ? at : nullptr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

cudaError_t launch_pool_norm(const float *keys, int64_t item_begin, int64_t item_end, float *pooled,
                             cudaStream_t st, int n_sm);
cudaError_t launch_ward(const float *pooled, int64_t blk_begin, int64_t blk_end, int cap, uint8_t *item_bucket,
                        int32_t *members, int32_t *count, float *centroid, uint16_t *centroid_bf16,
                        cudaStream_t st);
// Leaves from bucket g_first on (g_first = 0: the whole tree) and, level by
// level, the runs of 128 nodes from the first changed node on.
cudaError_t launch_tree(const float *pooled, const int32_t *members, const int32_t *count, int64_t g_first,
                        int64_t nb, const TreeDev &tr, const int64_t *level_size, const int64_t *level_offset,
                        int n_levels, cudaStream_t st, int n_sm);

struct IndexArgs {
    const float *qidx;
    const int64_t *pos;
    int64_t nq;
    int64_t n_blocks;
    const int32_t *members;
    const int32_t *count;
    const uint16_t *centroid_bf16;
    int32_t *lists;
    int32_t *lens;
    int32_t Lmax;
    int32_t k, sink, window, beam, mode;
    int32_t P;  // top buckets kept
    int32_t heads;  // index queries per token (Flat: a bucket ranks by its best head score)
    int64_t pos_shift;  // subtracted from pos for the horizon (a shard's first position; 0 otherwise)
    int32_t no_expand;  // stop after the merged candidate set (a shard's local step)
    uint32_t wait_limit;  // tries per bounded device-side wait
    uint32_t extra_tx;    // test hook (see lsa_debug_wait_test)
    int32_t sample;       // sampled threshold pass (see ScoreTcArgs; <= 1: off)
    float sample_margin;
    int64_t sample_min_n;
};

// Flat scoring on the tensor cores (lsa_score_tc.cu).  mode 0: threshold
// histogram of group maxima; mode 1: append the groups of 4 buckets whose
// best score is >= tau.
struct ScoreTcArgs {
    int64_t nq;
    int64_t nb_total;
    int32_t P;
    int32_t mode;
    int32_t whole_range;  // set by the launcher: one CTA covers each query's buckets
    int64_t chunk_tiles;
    uint32_t wait_limit;  // tries per bounded mbarrier wait
    uint32_t extra_tx;    // test hook: non-zero skips the query-tile copy, so its barrier never completes
    // threshold pass (mode 0) from a sample: a CTA whose rows all see at least
    // sample_min_n buckets, and that covers their whole range, scores only
    // every sample-th centroid tile and sets tau at the score above which
    // sample_margin x P x (sampled / visible buckets) of its sampled scores lie
    // (sample <= 1: off; the expansion redoes a query exactly if its
    // candidates then hold fewer than k far keys)
    int32_t sample;
    float sample_margin;
    int64_t sample_min_n;
};
cudaError_t launch_score_tc(const ScoreTcArgs &a, const IndexWs &ws, const uint16_t *centroid_bf16, cudaStream_t st,
                            int n_sm, int *whole_range);
int read_device_error(int clear);

// Step 1, "Shrink": x_t = W v_t for t in [t_begin, t_end), optional fp32
// keys [T, 64] and pooled items (t_begin % 4 == 0).
struct ShrinkArgs {
    int64_t t_begin, t_end, D;
    float *keys;
    float *pooled;
    uint32_t wait_limit;
};
cudaError_t launch_shrink(const uint16_t *V, const uint16_t *W, const ShrinkArgs &a, cudaStream_t st);
int read_shrink_error(int clear);
int read_bounds_error_attn(int clear);   // debug-build bounds words (lsa_common.cuh)
int read_bounds_error_index(int clear);

// ws holds one row per (query, index head); with several heads `merged`
// receives each query's merged candidates (nullptr for one head).
cudaError_t launch_index(const IndexArgs &a, const IndexWs &ws, const IndexWs *merged, const TreeView *tree,
                         cudaStream_t st, int n_sm);
cudaError_t launch_expand_merged(const IndexArgs &a, const IndexWs &m, cudaStream_t st);

// Context-parallel pieces (lsa_shard.cu).  Exchange block of one rank:
// int32 cnt[nq], then {float score, int32 global bucket} [nq][slots].
cudaError_t launch_shard_pack(const IndexWs &m, int64_t nq, int64_t g0, void *xchg, cudaStream_t st);
cudaError_t launch_shard_merge(const void *xchg_all, int n_shards, int64_t nq, int slots, int P, const IndexWs &m,
                               cudaStream_t st);
cudaError_t launch_local_lists(const int32_t *lists, const int32_t *lens, int64_t nq, int32_t Lmax, int64_t t0,
                               int64_t t1, int32_t *out_lists, int32_t *out_lens, cudaStream_t st);
cudaError_t launch_publish_members(const int32_t *members, const int32_t *count, int64_t nb, int64_t g0,
                                   int64_t pos0, int32_t *members_out, int32_t *count_out, cudaStream_t st);
cudaError_t launch_combine_parts(const uint16_t *O_parts, const float *lse_parts, int n_parts, int64_t nq, int Hq,
                                 uint16_t *O, float *lse, cudaStream_t st);

// Shared memory the expansion kernel needs for `cap` candidates over a cache
// of n_blocks blocks.
size_t rank_expand_smem_bytes(int cap, int64_t n_blocks);

struct AttnArgs {
    const uint16_t *Q, *K, *V;
    int64_t nq;
    int32_t Hq, Hkv;
    int64_t Tk;
    const int32_t *lists, *lens;
    int32_t Lmax;
    float scale;
    uint16_t *O;
    float *lse;
    float *part_o;   // [nq, Hq, nsplit, 128] (nsplit > 1 only)
    float *part_ml;  // [nq, Hq, nsplit, 2]
    int32_t nsplit;
    // near-set split (nsplit == 1 only; NULL = off): per query the sink
    // prefix and window suffix of its list taken densely, and their partial
    // results [nq, Hq, 128] / [nq, Hq, 2] (running max in log2 units, sum)
    int2 *near_plan;
    int4 *near_tile;  // per tile: {usable, first position, lowest near key, longest sink prefix}
    float *near_o;
    float *near_ml;
    // position-range phases (nsplit == 1 and no near plan; NULL = off): the
    // keys are cut into n_ranges ranges of range_rows positions, and one
    // launch per (KV head phase_g, range phase_r) runs every query's list
    // entries in that range, carrying a running result per (query, head)
    // from launch to launch, so that the K/V rows the launch gathers (one
    // head's rows of one range) stay in L2 while every query reads them
    int32_t *range_off;  // [nq, n_ranges + 1]: index of the first list entry at or past each range start
    float *state_o;      // [nq, Hq, 128] unnormalised O, relative to the running max
    float *state_ml;     // [nq, Hq, 2] running max (log2 units; -inf = nothing yet), running sum
    int32_t n_ranges;
    int64_t range_rows;
    int32_t phase_g, phase_r;
    uint32_t wait_limit;  // tries per bounded device-side wait (tensor-core near tiles)
};

// Queries per near-set tile for G query heads per KV head, 0 = no near path.
constexpr int NEAR_ROWS = 128;
__host__ __device__ inline int near_tile_queries(int G) { return (G >= 1 && NEAR_ROWS % G == 0) ? NEAR_ROWS / G : 0; }

cudaError_t launch_attention(const AttnArgs &a, cudaStream_t st, int n_sm);
cudaError_t launch_attention_near_tc(const AttnArgs &a, int tiles, cudaStream_t st);
int read_near_error(int clear);
int attention_list_cap();

}  // namespace lsa
