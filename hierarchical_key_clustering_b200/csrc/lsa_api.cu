// C ABI of the LSA hot path (see include/lsa.h for the contract of every
// entry point).  This file only checks arguments, carves caller buffers and
// enqueues the kernels of lsa_build.cu, lsa_index.cu and lsa_attn.cu on the
// caller's stream.  It never allocates device memory and never synchronises.
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <vector>

#include "lsa.h"
#include "lsa_common.cuh"
#include "lsa_kernels.h"

static_assert(LSA_MAX_INDEX_HEADS == LSA_MAXHEADS, "index head limit of the header and the kernels");

namespace {

std::atomic<int64_t> g_launches{0};
thread_local char g_err[512] = "no error";

int fail(int code, const char *fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof(g_err), fmt, ap);
    va_end(ap);
    return code;
}

int cuda_fail(cudaError_t e, const char *what)
{
    return fail(LSA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void *p)
{
    return ((uintptr_t)p & 15u) == 0;
}

int64_t align256(int64_t x)
{
    return (x + 255) & ~(int64_t)255;
}

int sm_count()
{
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 148;
}

int64_t l2_bytes()
{
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrL2CacheSize, dev);
    return n > 0 ? n : (int64_t)126 << 20;
}

int check_params(const lsa_params *p)
{
    if (!p) return fail(LSA_ERR_ARG, "params is NULL");
    if (p->n_pool != LSA_N_POOL || p->block != LSA_BLOCK || p->n_buckets != LSA_BUCKETS ||
        p->cap_items != LSA_N_POOL)
        return fail(LSA_ERR_ARG,
                    "only n_pool=4, block=512, n_buckets=64, cap_items=4 are built (got %d, %d, %d, %d)",
                    p->n_pool, p->block, p->n_buckets, p->cap_items);
    if (p->sink < 0 || p->window < 0 || p->k < 0) return fail(LSA_ERR_ARG, "sink, window and k must be >= 0");
    if (p->k > (1 << 20)) return fail(LSA_ERR_ARG, "k = %d is above the supported 1048576", p->k);
    if (p->mode != LSA_MODE_FLAT && p->mode != LSA_MODE_TREE) return fail(LSA_ERR_ARG, "mode must be 0 or 1");
    if (p->mode == LSA_MODE_TREE && p->beam < 1) return fail(LSA_ERR_ARG, "beam must be >= 1");
    if (p->index_heads < 1 || p->index_heads > LSA_MAX_INDEX_HEADS)
        return fail(LSA_ERR_ARG, "index_heads = %d must be in 1..%d", p->index_heads, LSA_MAX_INDEX_HEADS);
    if (p->mode == LSA_MODE_TREE && p->index_heads != 1)
        return fail(LSA_ERR_ARG, "Tree search takes one index head (index_heads = %d)", p->index_heads);
    return LSA_OK;
}

int64_t top_buckets(const lsa_params *p)
{
    return ((int64_t)p->k + p->sink + p->window + LSA_N_POOL - 1) / LSA_N_POOL;
}

int64_t cand_cap(const lsa_params *p)
{
    const int64_t P = top_buckets(p);
    int64_t cap = p->cand_cap > 0 ? p->cand_cap : lsa::pow2_ceil64(2 * P);
    if (p->mode == LSA_MODE_TREE) {
        int64_t need = p->beam > P ? p->beam : P;
        if (cap < need) cap = need;
    }
    return cap;
}

struct CacheLayout {
    int64_t off[6];
    int64_t bytes;
};

CacheLayout cache_layout(int64_t capacity)
{
    const int64_t items = capacity / LSA_N_POOL, nblk = capacity / LSA_BLOCK, nb = nblk * LSA_BUCKETS;
    const int64_t sz[6] = {items * LSA_DIM * 4, nblk * LSA_ITEMS, nb * LSA_SLOTS * 4, nb * 4, nb * LSA_DIM * 4,
                           nb * LSA_DIM * 2};
    CacheLayout L;
    int64_t o = 0;
    for (int i = 0; i < 6; ++i) {
        L.off[i] = o;
        o += align256(sz[i]);
    }
    L.bytes = o;
    return L;
}

int tree_levels(int64_t nb, int64_t *size, int64_t *offset)
{
    int L = 0;
    int64_t n = nb, o = 0;
    while (L < LSA_MAX_LEVELS) {
        size[L] = n;
        offset[L] = o;
        o += n;
        ++L;
        if (n <= 1) break;
        n = (n + 1) / 2;
    }
    offset[L] = o;
    return L;
}

struct TreeLayout {
    int64_t off[8];
    int64_t bytes;
    int64_t nodes;
};

TreeLayout tree_layout(int64_t nblk)
{
    int64_t size[LSA_MAX_LEVELS + 1], offset[LSA_MAX_LEVELS + 2];
    int L = tree_levels(nblk * LSA_BUCKETS, size, offset);
    const int64_t n = offset[L];
    const int64_t sz[8] = {n * 2 * 4, n * 4, n * 4, n * 4, n * 4, n * LSA_DIM * 4, n * LSA_DIM * 4, n * LSA_DIM * 2};
    TreeLayout T;
    int64_t o = 0;
    for (int i = 0; i < 8; ++i) {
        T.off[i] = o;
        o += align256(sz[i]);
    }
    T.bytes = o;
    T.nodes = n;
    return T;
}

// Entries the expansion kernel holds in shared memory per query: the filter
// keeps about 1.2-1.45 P candidates on the measured workloads; a query with
// more takes the exact path.
int64_t expand_slots(int64_t cap, int64_t P)
{
    const int64_t kc = lsa::pow2_ceil64((P * 3 + 1) / 2);
    return cap < kc ? cap : kc;
}

// The scorer's arrays are per row, a row being one (query, index head); with
// several index heads the merged candidates of each query follow (one bucket
// per entry, expand_slots entries per query).
struct IndexLayout {
    int64_t off[13];
    int64_t bytes;
    int64_t gstride;
    int64_t sstride;
    int64_t cap;
    int64_t mcap;
};

IndexLayout index_layout(int64_t nq, int64_t nblk, const lsa_params *p, bool shard_local = false)
{
    const int64_t N = nblk * LSA_BUCKETS;
    const int64_t heads = p->index_heads > 1 ? p->index_heads : 1;
    const int64_t rows = nq * heads;
    const bool merged = heads > 1 || shard_local;
    IndexLayout L;
    L.gstride = lsa::HIST_BINS;  // group-maximum histogram per row
    L.cap = cand_cap(p);
    L.mcap = merged ? expand_slots(L.cap, top_buckets(p)) : 0;
    const int64_t mq = merged ? nq : 0;
    // small batches (decode) keep every score for the filter pass
    L.sstride = (rows <= lsa::SMALL_NQ && p->mode == LSA_MODE_FLAT) ? N : 0;
    const int64_t sz[13] = {rows * LSA_DIM * 2, rows * 4,        rows * 4, rows * 4, rows * L.gstride * 4,
                            rows * L.cap * 16,  rows * L.cap * 4, rows * L.sstride * 4,
                            mq * 4,             mq * 4,          mq * 4,   mq * L.mcap * 16, mq * L.mcap * 4};
    int64_t o = 0;
    for (int i = 0; i < 13; ++i) {
        L.off[i] = o;
        o += align256(sz[i]);
    }
    L.bytes = o;
    return L;
}

// Bounded device-side waits: tries per wait, and the test hook that makes one
// wait run out (lsa_debug_wait_test).
uint32_t g_wait_limit = 1u << 20;
uint32_t g_extra_tx = 0;
// Sampled threshold pass of Flat search (lsa_debug_score_sample): every 16th
// centroid tile, tau set so that about 0.9 P buckets lie above it, for
// queries that see at least 16 x 128 x 32 buckets.
int32_t g_sample = 16;
float g_sample_margin = 0.9f;
constexpr int64_t SAMPLE_MIN_TILES = 32;

// Key splits per query for small batches (one warp per (query, KV head,
// split)), at least 32 keys per split.
int attention_nsplit(int64_t nq, int32_t Hkv, int32_t Lmax)
{
    // few queries: split each list so that about 512 warps run (measured at
    // 1M decode: 512 -> 57.5 us/token, 1024 -> 58.5, 2048 -> 60.5, 256 -> 59.5;
    // more splits cost more in the merge than they save in the gather)
    const int64_t units = nq * (int64_t)Hkv;
    if (units >= 2048) return 1;
    int64_t s = (512 + units - 1) / units;
    const int64_t chunks = (Lmax + 31) / 32;
    if (s > chunks) s = chunks;
    if (s > 1024) s = 1024;  // the merge kernel holds at most 1024 split weights
    return (int)(s < 1 ? 1 : s);
}



int64_t attention_ws_bytes(int64_t nq, int32_t Hq, int32_t nsplit)
{
    if (nsplit <= 1) return 0;
    return align256(nq * Hq * (int64_t)nsplit * LSA_HEAD_DIM * 4) + align256(nq * Hq * (int64_t)nsplit * 2 * 4);
}

// Batches of at least this many queries take the near-set path (a tile of
// consecutive queries shares its sink and window rows); its workspace holds
// one partial result per (query, head) and one plan per query.
constexpr int64_t NEAR_MIN_NQ = 64;
int64_t near_ws_bytes(int64_t nq, int32_t Hq)
{
    if (nq < NEAR_MIN_NQ) return 0;
    // tiles hold at least one query: nq tile records bound every tile count
    return align256(nq * Hq * (int64_t)LSA_HEAD_DIM * 4) + align256(nq * Hq * (int64_t)2 * 4) + align256(nq * 8) +
           align256(nq * 16);
}

// Position-range phases of the gather (AttnArgs::state_o): for batches of at
// least PHASE_MIN_NQ queries whose KV head's K + V rows (Tk x 512 B) exceed
// three quarters of L2.  A range holds about half of L2 of one head's rows,
// so the rows a launch gathers stay in L2 while every query reads them; the
// workspace holds the range bounds of every query and one running result
// per (query, head).  Each (query, range) costs a few dependent memory round
// trips before its rows stream, so the phases pay only while a list holds
// enough entries per range: measured on the 4613-entry lists of the 1M and
// 10M workloads, 8 ranges per head (~580 entries each) took 49.5 ms against
// 66.0 for the plain gather, 77 ranges (~60 each) 185 against 155.
constexpr int64_t PHASE_MIN_NQ = 512;
constexpr int64_t PHASE_MIN_ROWS = 256;  // list budget per range
int64_t g_phase_rows = 0;  // test hook (lsa_debug_attention_ranges): > 0 forced range size, < 0 never, 0 automatic
int64_t phase_ranges(int64_t Tk)
{
    const int64_t rows = g_phase_rows > 0 ? g_phase_rows : (l2_bytes() / 2) / (2 * LSA_HEAD_DIM * 2);
    return (Tk + rows - 1) / rows;
}
bool phases_pay(int64_t nq, int64_t Tk, int32_t Lmax)
{
    if (g_phase_rows < 0) return false;
    if (g_phase_rows > 0) return nq >= 1 && Tk >= 1;
    return nq >= PHASE_MIN_NQ && Tk * 2 * LSA_HEAD_DIM * 2 > l2_bytes() * 3 / 4 &&
           (int64_t)Lmax >= PHASE_MIN_ROWS * phase_ranges(Tk);
}
int64_t phase_ws_bytes(int64_t nq, int32_t Hq, int64_t Tk, int32_t Lmax)
{
    if (!phases_pay(nq, Tk, Lmax)) return 0;
    return align256(nq * (phase_ranges(Tk) + 1) * 4) + align256(nq * Hq * (int64_t)LSA_HEAD_DIM * 4) +
           align256(nq * Hq * (int64_t)2 * 4);
}

// A shard's local step (lsa_index_shard_local): positions shifted to the
// shard's first token, the merged candidate set packed into `xchg` with
// global bucket ids instead of an expansion.
struct ShardLocal {
    int64_t b_first;
    void *xchg;
};

int index_impl(const float *qidx, const int64_t *pos, int64_t nq, const lsa_cache *cache, const lsa_tree *tree,
               int32_t *lists, int32_t *lens, int32_t Lmax, const lsa_params *p, void *ws, int64_t ws_bytes,
               void *stream, const ShardLocal *sl = nullptr)
{
    int rc = check_params(p);
    if (rc) return rc;
    if (nq < 0) return fail(LSA_ERR_SHAPE, "nq < 0");
    if (!cache) return fail(LSA_ERR_ARG, "cache is NULL");
    if (nq == 0) return LSA_OK;
    if (sl) {
        if (!qidx || !pos || !sl->xchg) return fail(LSA_ERR_ARG, "qidx, pos and xchg must be non-NULL");
        if (!aligned16(qidx) || ((uintptr_t)sl->xchg & 255u)) return fail(LSA_ERR_ARG, "qidx must be 16-byte and xchg 256-byte aligned");
        if (p->mode != LSA_MODE_FLAT) return fail(LSA_ERR_ARG, "context-parallel search is Flat only");
        if (sl->b_first < 0) return fail(LSA_ERR_SHAPE, "b_first < 0");
    } else {
        if (!qidx || !pos || !lists || !lens) return fail(LSA_ERR_ARG, "qidx, pos, lists and lens must be non-NULL");
        if (!aligned16(qidx) || !aligned16(lists)) return fail(LSA_ERR_ARG, "qidx and lists must be 16-byte aligned");
        if (Lmax < lsa_list_budget(p))
            return fail(LSA_ERR_SHAPE, "Lmax %d < list budget %d", Lmax, lsa_list_budget(p));
    }
    if (cache->n_blocks < 0 || cache->n_blocks * LSA_BLOCK > cache->capacity)
        return fail(LSA_ERR_SHAPE, "cache n_blocks %lld out of range", (long long)cache->n_blocks);
    if (cache->n_blocks > 0 && (!cache->members || !cache->count || !cache->centroid_bf16))
        return fail(LSA_ERR_ARG, "cache arrays are NULL");
    if (p->mode == LSA_MODE_TREE) {
        if (!tree) return fail(LSA_ERR_ARG, "Tree mode needs a tree");
        if (cache->n_blocks > 0 && tree->n_blocks != cache->n_blocks)
            return fail(LSA_ERR_SHAPE, "tree covers %lld blocks, cache has %lld", (long long)tree->n_blocks,
                        (long long)cache->n_blocks);
        const int64_t P = top_buckets(p);
        const int64_t B1 = ((P + 1) / 2) > p->beam ? (P + 1) / 2 : p->beam;
        if (2 * B1 + LSA_ITEMS + 2 > 8192)
            return fail(LSA_ERR_ARG, "beam %d / k %d too large for the beam kernel", p->beam, p->k);
    }
    const int64_t P = top_buckets(p);
    // Flat threshold histograms count at most 2^16 - 1 group maxima per query
    // (groups of up to 64 buckets, 4P..8P of them)
    if (p->mode == LSA_MODE_FLAT && (cache->n_blocks > 65535 || P >= 8192))
        return fail(LSA_ERR_SHAPE, "Flat search supports up to 65535 blocks and k + sink + window < 32768");
    IndexLayout L = index_layout(nq, cache->n_blocks, p, sl != nullptr);
    if (L.cap < P) return fail(LSA_ERR_ARG, "cand_cap %lld < top buckets %lld", (long long)L.cap, (long long)P);
    if (L.cap > 8192) return fail(LSA_ERR_ARG, "cand_cap %lld above 8192", (long long)L.cap);
    if (lsa::rank_expand_smem_bytes((int)L.cap, cache->n_blocks) > 227 * 1024)
        return fail(LSA_ERR_ARG, "cand_cap %lld / %lld blocks too large for the expansion kernel", (long long)L.cap,
                    (long long)cache->n_blocks);
    if (!ws || ws_bytes < L.bytes)
        return fail(LSA_ERR_WORKSPACE, "index workspace %lld bytes < %lld", (long long)ws_bytes, (long long)L.bytes);
    if (((uintptr_t)ws & 255u) != 0) return fail(LSA_ERR_ARG, "workspace must be 256-byte aligned");
    char *w = (char *)ws;
    lsa::IndexWs iw;
    iw.qhat = (uint16_t *)(w + L.off[0]);
    iw.horizon = (int32_t *)(w + L.off[1]);
    iw.tau = (float *)(w + L.off[2]);
    iw.cnt = (int32_t *)(w + L.off[3]);
    iw.ghist = (uint32_t *)(w + L.off[4]);
    iw.cand4 = (float *)(w + L.off[5]);
    iw.cand_g = (int32_t *)(w + L.off[6]);
    iw.scores = L.sstride ? (float *)(w + L.off[7]) : nullptr;
    iw.score_stride = L.sstride;
    iw.cap = (int32_t)L.cap;
    lsa::IndexWs mw = iw;  // merged candidates of multi-head queries or of a shard
    const bool merged = p->index_heads > 1 || sl;
    if (merged) {
        mw.horizon = (int32_t *)(w + L.off[8]);
        mw.tau = (float *)(w + L.off[9]);
        mw.cnt = (int32_t *)(w + L.off[10]);
        mw.cand4 = (float *)(w + L.off[11]);
        mw.cand_g = (int32_t *)(w + L.off[12]);
        mw.ghist = nullptr;
        mw.scores = nullptr;
        mw.score_stride = 0;
        mw.cap = (int32_t)L.mcap;
    }
    lsa::IndexArgs a;
    a.qidx = qidx;
    a.pos = pos;
    a.nq = nq;
    a.n_blocks = cache->n_blocks;
    a.members = cache->members;
    a.count = cache->count;
    a.centroid_bf16 = cache->centroid_bf16;
    a.lists = lists;
    a.lens = lens;
    a.Lmax = Lmax;
    a.k = p->k;
    a.sink = p->sink;
    a.window = p->window;
    a.beam = p->beam;
    a.mode = p->mode;
    a.P = (int32_t)P;
    a.heads = p->index_heads;
    a.pos_shift = sl ? sl->b_first * LSA_BLOCK : 0;
    a.no_expand = sl ? 1 : 0;
    a.wait_limit = g_wait_limit;
    a.extra_tx = g_extra_tx;
    g_extra_tx = 0;
    a.sample = g_sample;
    a.sample_margin = g_sample_margin;
    a.sample_min_n = (int64_t)(g_sample > 1 ? g_sample : 1) * 128 * SAMPLE_MIN_TILES;
    lsa::TreeView tv;
    const lsa::TreeView *tvp = nullptr;
    if (p->mode == LSA_MODE_TREE && cache->n_blocks > 0) {
        tv.child = tree->child;
        tv.parent = tree->parent;
        tv.max_block = tree->max_block;
        tv.centroid_bf16 = tree->centroid_bf16;
        tv.n_levels = tree->n_levels;
        for (int l = 0; l < 40; ++l) tv.level_size[l] = tree->level_size[l];
        for (int l = 0; l < 41; ++l) tv.level_offset[l] = tree->level_offset[l];
        tvp = &tv;
    }
    cudaError_t e = lsa::launch_index(a, iw, merged ? &mw : nullptr, tvp, (cudaStream_t)stream, sm_count());
    if (e != cudaSuccess) return cuda_fail(e, "index launch");
    if (sl) {
        e = lsa::launch_shard_pack(mw, nq, sl->b_first * LSA_BUCKETS, sl->xchg, (cudaStream_t)stream);
        if (e != cudaSuccess) return cuda_fail(e, "shard pack launch");
    }
    return LSA_OK;
}

}  // namespace

namespace lsa {
void count_launches(int n)
{
    g_launches.fetch_add(n, std::memory_order_relaxed);
}

// Per-kernel timing: one record (name, start event, end event) per launch
// while timing is on; events come from a pool and go back to it on read.
namespace {
struct KtRec {
    const char *name;
    cudaEvent_t a, b;
    bool ended;
};
bool g_kt_on = false;
std::vector<KtRec> g_kt;
std::vector<cudaEvent_t> g_kt_pool;

cudaEvent_t kt_event()
{
    cudaEvent_t e = nullptr;
    if (!g_kt_pool.empty()) {
        e = g_kt_pool.back();
        g_kt_pool.pop_back();
    } else if (cudaEventCreate(&e) != cudaSuccess) {
        e = nullptr;
    }
    return e;
}
}  // namespace

int kt_begin(const char *name, cudaStream_t st)
{
    if (!g_kt_on) return -1;
    cudaEvent_t a = kt_event(), b = kt_event();
    if (!a || !b || cudaEventRecord(a, st) != cudaSuccess) {
        if (a) g_kt_pool.push_back(a);
        if (b) g_kt_pool.push_back(b);
        return -1;
    }
    g_kt.push_back(KtRec{name, a, b, false});
    return (int)g_kt.size() - 1;
}

void kt_end(int handle, cudaStream_t st)
{
    if (handle < 0 || handle >= (int)g_kt.size()) return;
    g_kt[handle].ended = cudaEventRecord(g_kt[handle].b, st) == cudaSuccess;
}

int report_error(int code, const char *msg)
{
    return fail(code, "%s", msg);
}

int check_index_params(const lsa_params *p)
{
    return check_params(p);
}
}  // namespace lsa

extern "C" {

int64_t lsa_launch_count(void)
{
    return g_launches.load(std::memory_order_relaxed);
}

int lsa_check_device_errors(void)
{
    int v = lsa::read_device_error(1);
    if (v < 0) return fail(LSA_ERR_CUDA, "could not read the device error word");
    if (v & 1) fail(LSA_ERR_TIMEOUT, "a bounded device-side wait ran out");
    else if (v) fail(LSA_ERR_SHAPE, "a bounds check of the debug build failed (code %d)", v);
    return v;
}

void lsa_kernel_timing(int32_t enable)
{
    lsa::g_kt_on = enable != 0;
}

int lsa_kernel_timing_read(char *names, int32_t name_len, double *ms, int64_t *launches, int32_t max_kernels)
{
    int n = 0;
    cudaError_t err = cudaSuccess;
    std::vector<const char *> seen;
    for (auto &r : lsa::g_kt) {
        float x = 0.0f;
        cudaError_t e = r.ended ? cudaEventSynchronize(r.b) : cudaErrorNotReady;
        if (e == cudaSuccess) e = cudaEventElapsedTime(&x, r.a, r.b);
        if (e != cudaSuccess && r.ended) err = e;
        lsa::g_kt_pool.push_back(r.a);
        lsa::g_kt_pool.push_back(r.b);
        if (e != cudaSuccess) continue;
        int i = 0;
        while (i < (int)seen.size() && strcmp(seen[i], r.name) != 0) ++i;
        if (i == (int)seen.size()) {
            seen.push_back(r.name);
            if (i < max_kernels) {
                if (names && name_len > 0) snprintf(names + (int64_t)i * name_len, (size_t)name_len, "%s", r.name);
                if (ms) ms[i] = 0.0;
                if (launches) launches[i] = 0;
            }
        }
        if (i < max_kernels) {
            if (ms) ms[i] += x;
            if (launches) launches[i] += 1;
        }
    }
    lsa::g_kt.clear();
    n = (int)seen.size();
    if (err != cudaSuccess) return cuda_fail(err, "kernel timing events");
    return n;
}

void lsa_debug_score_sample(int32_t stride, float margin)
{
    g_sample = stride;
    g_sample_margin = margin > 0.0f ? margin : 0.9f;
}

void lsa_debug_attention_ranges(int64_t range_rows)
{
    g_phase_rows = range_rows;
}

void lsa_debug_wait_test(int32_t enable)
{
    g_extra_tx = enable ? 16u : 0u;
    g_wait_limit = enable ? 1024u : (1u << 20);
}

void lsa_default_params(lsa_params *p)
{
    if (!p) return;
    p->n_pool = LSA_N_POOL;
    p->block = LSA_BLOCK;
    p->n_buckets = LSA_BUCKETS;
    p->cap_items = LSA_N_POOL;
    p->sink = 4;
    p->window = 512;
    p->k = 4096;
    p->beam = 32;
    p->mode = LSA_MODE_FLAT;
    p->cand_cap = 0;
    p->index_heads = 1;
}

const char *lsa_last_error_string(void)
{
    return g_err;
}

int32_t lsa_list_budget(const lsa_params *p)
{
    return p ? p->k + p->sink + p->window + 1 : -1;
}

int32_t lsa_top_buckets(const lsa_params *p)
{
    return p ? (int32_t)top_buckets(p) : -1;
}

int64_t lsa_cache_bytes(int64_t capacity)
{
    if (capacity < 0) return -1;
    return cache_layout(capacity).bytes;
}

int lsa_cache_bind(void *base, int64_t bytes, int64_t capacity, lsa_cache *out)
{
    if (!out) return fail(LSA_ERR_ARG, "out is NULL");
    if (capacity < 0) return fail(LSA_ERR_SHAPE, "capacity < 0");
    CacheLayout L = cache_layout(capacity);
    if (!base || ((uintptr_t)base & 255u)) return fail(LSA_ERR_ARG, "cache buffer must be non-NULL and 256-byte aligned");
    if (bytes < L.bytes) return fail(LSA_ERR_SHAPE, "cache buffer %lld bytes < %lld", (long long)bytes, (long long)L.bytes);
    char *b = (char *)base;
    out->capacity = capacity;
    out->n_blocks = 0;
    out->pooled = (float *)(b + L.off[0]);
    out->item_bucket = (uint8_t *)(b + L.off[1]);
    out->members = (int32_t *)(b + L.off[2]);
    out->count = (int32_t *)(b + L.off[3]);
    out->centroid = (float *)(b + L.off[4]);
    out->centroid_bf16 = (uint16_t *)(b + L.off[5]);
    return LSA_OK;
}

int64_t lsa_tree_bytes(int64_t n_blocks)
{
    if (n_blocks < 0) return -1;
    return tree_layout(n_blocks).bytes;
}

int lsa_tree_bind(void *base, int64_t bytes, int64_t n_blocks, lsa_tree *out)
{
    if (!out) return fail(LSA_ERR_ARG, "out is NULL");
    if (n_blocks < 1) return fail(LSA_ERR_SHAPE, "a tree needs at least one block");
    TreeLayout T = tree_layout(n_blocks);
    if (!base || ((uintptr_t)base & 255u)) return fail(LSA_ERR_ARG, "tree buffer must be non-NULL and 256-byte aligned");
    if (bytes < T.bytes) return fail(LSA_ERR_SHAPE, "tree buffer %lld bytes < %lld", (long long)bytes, (long long)T.bytes);
    memset(out, 0, sizeof(*out));
    int64_t size[LSA_MAX_LEVELS + 1], offset[LSA_MAX_LEVELS + 2];
    int L = tree_levels(n_blocks * LSA_BUCKETS, size, offset);
    out->n_blocks = 0;
    out->cap_blocks = (int32_t)n_blocks;
    out->n_levels = L;
    for (int l = 0; l < L; ++l) {
        out->level_size[l] = size[l];
        out->level_offset[l] = offset[l];
    }
    out->level_offset[L] = offset[L];
    char *b = (char *)base;
    out->child = (int32_t *)(b + T.off[0]);
    out->parent = (int32_t *)(b + T.off[1]);
    out->weight = (int32_t *)(b + T.off[2]);
    out->min_block = (int32_t *)(b + T.off[3]);
    out->max_block = (int32_t *)(b + T.off[4]);
    out->sum = (float *)(b + T.off[5]);
    out->centroid = (float *)(b + T.off[6]);
    out->centroid_bf16 = (uint16_t *)(b + T.off[7]);
    return LSA_OK;
}

int64_t lsa_index_workspace_bytes(int64_t nq, int64_t n_blocks, const lsa_params *p)
{
    if (!p || nq < 0 || n_blocks < 0) return -1;
    return index_layout(nq, n_blocks, p).bytes;
}

int64_t lsa_attention_workspace_bytes(int64_t nq, int32_t Hq, int32_t head_dim, int32_t Lmax, int64_t Tk)
{
    if (nq < 0 || Hq < 1 || head_dim != LSA_HEAD_DIM || Lmax < 1 || Tk < 0) return -1;
    const int64_t split = attention_ws_bytes(nq, Hq, attention_nsplit(nq, 1, Lmax));
    const int64_t near = near_ws_bytes(nq, Hq);
    const int64_t phase = phase_ws_bytes(nq, Hq, Tk, Lmax);
    const int64_t m = split > near ? split : near;
    return m > phase ? m : phase;
}

int lsa_build_cache(const float *keys, int64_t t_begin, int64_t t_end, lsa_cache *cache, const lsa_params *p,
                    void *stream)
{
    int rc = check_params(p);
    if (rc) return rc;
    if (!cache) return fail(LSA_ERR_ARG, "cache is NULL");
    if (t_begin < 0 || t_end < t_begin) return fail(LSA_ERR_SHAPE, "need 0 <= t_begin <= t_end");
    if (t_end > cache->capacity)
        return fail(LSA_ERR_SHAPE, "t_end %lld > cache capacity %lld", (long long)t_end, (long long)cache->capacity);
    const int64_t i0 = t_begin / LSA_N_POOL, i1 = t_end / LSA_N_POOL;
    const int64_t b0 = t_begin / LSA_BLOCK, b1 = t_end / LSA_BLOCK;
    if (i1 > i0 || b1 > b0) {
        if (keys && !aligned16(keys)) return fail(LSA_ERR_ARG, "keys must be 16-byte aligned");
        if (!cache->pooled || !cache->item_bucket || !cache->members || !cache->count || !cache->centroid ||
            !cache->centroid_bf16)
            return fail(LSA_ERR_ARG, "cache arrays are NULL (bind the cache first)");
    }
    cudaStream_t st = (cudaStream_t)stream;
    cudaError_t e = keys ? lsa::launch_pool_norm(keys, i0, i1, cache->pooled, st, sm_count()) : cudaSuccess;
    if (e != cudaSuccess) return cuda_fail(e, "pool launch");
    e = lsa::launch_ward(cache->pooled, b0, b1, p->cap_items, cache->item_bucket, cache->members, cache->count,
                         cache->centroid, cache->centroid_bf16, st);
    if (e != cudaSuccess) return cuda_fail(e, "ward launch");
    if (b1 > cache->n_blocks) cache->n_blocks = b1;
    return LSA_OK;
}

// Shared by lsa_build_tree and lsa_update_tree: the tree's level sizes for
// the cache's blocks, its offsets fixed by the capacity it was bound for, and
// the launches for the leaves from block b_first on and the runs above them.
static int tree_grow(const lsa_cache *cache, lsa_tree *tree, const lsa_params *p, int64_t b_first, void *stream)
{
    int rc = check_params(p);
    if (rc) return rc;
    if (!cache || !tree) return fail(LSA_ERR_ARG, "cache and tree must be non-NULL");
    if (cache->n_blocks < 1) return fail(LSA_ERR_SHAPE, "the cache has no complete block");
    if (!tree->child || !tree->sum || tree->cap_blocks < 1)
        return fail(LSA_ERR_ARG, "tree is not bound (lsa_tree_bind)");
    if (cache->n_blocks > tree->cap_blocks)
        return fail(LSA_ERR_SHAPE, "tree bound for %d blocks, the cache holds %lld", tree->cap_blocks,
                    (long long)cache->n_blocks);
    int64_t size[LSA_MAX_LEVELS + 1], offset[LSA_MAX_LEVELS + 2];
    int64_t csize[LSA_MAX_LEVELS + 1], coff[LSA_MAX_LEVELS + 2];
    const int L = tree_levels(cache->n_blocks * LSA_BUCKETS, size, offset);
    const int LC = tree_levels((int64_t)tree->cap_blocks * LSA_BUCKETS, csize, coff);
    if (L > LC) return fail(LSA_ERR_SHAPE, "tree levels exceed its capacity");
    tree->n_levels = L;
    for (int l = 0; l < LSA_MAX_LEVELS; ++l) tree->level_size[l] = l < L ? size[l] : 0;
    for (int l = 0; l <= LSA_MAX_LEVELS; ++l) tree->level_offset[l] = l <= LC ? coff[l] : coff[LC];
    lsa::TreeDev td{tree->child, tree->parent, tree->weight, tree->min_block, tree->max_block,
                    tree->sum, tree->centroid, tree->centroid_bf16};
    cudaError_t e = lsa::launch_tree(cache->pooled, cache->members, cache->count, b_first * LSA_BUCKETS, size[0], td,
                                     size, tree->level_offset, L, (cudaStream_t)stream, sm_count());
    if (e != cudaSuccess) return cuda_fail(e, "tree launch");
    tree->n_blocks = cache->n_blocks;
    return LSA_OK;
}

int lsa_shrink(const uint16_t *V, int64_t D, const uint16_t *W, int64_t t_begin, int64_t t_end, float *keys,
               float *pooled, void *stream)
{
    if (!V || !W) return fail(LSA_ERR_ARG, "V and W must be non-NULL");
    if (!keys && !pooled) return fail(LSA_ERR_ARG, "keys and pooled are both NULL");
    if (D < 64 || D % 64 != 0 || D > 16384) return fail(LSA_ERR_SHAPE, "D = %lld must be a multiple of 64 <= 16384",
                                                        (long long)D);
    if (t_begin < 0 || t_end < t_begin) return fail(LSA_ERR_SHAPE, "need 0 <= t_begin <= t_end");
    if (pooled && t_begin % LSA_N_POOL != 0) return fail(LSA_ERR_SHAPE, "pooled output needs t_begin %% 4 == 0");
    if (!aligned16(V) || !aligned16(W) || (keys && !aligned16(keys)) || (pooled && !aligned16(pooled)))
        return fail(LSA_ERR_ARG, "V, W, keys and pooled must be 16-byte aligned");
    if (t_end == t_begin) return LSA_OK;
    lsa::ShrinkArgs a;
    a.t_begin = t_begin;
    a.t_end = t_end;
    a.D = D;
    a.keys = keys;
    a.pooled = pooled;
    a.wait_limit = g_wait_limit;
    cudaError_t e = lsa::launch_shrink(V, W, a, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "shrink launch");
    return LSA_OK;
}

int lsa_build_tree(const lsa_cache *cache, lsa_tree *tree, const lsa_params *p, void *stream)
{
    return tree_grow(cache, tree, p, 0, stream);
}

int lsa_update_tree(const lsa_cache *cache, lsa_tree *tree, const lsa_params *p, void *stream)
{
    if (!cache || !tree) return fail(LSA_ERR_ARG, "cache and tree must be non-NULL");
    if (cache->n_blocks < tree->n_blocks)
        return fail(LSA_ERR_SHAPE, "the cache holds %lld blocks, fewer than the tree's %lld",
                    (long long)cache->n_blocks, (long long)tree->n_blocks);
    if (tree->n_blocks > 0 && cache->n_blocks == tree->n_blocks) return check_params(p);
    return tree_grow(cache, tree, p, tree->n_blocks, stream);
}

int lsa_index_prefill(const float *qidx, const int64_t *pos, int64_t nq, const lsa_cache *cache,
                      const lsa_tree *tree, int32_t *lists, int32_t *lens, int32_t Lmax, const lsa_params *p,
                      void *ws, int64_t ws_bytes, void *stream)
{
    return index_impl(qidx, pos, nq, cache, tree, lists, lens, Lmax, p, ws, ws_bytes, stream);
}

int lsa_index_decode(const float *qidx, const int64_t *pos, int64_t nq, const lsa_cache *cache,
                     const lsa_tree *tree, int32_t *lists, int32_t *lens, int32_t Lmax, const lsa_params *p,
                     void *ws, int64_t ws_bytes, void *stream)
{
    return index_impl(qidx, pos, nq, cache, tree, lists, lens, Lmax, p, ws, ws_bytes, stream);
}

int lsa_sparse_attention(const uint16_t *Q, const uint16_t *K, const uint16_t *V, int64_t nq, int32_t Hq,
                         int32_t Hkv, int32_t head_dim, int64_t Tk, const int32_t *lists, const int32_t *lens,
                         int32_t Lmax, float scale, uint16_t *O, float *lse, void *ws, int64_t ws_bytes,
                         void *stream)
{
    if (nq < 0) return fail(LSA_ERR_SHAPE, "nq < 0");
    if (nq == 0) return LSA_OK;
    if (head_dim != LSA_HEAD_DIM) return fail(LSA_ERR_ARG, "head_dim must be %d", LSA_HEAD_DIM);
    if (Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || Hq / Hkv > 16)
        return fail(LSA_ERR_ARG, "need Hq a multiple of Hkv with Hq/Hkv <= 16 (Hq=%d Hkv=%d)", Hq, Hkv);
    if (Tk < 1 || Lmax < 1) return fail(LSA_ERR_SHAPE, "Tk and Lmax must be >= 1");
    if (!Q || !K || !V || !lists || !lens || !O) return fail(LSA_ERR_ARG, "tensor pointers must be non-NULL");
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O))
        return fail(LSA_ERR_ARG, "Q, K, V and O must be 16-byte aligned");
    if (!(scale > 0.0f)) return fail(LSA_ERR_ARG, "scale must be > 0");
    int nsplit = attention_nsplit(nq, Hkv, Lmax);
    while (nsplit > 1 && (!ws || ws_bytes < attention_ws_bytes(nq, Hq, nsplit))) nsplit >>= 1;
    lsa::AttnArgs a;
    a.Q = Q;
    a.K = K;
    a.V = V;
    a.nq = nq;
    a.Hq = Hq;
    a.Hkv = Hkv;
    a.Tk = Tk;
    a.lists = lists;
    a.lens = lens;
    a.Lmax = Lmax;
    a.scale = scale;
    a.O = O;
    a.lse = lse;
    a.nsplit = nsplit;
    a.part_o = nullptr;
    a.part_ml = nullptr;
    a.near_plan = nullptr;
    a.near_tile = nullptr;
    a.near_o = nullptr;
    a.near_ml = nullptr;
    a.range_off = nullptr;
    a.state_o = nullptr;
    a.state_ml = nullptr;
    a.wait_limit = g_wait_limit;
    a.n_ranges = 0;
    a.range_rows = 0;
    a.phase_g = a.phase_r = 0;
    // The near-set tiles pay where the gather is bound by L2 throughput: when
    // one KV head's K + V (Tk x 512 B) stays in L2 while its queries run, the
    // window rows that every query re-reads cost as much as its far rows.
    // Past that the gather is bound by HBM, where the re-read window rows are
    // L2 hits that cost little, and the tiles would only add their own time.
    const int64_t nb = near_ws_bytes(nq, Hq);
    const int64_t pb = phase_ws_bytes(nq, Hq, Tk, Lmax);
    const bool phased = nsplit == 1 && pb > 0 && ws && ws_bytes >= pb && ((uintptr_t)ws & 255u) == 0;
    const bool near_pays = Tk * 2 * LSA_HEAD_DIM * 2 <= l2_bytes() * 3 / 4;
    if (!phased && nsplit == 1 && nb > 0 && near_pays && lsa::near_tile_queries(Hq / Hkv) > 0 && ws && ws_bytes >= nb &&
        ((uintptr_t)ws & 255u) == 0) {
        a.near_o = (float *)ws;
        a.near_ml = (float *)((char *)ws + align256(nq * Hq * (int64_t)LSA_HEAD_DIM * 4));
        a.near_plan = (int2 *)((char *)a.near_ml + align256(nq * Hq * (int64_t)2 * 4));
        a.near_tile = (int4 *)((char *)a.near_plan + align256(nq * 8));
    }
    if (nsplit > 1) {
        if (((uintptr_t)ws & 255u) != 0) return fail(LSA_ERR_ARG, "workspace must be 256-byte aligned");
        a.part_o = (float *)ws;
        a.part_ml = (float *)((char *)ws + align256(nq * Hq * (int64_t)nsplit * LSA_HEAD_DIM * 4));
    }
    if (phased) {
        const int64_t R = phase_ranges(Tk);
        a.n_ranges = (int32_t)R;
        a.range_rows = (Tk + R - 1) / R;
        a.range_off = (int32_t *)ws;
        a.state_o = (float *)((char *)ws + align256(nq * (R + 1) * 4));
        a.state_ml = (float *)((char *)a.state_o + align256(nq * Hq * (int64_t)LSA_HEAD_DIM * 4));
    }
    cudaError_t e = lsa::launch_attention(a, (cudaStream_t)stream, sm_count());
    if (e != cudaSuccess) return cuda_fail(e, "attention launch");
    return LSA_OK;
}

// ---- context parallelism (token ranges over ranks) ----

int32_t lsa_shard_slots(const lsa_params *p)
{
    if (!p) return -1;
    return (int32_t)expand_slots(cand_cap(p), top_buckets(p));
}

int64_t lsa_shard_exchange_bytes(int64_t nq, const lsa_params *p)
{
    if (!p || nq < 0) return -1;
    return align256(nq * 4) + nq * (int64_t)lsa_shard_slots(p) * 8;
}

int64_t lsa_shard_local_workspace_bytes(int64_t nq, int64_t n_blocks, const lsa_params *p)
{
    if (!p || nq < 0 || n_blocks < 0) return -1;
    return index_layout(nq, n_blocks, p, true).bytes;
}

int lsa_index_shard_local(const float *qidx, const int64_t *pos, int64_t nq, const lsa_cache *cache, int64_t b_first,
                          void *xchg, const lsa_params *p, void *ws, int64_t ws_bytes, void *stream)
{
    ShardLocal sl{b_first, xchg};
    return index_impl(qidx, pos, nq, cache, nullptr, nullptr, nullptr, 0, p, ws, ws_bytes, stream, &sl);
}

int64_t lsa_shard_merge_workspace_bytes(int64_t nq, const lsa_params *p)
{
    if (!p || nq < 0) return -1;
    const int64_t KC = lsa_shard_slots(p);
    return 3 * align256(nq * 4) + align256(nq * KC * 16) + align256(nq * KC * 4);
}

int lsa_index_shard_merge(const void *xchg_all, int32_t n_shards, const int64_t *pos, int64_t nq,
                          const int32_t *members, const int32_t *count, int64_t n_blocks, int32_t *lists,
                          int32_t *lens, int32_t Lmax, const lsa_params *p, void *ws, int64_t ws_bytes, void *stream)
{
    int rc = check_params(p);
    if (rc) return rc;
    if (p->mode != LSA_MODE_FLAT) return fail(LSA_ERR_ARG, "context-parallel search is Flat only");
    if (nq < 0 || n_blocks < 0) return fail(LSA_ERR_SHAPE, "nq and n_blocks must be >= 0");
    if (nq == 0) return LSA_OK;
    const int64_t KC = lsa_shard_slots(p);
    if (n_shards < 1 || n_shards > 32) return fail(LSA_ERR_ARG, "n_shards = %d: need 1..32", n_shards);
    if (!xchg_all || !pos || !lists || !lens || (n_blocks > 0 && (!members || !count)))
        return fail(LSA_ERR_ARG, "xchg_all, pos, members, count, lists and lens must be non-NULL");
    if (((uintptr_t)xchg_all & 255u) || !aligned16(lists) || (members && !aligned16(members)))
        return fail(LSA_ERR_ARG, "xchg_all must be 256-byte, lists and members 16-byte aligned");
    if (Lmax < lsa_list_budget(p)) return fail(LSA_ERR_SHAPE, "Lmax %d < list budget %d", Lmax, lsa_list_budget(p));
    if (lsa::rank_expand_smem_bytes((int)KC, n_blocks) > 227 * 1024)
        return fail(LSA_ERR_ARG, "%lld blocks too many for the expansion kernel", (long long)n_blocks);
    const int64_t need = lsa_shard_merge_workspace_bytes(nq, p);
    if (!ws || ws_bytes < need)
        return fail(LSA_ERR_WORKSPACE, "merge workspace %lld bytes < %lld", (long long)ws_bytes, (long long)need);
    if (((uintptr_t)ws & 255u) != 0) return fail(LSA_ERR_ARG, "workspace must be 256-byte aligned");
    char *w = (char *)ws;
    lsa::IndexWs m{};
    m.tau = (float *)w;
    m.cnt = (int32_t *)(w + align256(nq * 4));
    m.horizon = (int32_t *)(w + 2 * align256(nq * 4));
    m.cand4 = (float *)(w + 3 * align256(nq * 4));
    m.cand_g = (int32_t *)(w + 3 * align256(nq * 4) + align256(nq * KC * 16));
    m.cap = (int32_t)KC;
    cudaStream_t st = (cudaStream_t)stream;
    cudaError_t e = lsa::launch_shard_merge(xchg_all, n_shards, nq, (int)KC, (int)top_buckets(p), m, st);
    if (e != cudaSuccess) return cuda_fail(e, "shard merge launch");
    lsa::IndexArgs a{};
    a.pos = pos;
    a.nq = nq;
    a.n_blocks = n_blocks;
    a.members = members;
    a.count = count;
    a.centroid_bf16 = nullptr;
    a.lists = lists;
    a.lens = lens;
    a.Lmax = Lmax;
    a.k = p->k;
    a.sink = p->sink;
    a.window = p->window;
    a.P = (int32_t)top_buckets(p);
    e = lsa::launch_expand_merged(a, m, st);
    if (e != cudaSuccess) return cuda_fail(e, "expansion launch");
    return LSA_OK;
}

int lsa_shard_publish_members(const lsa_cache *cache, int64_t b_first, int32_t *members_out, int32_t *count_out,
                              void *stream)
{
    if (!cache || !members_out || !count_out) return fail(LSA_ERR_ARG, "cache and tables must be non-NULL");
    if (b_first < 0) return fail(LSA_ERR_SHAPE, "b_first < 0");
    if (cache->n_blocks == 0) return LSA_OK;
    if (!cache->members || !cache->count) return fail(LSA_ERR_ARG, "cache arrays are NULL");
    cudaError_t e = lsa::launch_publish_members(cache->members, cache->count, cache->n_blocks * LSA_BUCKETS, 0,
                                                b_first * LSA_BLOCK, members_out, count_out, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "publish launch");
    return LSA_OK;
}

int lsa_shard_local_lists(const int32_t *lists, const int32_t *lens, int64_t nq, int32_t Lmax, int64_t t_begin,
                          int64_t t_end, int32_t *out_lists, int32_t *out_lens, void *stream)
{
    if (nq < 0 || Lmax < 1 || t_begin < 0 || t_end < t_begin) return fail(LSA_ERR_SHAPE, "bad nq, Lmax or range");
    if (nq == 0) return LSA_OK;
    if (!lists || !lens || !out_lists || !out_lens) return fail(LSA_ERR_ARG, "pointers must be non-NULL");
    if (out_lists == lists) return fail(LSA_ERR_ARG, "out_lists must not alias lists");
    cudaError_t e = lsa::launch_local_lists(lists, lens, nq, Lmax, t_begin, t_end, out_lists, out_lens,
                                            (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "local lists launch");
    return LSA_OK;
}

int lsa_attention_combine(const uint16_t *O_parts, const float *lse_parts, int32_t n_parts, int64_t nq, int32_t Hq,
                          int32_t head_dim, uint16_t *O, float *lse, void *stream)
{
    if (head_dim != LSA_HEAD_DIM) return fail(LSA_ERR_ARG, "head_dim must be %d", LSA_HEAD_DIM);
    if (n_parts < 1 || nq < 0 || Hq < 1) return fail(LSA_ERR_SHAPE, "need n_parts >= 1, nq >= 0, Hq >= 1");
    if (nq == 0) return LSA_OK;
    if (!O_parts || !lse_parts || !O) return fail(LSA_ERR_ARG, "O_parts, lse_parts and O must be non-NULL");
    if (((uintptr_t)O_parts & 7u) || ((uintptr_t)O & 7u)) return fail(LSA_ERR_ARG, "O_parts and O must be 8-byte aligned");
    cudaError_t e = lsa::launch_combine_parts(O_parts, lse_parts, n_parts, nq, Hq, O, lse, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "combine launch");
    return LSA_OK;
}

}  // extern "C"
