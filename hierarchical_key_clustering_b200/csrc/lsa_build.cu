// Build path of the LSA indexer on sm_100a: normalise + pool, per-block Ward
// clustering into the bucket cache, and the tree of merged buckets.
//
// Method: Latent Sparse Attention pages -- learnaivisually explainer, "How
// the hierarchy is built" (normalise, sum n_pool = 4 consecutive keys, Ward
// merge of each full block into a fixed number of buckets, centroid + key
// table per bucket, and the same merging again on the buckets for the
// tree); zhichai forum post, "Key points" (64-dim, 512-key blocks, buckets of
// ~8 and at most 16 keys); sotaaz blog, "The same steps in general", step 2.
#include "lsa_common.cuh"
#include "lsa_kernels.h"

namespace lsa {

// ---------------------------------------------------------------------------
// a1: one warp per pooled item; lane l owns dims l and l + 32 of each key.
// 1 KB read + 256 B written per item, fully coalesced.
__global__ void __launch_bounds__(256) k_pool_norm(const float *__restrict__ keys, int64_t item_begin,
                                                   int64_t item_end, float *__restrict__ pooled)
{
    const int lane = threadIdx.x & 31;
    const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t j = item_begin + warp; j < item_end; j += nwarps) {
        const float *x = keys + j * (LSA_NP * LSA_D);
        float a[LSA_NP], b[LSA_NP];
#pragma unroll
        for (int e = 0; e < LSA_NP; ++e) {
            a[e] = __ldcs(x + e * LSA_D + lane);
            b[e] = __ldcs(x + e * LSA_D + lane + 32);
        }
        float ya = 0.0f, yb = 0.0f;
#pragma unroll
        for (int e = 0; e < LSA_NP; ++e) {
            float na = a[e], nb = b[e];
            warp_normalize(na, nb);
            if (e == 0) {
                ya = na;
                yb = nb;
            } else {
                ya = __fadd_rn(ya, na);
                yb = __fadd_rn(yb, nb);
            }
        }
        pooled[j * LSA_D + lane] = ya;
        pooled[j * LSA_D + lane + 32] = yb;
    }
}

// ---------------------------------------------------------------------------
// Shared-memory layout of the Ward / pairing CTA (128 threads, one per item).
constexpr int YS = LSA_D + 1;       // padded row of an item (conflict-free)
constexpr int DS = LSA_NITEMS + 1;  // padded row of the cost matrix
constexpr size_t WARD_SMEM = sizeof(float) * (LSA_NITEMS * YS + LSA_NITEMS * DS);

struct ArgMin {
    float d;
    int ij;  // i * 128 + j, i < j
};

__device__ __forceinline__ bool better(float d, int ij, float d2, int ij2)
{
    return d < d2 || (d == d2 && ij < ij2);
}

// Block-wide argmin of (d, ij) over 128 threads; every thread gets the result.
__device__ __forceinline__ ArgMin block_argmin128(float d, int ij, float *red_d, int *red_ij)
{
#pragma unroll
    for (int s = 16; s >= 1; s >>= 1) {
        float d2 = __shfl_xor_sync(LSA_FULL, d, s);
        int ij2 = __shfl_xor_sync(LSA_FULL, ij, s);
        if (better(d2, ij2, d, ij)) {
            d = d2;
            ij = ij2;
        }
    }
    const int w = threadIdx.x >> 5;
    if ((threadIdx.x & 31) == 0) {
        red_d[w] = d;
        red_ij[w] = ij;
    }
    __syncthreads();
    ArgMin r{red_d[0], red_ij[0]};
#pragma unroll
    for (int k = 1; k < 4; ++k)
        if (better(red_d[k], red_ij[k], r.d, r.ij)) {
            r.d = red_d[k];
            r.ij = red_ij[k];
        }
    __syncthreads();
    return r;
}

// Minimum of row r over the columns j < m, j != r, with ok(j), ties to the
// lowest j -- exactly what an ascending scan keeping the first strictly
// smaller value finds ((+inf, -1) when no column qualifies).  The whole warp
// computes it (lane l looks at columns l, l + 32, l + 64, l + 96) and every
// lane gets it.
template <typename Ok>
__device__ __forceinline__ void warp_row_min(const float *row, int r, int m, Ok ok, float &best, int &bj)
{
    const int lane = threadIdx.x & 31;
    float b = __int_as_float(0x7f800000);
    int jb = -1;
#pragma unroll
    for (int k = 0; k < LSA_NITEMS / 32; ++k) {
        const int j = lane + 32 * k;
        if (j < m && j != r && ok(j)) {
            const float v = row[j];
            if (v < b) {
                b = v;
                jb = j;
            }
        }
    }
#pragma unroll
    for (int s = 16; s >= 1; s >>= 1) {
        const float b2 = __shfl_xor_sync(LSA_FULL, b, s);
        const int j2 = __shfl_xor_sync(LSA_FULL, jb, s);
        if (j2 >= 0 && (jb < 0 || b2 < b || (b2 == b && j2 < jb))) {
            b = b2;
            jb = j2;
        }
    }
    best = b;
    bj = jb;
}

// Fill D[i][j] = f_ij * |Y_i - Y_j|^2 (fixed order), where f_ij = fac(i, j).
// Thread t handles pairs (t, (t + delta) mod 128), delta = 1..63, and
// delta = 64 for t < 64: every unordered pair exactly once.
template <typename Fac>
__device__ void fill_costs(const float *Y, float *D, int m, Fac fac)
{
    const int t = threadIdx.x;
    if (t < m) {
        float yi[LSA_D];
#pragma unroll
        for (int d = 0; d < LSA_D; ++d) yi[d] = Y[t * YS + d];
        for (int delta = 1; delta <= 64; ++delta) {
            if (delta == 64 && t >= 64) break;
            int j = (t + delta) & (LSA_NITEMS - 1);
            if (j >= m) continue;
            float tt[32];
#pragma unroll
            for (int l = 0; l < 32; ++l) {
                float e0 = __fsub_rn(yi[l], Y[j * YS + l]);
                float e1 = __fsub_rn(yi[l + 32], Y[j * YS + l + 32]);
                tt[l] = __fadd_rn(__fmul_rn(e0, e0), __fmul_rn(e1, e1));
            }
            float v = __fmul_rn(fac(t, j), thread_tree32(tt));
            D[t * DS + j] = v;
            D[j * DS + t] = v;
        }
    }
}

// ---------------------------------------------------------------------------
// a2: one CTA per complete block.  128 pooled items, unit weight.  Merge the
// cheapest pair with n_i + n_j <= cap (ties to the lowest (i, j)), keep the
// lower id, update costs by Lance-Williams for Ward:
//   D(k, i+j) = ((n_i+n_k) D(k,i) + (n_j+n_k) D(k,j) - n_k D(i,j)) / (n_i+n_j+n_k)
// until 64 buckets remain.  Then write bucket ids, member tables, counts and
// normalised centroids (sum of member pooled keys in ascending item order).
__global__ void __launch_bounds__(128) k_ward(const float *__restrict__ pooled, int64_t blk_begin, int cap,
                                              uint8_t *__restrict__ item_bucket, int32_t *__restrict__ members,
                                              int32_t *__restrict__ count, float *__restrict__ centroid,
                                              uint16_t *__restrict__ centroid_bf16)
{
    extern __shared__ float smem[];
    float *Y = smem;
    float *D = smem + LSA_NITEMS * YS;
    __shared__ int nl[LSA_NITEMS];  // cluster size, or 1000 once merged away
    __shared__ int root[LSA_NITEMS];
    __shared__ int rank_of[LSA_NITEMS];
    __shared__ int mlist[LSA_NITEMS][4];
    __shared__ float red_d[4];
    __shared__ int red_ij[4];
    __shared__ int warp_live[4];

    const int t = threadIdx.x;
    const int64_t b = blk_begin + blockIdx.x;
    const float *src = pooled + b * (LSA_NITEMS * LSA_D);
    for (int i = t; i < LSA_NITEMS * LSA_D; i += 128) Y[(i >> 6) * YS + (i & 63)] = src[i];
    nl[t] = 1;
    root[t] = t;
    __syncthreads();
    fill_costs(Y, D, LSA_NITEMS, [](int, int) { return 0.5f; });
    __syncthreads();

    const int DEAD = 1000;
    const float INF = __int_as_float(0x7f800000);
    bool failed = false;
    // Row minima: thread t keeps the cheapest eligible partner of cluster t
    // (n_t + n_j <= cap, ties to the lowest j).  A merge of (i, j) into i
    // changes only column i (new costs) and column j (gone), so a row needs a
    // rescan only if it is row i or its partner was i or j; every other row
    // just weighs its new cost to i.
    float best = INF;
    int bj = -1;
    {
        const float *row = D + t * DS;
        for (int j = 0; j < LSA_NITEMS; ++j) {
            if (j == t || 1 + nl[j] > cap) continue;
            const float v = row[j];
            if (v < best) {
                best = v;
                bj = j;
            }
        }
    }
    for (int it = 0; it < LSA_NITEMS - LSA_NBKT; ++it) {
        const int nt = nl[t];
        int ij = (bj < 0) ? 0x7fffffff : (min(t, bj) * LSA_NITEMS + max(t, bj));
        ArgMin am = block_argmin128(best, ij, red_d, red_ij);
        if (am.ij == 0x7fffffff) {  // no finite eligible cost: non-finite keys
            failed = true;
            break;
        }
        const int bi = am.ij >> 7, bjj = am.ij & 127;
        const float dij = D[bi * DS + bjj];
        const int ni = nl[bi], nj = nl[bjj];
        if (nt < DEAD && t != bi && t != bjj) {
            float a = __fmul_rn((float)(ni + nt), D[t * DS + bi]);
            float c2 = __fmul_rn((float)(nj + nt), D[t * DS + bjj]);
            float c3 = __fmul_rn((float)nt, dij);
            float v = __fdiv_rn(__fsub_rn(__fadd_rn(a, c2), c3), (float)(ni + nj + nt));
            D[t * DS + bi] = v;
            D[bi * DS + t] = v;
        }
        if (root[t] == bjj) root[t] = bi;
        __syncthreads();
        if (t == bi) nl[t] = ni + nj;
        if (t == bjj) nl[t] = DEAD;
        __syncthreads();
        const int ntn = nl[t];
        const bool live = ntn < DEAD;
        const bool need = live && (t == bi || bj == bi || bj == bjj);
        if (!live) {
            best = INF;
            bj = -1;
        } else if (!need && ntn + nl[bi] <= cap) {
            const float v = D[t * DS + bi];
            if (v < best || (v == best && bi < bj)) {
                best = v;
                bj = bi;
            }
        }
        for (unsigned pend = __ballot_sync(LSA_FULL, need); pend; pend &= pend - 1) {
            const int l = __ffs(pend) - 1;
            const int r = (t & ~31) + l;
            const int nr = nl[r];
            float b2;
            int j2;
            warp_row_min(D + r * DS, r, LSA_NITEMS, [&](int j) { return nr + nl[j] <= cap; }, b2, j2);
            if ((t & 31) == l) {
                best = b2;
                bj = j2;
            }
        }
    }

    if (failed) {  // leave this block's buckets empty rather than write out of range
        item_bucket[b * LSA_NITEMS + t] = 0xff;
        if (t < LSA_NBKT) {
            const int64_t g = b * LSA_NBKT + t;
            count[g] = 0;
            for (int s = 0; s < LSA_NSLOT; ++s) members[g * LSA_NSLOT + s] = -1;
            for (int d = 0; d < LSA_D; ++d) {
                centroid[g * LSA_D + d] = 0.0f;
                centroid_bf16[g * LSA_D + d] = 0;
            }
        }
        return;
    }

    // rank of each surviving cluster id (ascending ids)
    const bool live = nl[t] < DEAD;
    unsigned bal = __ballot_sync(LSA_FULL, live);
    if ((t & 31) == 0) warp_live[t >> 5] = __popc(bal);
    __syncthreads();
    int before = 0;
    for (int w = 0; w < (t >> 5); ++w) before += warp_live[w];
    if (live) rank_of[t] = before + __popc(bal & ((1u << (t & 31)) - 1u));
    // slot of item t inside its cluster (ascending items)
    const int r = root[t];
    int slot = 0;
    for (int u = 0; u < t; ++u) slot += (root[u] == r);
    mlist[r][slot] = t;
    __syncthreads();
    item_bucket[b * LSA_NITEMS + t] = (uint8_t)rank_of[r];

    // one warp per bucket: member table, count and centroid
    const int lane = t & 31;
    for (int c = t >> 5; c < LSA_NITEMS; c += 4) {
        if (nl[c] >= DEAD) continue;
        const int n = nl[c];
        const int64_t g = b * LSA_NBKT + rank_of[c];
        if (lane < LSA_NSLOT) {
            int s = lane >> 2;
            members[g * LSA_NSLOT + lane] = (s < n) ? (int32_t)(b * LSA_BLK + LSA_NP * mlist[c][s] + (lane & 3)) : -1;
        }
        if (lane == 0) count[g] = LSA_NP * n;
        float sa = 0.0f, sb = 0.0f;
        for (int s = 0; s < n; ++s) {
            sa = __fadd_rn(sa, Y[mlist[c][s] * YS + lane]);
            sb = __fadd_rn(sb, Y[mlist[c][s] * YS + lane + 32]);
        }
        warp_normalize(sa, sb);
        centroid[g * LSA_D + lane] = sa;
        centroid[g * LSA_D + lane + 32] = sb;
        centroid_bf16[g * LSA_D + lane] = f2bf_bits(sa);
        centroid_bf16[g * LSA_D + lane + 32] = f2bf_bits(sb);
    }
}

// ---------------------------------------------------------------------------
// a3, level 0 of the tree: one warp per bucket.  sum = member pooled keys in
// ascending item order, weight = items, min/max block = its block.
__global__ void __launch_bounds__(256) k_tree_leaves(const float *__restrict__ pooled,
                                                     const int32_t *__restrict__ members,
                                                     const int32_t *__restrict__ count, int64_t g_first,
                                                     int64_t nb, TreeDev tr)
{
    const int lane = threadIdx.x & 31;
    const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t g = g_first + warp; g < nb; g += nwarps) {
        const int cnt = count[g];
        float sa = 0.0f, sb = 0.0f;
        for (int e = 0; e < cnt; e += LSA_NP) {
            int64_t item = members[g * LSA_NSLOT + e] / LSA_NP;
            sa = __fadd_rn(sa, pooled[item * LSA_D + lane]);
            sb = __fadd_rn(sb, pooled[item * LSA_D + lane + 32]);
        }
        tr.sum[g * LSA_D + lane] = sa;
        tr.sum[g * LSA_D + lane + 32] = sb;
        warp_normalize(sa, sb);
        tr.centroid[g * LSA_D + lane] = sa;
        tr.centroid[g * LSA_D + lane + 32] = sb;
        tr.centroid_bf16[g * LSA_D + lane] = f2bf_bits(sa);
        tr.centroid_bf16[g * LSA_D + lane + 32] = f2bf_bits(sb);
        if (lane == 0) {
            tr.weight[g] = cnt / LSA_NP;
            tr.min_block[g] = tr.max_block[g] = (int32_t)(g / LSA_NBKT);
            tr.child[2 * g] = tr.child[2 * g + 1] = -1;
            tr.parent[g] = -1;
        }
    }
}

// a3, one level: one CTA per run of (up to) 128 consecutive nodes of the level
// below.  Greedy Ward pairing: D(i,j) = (w_i w_j / (w_i + w_j)) |mu_i - mu_j|^2
// with mu = sum / w; repeatedly pair the cheapest two unpaired nodes (ties to
// the lowest (i, j)).  New nodes (pairs at their lower member, lone leftover
// as itself) are written in ascending order of that member.
__global__ void __launch_bounds__(128) k_tree_pair(TreeDev tr, int64_t run0, int64_t off_prev, int64_t n_prev,
                                                   int64_t off)
{
    extern __shared__ float smem[];
    float *Y = smem;
    float *D = smem + LSA_NITEMS * YS;
    __shared__ int w_s[LSA_NITEMS];
    __shared__ int partner[LSA_NITEMS];
    __shared__ int rank_of[LSA_NITEMS];
    __shared__ float red_d[4];
    __shared__ int red_ij[4];
    __shared__ int warp_cnt[4];

    const int t = threadIdx.x;
    const int64_t first = (run0 + blockIdx.x) * LSA_RUN;
    const int m = (int)min((int64_t)LSA_RUN, n_prev - first);
    const int64_t base = off_prev + first;
    if (t < m) w_s[t] = tr.weight[base + t];
    partner[t] = (t < m) ? -1 : -2;
    __syncthreads();
    for (int i = t; i < m * LSA_D; i += 128) {
        int node = i >> 6, d = i & 63;
        Y[node * YS + d] = __fdiv_rn(tr.sum[(base + node) * LSA_D + d], (float)w_s[node]);
    }
    __syncthreads();
    fill_costs(Y, D, m, [&](int i, int j) {
        return __fdiv_rn(__fmul_rn((float)w_s[i], (float)w_s[j]), (float)(w_s[i] + w_s[j]));
    });
    __syncthreads();

    // Row minima over unpaired partners (ties to the lowest j); pairing (i, j)
    // removes columns i and j, so only rows whose partner was i or j rescan.
    const float INF = __int_as_float(0x7f800000);
    float best = INF;
    int bj = -1;
    if (partner[t] == -1) {
        const float *row = D + t * DS;
        for (int j = 0; j < m; ++j) {
            if (j == t || partner[j] != -1) continue;
            const float v = row[j];
            if (v < best) {
                best = v;
                bj = j;
            }
        }
    }
    for (int it = 0; it < m / 2; ++it) {
        int ij = (bj < 0) ? 0x7fffffff : (min(t, bj) * LSA_NITEMS + max(t, bj));
        ArgMin am = block_argmin128(best, ij, red_d, red_ij);
        if (am.ij == 0x7fffffff) break;  // only non-finite costs left
        const int bi = am.ij >> 7, bjj = am.ij & 127;
        if (t == bi) partner[t] = bjj;
        if (t == bjj) partner[t] = bi;
        __syncthreads();
        const bool open = partner[t] == -1;
        const bool need = open && (bj == bi || bj == bjj);
        if (!open) {
            best = INF;
            bj = -1;
        }
        for (unsigned pend = __ballot_sync(LSA_FULL, need); pend; pend &= pend - 1) {
            const int l = __ffs(pend) - 1;
            const int r = (t & ~31) + l;
            float b2;
            int j2;
            warp_row_min(D + r * DS, r, m, [&](int j) { return partner[j] == -1; }, b2, j2);
            if ((t & 31) == l) {
                best = b2;
                bj = j2;
            }
        }
    }
    if (t == 0) {  // pair whatever is still unpaired in index order (no-op for finite costs)
        int open = -1, left = 0;
        for (int i = 0; i < m; ++i) left += (partner[i] == -1);
        for (int i = 0; i < m && left > 1; ++i) {
            if (partner[i] != -1) continue;
            if (open < 0) {
                open = i;
            } else {
                partner[open] = i;
                partner[i] = open;
                open = -1;
                left -= 2;
            }
        }
    }
    __syncthreads();

    // heads: lower member of each pair, or a lone node
    const bool head = (t < m) && (partner[t] < 0 || partner[t] > t);
    unsigned bal = __ballot_sync(LSA_FULL, head);
    if ((t & 31) == 0) warp_cnt[t >> 5] = __popc(bal);
    __syncthreads();
    int before = 0;
    for (int w = 0; w < (t >> 5); ++w) before += warp_cnt[w];
    if (head) rank_of[t] = before + __popc(bal & ((1u << (t & 31)) - 1u));
    __syncthreads();

    const int lane = t & 31;
    const int64_t out0 = off + first / 2;
    for (int c = t >> 5; c < m; c += 4) {
        const int pc = partner[c];
        if (!(pc < 0 || pc > c)) continue;
        const int64_t out = out0 + rank_of[c];
        const int64_t a = base + c;
        const int64_t bb = (pc >= 0) ? base + pc : -1;
        float sa = tr.sum[a * LSA_D + lane], sb = tr.sum[a * LSA_D + lane + 32];
        if (bb >= 0) {
            sa = __fadd_rn(sa, tr.sum[bb * LSA_D + lane]);
            sb = __fadd_rn(sb, tr.sum[bb * LSA_D + lane + 32]);
        }
        tr.sum[out * LSA_D + lane] = sa;
        tr.sum[out * LSA_D + lane + 32] = sb;
        warp_normalize(sa, sb);
        tr.centroid[out * LSA_D + lane] = sa;
        tr.centroid[out * LSA_D + lane + 32] = sb;
        tr.centroid_bf16[out * LSA_D + lane] = f2bf_bits(sa);
        tr.centroid_bf16[out * LSA_D + lane + 32] = f2bf_bits(sb);
        if (lane == 0) {
            const int32_t local = (int32_t)(out - off);
            tr.child[2 * out] = (int32_t)(a - off_prev);
            tr.child[2 * out + 1] = (bb >= 0) ? (int32_t)(bb - off_prev) : -1;
            tr.parent[a] = local;
            if (bb >= 0) tr.parent[bb] = local;
            tr.parent[out] = -1;
            tr.weight[out] = tr.weight[a] + (bb >= 0 ? tr.weight[bb] : 0);
            int32_t mn = tr.min_block[a], mx = tr.max_block[a];
            if (bb >= 0) {
                mn = min(mn, tr.min_block[bb]);
                mx = max(mx, tr.max_block[bb]);
            }
            tr.min_block[out] = mn;
            tr.max_block[out] = mx;
        }
    }
}

// ---------------------------------------------------------------------------
// Launchers.

cudaError_t launch_pool_norm(const float *keys, int64_t item_begin, int64_t item_end, float *pooled,
                             cudaStream_t st, int n_sm)
{
    if (item_end <= item_begin) return cudaSuccess;
    int64_t warps = item_end - item_begin;
    int64_t blocks = (warps + 7) / 8;
    int64_t cap = (int64_t)n_sm * 16;
    if (blocks > cap) blocks = cap;
    const int kt = kt_begin("k_pool_norm", st);
    k_pool_norm<<<(unsigned)blocks, 256, 0, st>>>(keys, item_begin, item_end, pooled);
    kt_end(kt, st);
    count_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_ward(const float *pooled, int64_t blk_begin, int64_t blk_end, int cap, uint8_t *item_bucket,
                        int32_t *members, int32_t *count, float *centroid, uint16_t *centroid_bf16,
                        cudaStream_t st)
{
    if (blk_end <= blk_begin) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(k_ward, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)WARD_SMEM);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(k_tree_pair, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)WARD_SMEM);
    if (e != cudaSuccess) return e;
    int64_t n = blk_end - blk_begin;
    for (int64_t s = 0; s < n; s += 2147483647LL) {
        int64_t cnt = (n - s) < 2147483647LL ? (n - s) : 2147483647LL;
        const int kt = kt_begin("k_ward", st);
        k_ward<<<(unsigned)cnt, 128, WARD_SMEM, st>>>(pooled, blk_begin + s, cap, item_bucket, members, count,
                                                      centroid, centroid_bf16);
        kt_end(kt, st);
        count_launches(1);
    }
    return cudaGetLastError();
}

cudaError_t launch_tree(const float *pooled, const int32_t *members, const int32_t *count, int64_t g_first,
                        int64_t nb, const TreeDev &tr, const int64_t *level_size, const int64_t *level_offset,
                        int n_levels, cudaStream_t st, int n_sm)
{
    cudaError_t e = cudaFuncSetAttribute(k_tree_pair, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)WARD_SMEM);
    if (e != cudaSuccess) return e;
    int64_t blocks = (nb - g_first + 7) / 8;
    if (blocks > (int64_t)n_sm * 16) blocks = (int64_t)n_sm * 16;
    if (blocks < 1) blocks = 1;
    const int kt = kt_begin("k_tree_leaves", st);
    k_tree_leaves<<<(unsigned)blocks, 256, 0, st>>>(pooled, members, count, g_first, nb, tr);
    kt_end(kt, st);
    count_launches(1);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    // a run of 128 nodes is paired from its own nodes alone, and every run
    // but a level's last is full (its 64 parents start at 64 x its index):
    // only the runs from the first changed node on change, level by level
    int64_t changed = g_first;
    for (int l = 1; l < n_levels; ++l) {
        const int64_t n_prev = level_size[l - 1];
        const int64_t runs = (n_prev + LSA_RUN - 1) / LSA_RUN;
        const int64_t run0 = changed / LSA_RUN;
        if (runs > run0) {
            const int ktp = kt_begin("k_tree_pair", st);
            k_tree_pair<<<(unsigned)(runs - run0), 128, WARD_SMEM, st>>>(tr, run0, level_offset[l - 1], n_prev,
                                                                        level_offset[l]);
            kt_end(ktp, st);
            count_launches(1);
            e = cudaGetLastError();
            if (e != cudaSuccess) return e;
        }
        changed = run0 * (LSA_RUN / 2);
    }
    return cudaSuccess;
}

}  // namespace lsa
