// Query path of the LSA indexer on sm_100a: query normalisation, Flat search
// (fused score + top-P selection, score matrix never stored), Tree beam
// search, and best-first expansion into the sorted index list with the
// attention sink and the recent window.
//
// Method: Latent Sparse Attention pages -- learnaivisually explainer, "What
// one query actually does" and the "Search style" table; sotaaz blog, "The
// same steps in general" (steps 3-5 and read_list) and the window/skip rule
// that follows it; zhichai forum post, "Key points" (Flat vs Tree).
//
// Flat selection.  A query that sees N buckets needs its top P buckets,
// P = ceil((k + sink + window) / 4).  Pass 1 (tcgen05, lsa_score_tc.cu)
// scores every bucket and histograms the maximum of each group of g
// consecutive buckets (g a power of two giving 4P..8P groups).  The P-th
// largest group maximum is a score of P distinct buckets, so it is <= the
// P-th largest score, and so is tau, the lower edge of its histogram bin:
// every bucket scoring at least tau is kept by pass 2, which recomputes the same scores
// bit for bit on the tensor cores (or, for <= 16 queries, reads the scores
// pass 1 stored) and appends the passing (score, id) pairs.  A query whose
// candidates overflow their slots is redone exactly (radix select on the
// recomputed scores) by the fallback kernel.  The candidates are then ranked
// by (score desc, id asc) and expanded.
#include "lsa_common.cuh"
#include "lsa_kernels.h"

namespace lsa {


// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_qnorm(const float *__restrict__ qidx, const int64_t *__restrict__ pos,
                                               int64_t nq, int64_t n_blocks, IndexWs ws)
{
    const int lane = threadIdx.x & 31;
    const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t q = warp; q < nq; q += nwarps) {
        float a = qidx[q * LSA_D + lane], b = qidx[q * LSA_D + lane + 32];
        warp_normalize(a, b);
        ws.qhat[q * LSA_D + lane] = f2bf_bits(a);
        ws.qhat[q * LSA_D + lane + 32] = f2bf_bits(b);
        if (lane == 0) {
            int64_t p = pos[q];
            int64_t H = p < 0 ? 0 : p / LSA_BLK;
            if (H > n_blocks) H = n_blocks;
            ws.horizon[q] = (int32_t)H;
            ws.cnt[q] = 0;
        }
        for (int i = lane; i < HIST_BINS; i += 32) ws.ghist[q * HIST_BINS + i] = 0u;
    }
}

// Score of one bucket on the CUDA cores: fp32 FMA chain over d = 0..63 of the
// bf16 operands (k_fallback).  It can differ from the tensor cores' sum of
// the same products in the last bit, which only matters for scores within
// ~1e-6 of each other, at the one cut a Flat search makes.
__device__ __forceinline__ float dot_bf16_row(const float *qf, const uint16_t *__restrict__ c)
{
    const uint4 *c4 = reinterpret_cast<const uint4 *>(c);
    float acc = 0.0f;
#pragma unroll
    for (int v = 0; v < 8; ++v) {
        uint4 w = __ldg(c4 + v);
        uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            acc = fmaf(qf[v * 8 + 2 * h], __uint_as_float(ww[h] << 16), acc);
            acc = fmaf(qf[v * 8 + 2 * h + 1], __uint_as_float(ww[h] & 0xffff0000u), acc);
        }
    }
    return acc;
}

// Score of one tree node, rounded once to fp32 from the fp64 sum over
// d = 0..63 of the bf16 products taken in that order.  A product of two bf16
// values is exact in fp64, so each fused step rounds exactly like a separate
// add and the result is the same fp32 value as a plain fp64 dot product
// written out in index order.  A beam search cuts at every level; scoring
// this way makes those cuts independent of the accumulation order.
__device__ __forceinline__ float dot_bf16_row_f64(const float *qf, const uint16_t *__restrict__ c)
{
    const uint4 *c4 = reinterpret_cast<const uint4 *>(c);
    double acc = 0.0;
#pragma unroll
    for (int v = 0; v < 8; ++v) {
        uint4 w = __ldg(c4 + v);
        uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            acc = __fma_rn((double)qf[v * 8 + 2 * h], (double)__uint_as_float(ww[h] << 16), acc);
            acc = __fma_rn((double)qf[v * 8 + 2 * h + 1], (double)__uint_as_float(ww[h] & 0xffff0000u), acc);
        }
    }
    return __double2float_rn(acc);
}

// ---------------------------------------------------------------------------
// Flat pass 2 for small batches (decode): the tensor-core pass 1 stored every
// score; keep those >= tau (one thread per bucket, all queries of the batch).
__global__ void __launch_bounds__(256) k_dfilter(int64_t nq, IndexWs ws)
{
    __shared__ int Nq[SMALL_NQ];
    __shared__ float tq[SMALL_NQ];
    const int t = threadIdx.x;
    if (t < nq) {
        Nq[t] = ws.horizon[t] * LSA_NBKT;
        tq[t] = ws.tau[t];
    }
    __syncthreads();
    const int64_t b = (int64_t)blockIdx.x * 256 + t;
    for (int qi = 0; qi < nq; ++qi) {
        if (b >= Nq[qi]) continue;
        const float s = ws.scores[qi * ws.score_stride + b];
        if (s >= tq[qi]) {
            const int slot = atomicAdd(ws.cnt + qi, 1);
            if (slot < ws.cap) {
                ws.cand_s[qi * ws.cap + slot] = s;
                ws.cand_id[qi * ws.cap + slot] = (int32_t)b;
            }
        }
    }
}

// ---------------------------------------------------------------------------
// Radix select: the P-th largest key (u = f2ord(score)) among values produced
// by `get(i)` for i in [0, n); all threads of the block call it.
template <typename Get>
__device__ uint32_t block_select_kth_largest(int64_t n, int64_t P, Get get, int *hist, int *sh)
{
    uint32_t prefix = 0, mask = 0;
    int64_t rem = P;
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int i = threadIdx.x; i < 256; i += blockDim.x) hist[i] = 0;
        __syncthreads();
        const int64_t n_round = ((n + blockDim.x - 1) / blockDim.x) * blockDim.x;
        for (int64_t i = threadIdx.x; i < n_round; i += blockDim.x) {
            const bool valid = i < n;
            const uint32_t u = valid ? f2ord(get(i)) : 0u;
            const int bin = (valid && (u & mask) == prefix) ? (int)((u >> shift) & 255) : -1;
            // lanes with the same bin add once (scores cluster in few bins)
            const unsigned peers = __match_any_sync(LSA_FULL, bin);
            if (bin >= 0 && (threadIdx.x & 31) == __ffs(peers) - 1) atomicAdd(&hist[bin], __popc(peers));
        }
        __syncthreads();
        if (threadIdx.x < 32) {
            // warp 0: lane l owns bins 255-8l .. 248-8l (descending); find the
            // bin where the count from the top first reaches rem
            const int lane = threadIdx.x;
            int c8 = 0;
#pragma unroll
            for (int e = 0; e < 8; ++e) c8 += hist[255 - 8 * lane - e];
            int incl = c8;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(LSA_FULL, incl, o);
                if (lane >= o) incl += y;
            }
            const int excl = incl - c8;
            if (excl < rem && rem <= incl) {
                int acc = excl, digit = 255 - 8 * lane;
                for (int e = 0; e < 8; ++e) {
                    const int d = 255 - 8 * lane - e;
                    if (acc + hist[d] >= rem) {
                        digit = d;
                        break;
                    }
                    acc += hist[d];
                }
                sh[0] = digit;
                sh[1] = (int)(rem - acc);
            }
        }
        __syncthreads();
        prefix |= ((uint32_t)sh[0]) << shift;
        mask |= 255u << shift;
        rem = sh[1];
        __syncthreads();
    }
    return prefix;
}

// Threshold per query: P-th largest group maximum (or -inf when N <= P).
// Threshold per query from its global group-maximum histogram (used when a
// query's buckets were split over several score CTAs): tau = lower edge of
// the bin holding the P-th largest group maximum, -inf when there are <= P
// groups.  One warp per query.
__global__ void __launch_bounds__(256) k_tau(int64_t nq, int P, IndexWs ws)
{
    const int lane = threadIdx.x & 31;
    const int64_t q = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (q >= nq) return;
    const int64_t N = (int64_t)ws.horizon[q] * LSA_NBKT;
    const float NEG = __int_as_float(0xff800000);
    if (n_groups(N, P) <= P) {
        if (lane == 0) ws.tau[q] = NEG;
        return;
    }
    // lane l owns bins 255-8l .. 248-8l (descending)
    const uint32_t *h = ws.ghist + q * HIST_BINS;
    int c8 = 0;
    int cb[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        cb[e] = (int)h[HIST_BINS - 1 - 8 * lane - e];
        c8 += cb[e];
    }
    int incl = c8;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(LSA_FULL, incl, o);
        if (lane >= o) incl += y;
    }
    const int excl = incl - c8;
    if (excl < P && P <= incl) {
        int acc = excl;
        int bin = HIST_BINS - 1 - 8 * lane;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            acc += cb[e];
            if (acc >= P) {
                bin = HIST_BINS - 1 - 8 * lane - e;
                break;
            }
        }
        ws.tau[q] = bin > 0 ? HIST_LO + bin * (2.0f * -HIST_LO / HIST_BINS) : NEG;
    }
}

// Exact selection for queries whose candidates overflowed: radix select of
// the P-th largest recomputed score tau*, then all scores > tau* plus the
// lowest-id buckets scoring exactly tau* up to P in all.
__global__ void __launch_bounds__(256) k_fallback(int64_t nq, const uint16_t *__restrict__ cbf, int P, IndexWs ws)
{
    __shared__ int hist[256];
    __shared__ int sh[2];
    __shared__ float qf[LSA_D];
    __shared__ int n_out;
    __shared__ int wsum[8];
    for (int64_t q = blockIdx.x; q < nq; q += gridDim.x) {
        if (ws.cnt[q] <= ws.cap) continue;  // block-uniform
        const int64_t N = (int64_t)ws.horizon[q] * LSA_NBKT;
        if (threadIdx.x < LSA_D) qf[threadIdx.x] = bf_bits2f(ws.qhat[q * LSA_D + threadIdx.x]);
        if (threadIdx.x == 0) n_out = 0;
        __syncthreads();
        auto score = [&](int64_t b) { return dot_bf16_row(qf, cbf + b * LSA_D); };
        const float tau = ord2f(block_select_kth_largest(N, P, score, hist, sh));
        float *cs = ws.cand_s + q * ws.cap;
        int32_t *ci = ws.cand_id + q * ws.cap;
        for (int64_t b = threadIdx.x; b < N; b += blockDim.x) {
            float s = score(b);
            if (s > tau) {
                int slot = atomicAdd(&n_out, 1);
                cs[slot] = s;
                ci[slot] = (int32_t)b;
            }
        }
        __syncthreads();
        // ties at tau in ascending bucket order
        for (int64_t base = 0; base < N; base += blockDim.x) {
            if (n_out >= P) break;  // block-uniform (read after a barrier)
            int64_t b = base + threadIdx.x;
            bool tie = (b < N) && (score(b) == tau);
            unsigned bal = __ballot_sync(LSA_FULL, tie);
            const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
            if (lane == 0) wsum[w] = __popc(bal);
            __syncthreads();
            int before = n_out;
            for (int k = 0; k < w; ++k) before += wsum[k];
            before += __popc(bal & ((1u << lane) - 1u));
            if (tie && before < P) {
                cs[before] = tau;
                ci[before] = (int32_t)b;
            }
            __syncthreads();
            if (threadIdx.x == 0) {
                int tot = 0;
                for (int k = 0; k < (int)(blockDim.x >> 5); ++k) tot += wsum[k];
                n_out = min(P, n_out + tot);
            }
            __syncthreads();
        }
        if (threadIdx.x == 0) ws.cnt[q] = n_out;
        __syncthreads();
    }
}

// ---------------------------------------------------------------------------
// Tree beam search: one CTA per query, level by level from the root.
__global__ void __launch_bounds__(256) k_tree_beam(int64_t nq, TreeView tv, int W, int P, int CM, IndexWs ws)
{
    extern __shared__ uint64_t tsm[];
    uint64_t *keys = tsm;                                    // [CM]
    int32_t *cids = reinterpret_cast<int32_t *>(keys + CM);  // [CM]
    int32_t *kept = cids + CM;                               // [max(W, P)]
    __shared__ float qf[LSA_D];
    __shared__ int nc;
    __shared__ int n_kept;

    const int64_t q = blockIdx.x;
    const int t = threadIdx.x;
    const int H = ws.horizon[q];
    if (t < LSA_D) qf[t] = bf_bits2f(ws.qhat[q * LSA_D + t]);
    if (t == 0) n_kept = 0;
    __syncthreads();
    const int top = tv.n_levels - 1;
    for (int l = top; l >= 0; --l) {
        if (t == 0) nc = 0;
        __syncthreads();
        const int64_t off = tv.level_offset[l];
        const int64_t size = tv.level_size[l];
        for (int i = t; i < n_kept; i += blockDim.x) {
            const int64_t v = tv.level_offset[l + 1] + kept[i];
            const int32_t c0 = tv.child[2 * v], c1 = tv.child[2 * v + 1];
            int slot = atomicAdd(&nc, c1 >= 0 ? 2 : 1);
            cids[slot] = c0;
            if (c1 >= 0) cids[slot + 1] = c1;
        }
        if (l == top) {
            for (int64_t u = t; u < size; u += blockDim.x)
                if (tv.max_block[off + u] < H) cids[atomicAdd(&nc, 1)] = (int32_t)u;
        } else {
            // only the run of 128 nodes holding block H can mix visible
            // nodes with parents that are not visible
            const int64_t lo = ((int64_t)H >> (l + 1)) * LSA_RUN;
            const int64_t hi = min(lo + LSA_RUN, size);
            for (int64_t u = lo + t; u < hi; u += blockDim.x) {
                const int64_t v = off + u;
                if (tv.max_block[v] < H && tv.max_block[tv.level_offset[l + 1] + tv.parent[v]] >= H)
                    cids[atomicAdd(&nc, 1)] = (int32_t)u;
            }
        }
        __syncthreads();
        const int n = nc;
        const int S = (int)pow2_ceil64(n > 0 ? n : 1);
        for (int i = t; i < S; i += blockDim.x) {
            if (i < n) {
                const int32_t u = cids[i];
                keys[i] = rank_key(dot_bf16_row_f64(qf, tv.centroid_bf16 + (off + u) * LSA_D), u);
            } else {
                keys[i] = ~0ull;
            }
        }
        __syncthreads();
        block_bitonic_sort(keys, S);
        int64_t B = ((int64_t)P + ((int64_t)1 << l) - 1) >> l;
        if (B < W) B = W;
        const int nk = (int)min((int64_t)n, B);
        for (int i = t; i < nk; i += blockDim.x) kept[i] = rank_key_id(keys[i]);
        if (l == 0) {
            for (int i = t; i < nk; i += blockDim.x) {
                ws.cand_s[q * ws.cap + i] = rank_key_score(keys[i]);
                ws.cand_id[q * ws.cap + i] = rank_key_id(keys[i]);
            }
            if (t == 0) ws.cnt[q] = nk;
        }
        if (t == 0) n_kept = nk;
        __syncthreads();
    }
}

// ---------------------------------------------------------------------------
// Block-wide inclusive scan of a[0..n) in shared memory (256 threads).
__device__ void block_inclusive_scan(int *a, int n, int *wsum)
{
    const int t = threadIdx.x;
    const int per = (n + blockDim.x - 1) / blockDim.x;
    const int lo = min(n, t * per), hi = min(n, lo + per);
    int s = 0;
    for (int i = lo; i < hi; ++i) {
        s += a[i];
        a[i] = s;
    }
    // exclusive scan of per-thread totals
    const int lane = t & 31, w = t >> 5;
    int x = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(LSA_FULL, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) wsum[w] = x;
    __syncthreads();
    int before = x - s;
    for (int k = 0; k < w; ++k) before += wsum[k];
    for (int i = lo; i < hi; ++i) a[i] += before;
    __syncthreads();
}

// Weighted radix select over 64-bit rank keys (ascending = best first):
// the smallest key K with sum of w over keys <= K reaching `target`, and the
// weight still needed from K itself.  All threads of the block call it.
__device__ void block_weighted_select(const uint64_t *keys, const int32_t *w, int n, int target, int *hist,
                                      uint64_t *out_key, int *out_rem)
{
    __shared__ int sh_digit, sh_rem;
    uint64_t prefix = 0, mask = 0;
    int rem = target;
    for (int shift = 56; shift >= 0; shift -= 8) {
        for (int i = threadIdx.x; i < 256; i += blockDim.x) hist[i] = 0;
        __syncthreads();
        const int n_round = ((n + blockDim.x - 1) / blockDim.x) * blockDim.x;
        for (int i = threadIdx.x; i < n_round; i += blockDim.x) {
            int bin = -1, wt = 0;
            if (i < n && (keys[i] & mask) == prefix) {
                bin = (int)((keys[i] >> shift) & 255);
                wt = w[i];
            }
            const unsigned peers = __match_any_sync(LSA_FULL, bin);
            const int sum = __reduce_add_sync(peers, wt);
            if (bin >= 0 && (threadIdx.x & 31) == __ffs(peers) - 1) atomicAdd(&hist[bin], sum);
        }
        __syncthreads();
        if (threadIdx.x < 32) {  // ascending bins: lane l owns 8l .. 8l+7
            const int lane = threadIdx.x;
            int c8 = 0;
#pragma unroll
            for (int e = 0; e < 8; ++e) c8 += hist[8 * lane + e];
            int incl = c8;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(LSA_FULL, incl, o);
                if (lane >= o) incl += y;
            }
            const int excl = incl - c8;
            if (excl < rem && rem <= incl) {
                int acc = excl;
                for (int e = 0; e < 8; ++e) {
                    const int d = 8 * lane + e;
                    if (acc + hist[d] >= rem) {
                        sh_digit = d;
                        sh_rem = rem - acc;
                        break;
                    }
                    acc += hist[d];
                }
            }
        }
        __syncthreads();
        prefix |= (uint64_t)sh_digit << shift;
        mask |= (uint64_t)255 << shift;
        rem = sh_rem;
        __syncthreads();
    }
    *out_key = prefix;
    *out_rem = rem;
}

// Rank the candidates of one query and expand them into its index list.
//   1. count each candidate bucket's members outside near (its weight);
//   2. the walk over buckets in (score desc, id asc) order stops at the
//      bucket where the weights reach k: find that bucket (and how many of
//      its keys are still needed) by a weighted radix select -- buckets
//      ranked before it are taken whole, their order does not matter;
//   3. mark the chosen positions in one 512-bit mask per touched block
//      (blocks found through a bitmap over all visible blocks) and emit them
//      block by block in ascending order -- the far keys come out sorted
//      without sorting them;
//   4. write sink, far keys and window.
// Every bucket has >= 4 keys and at most sink + window clustered keys are
// near, so when a query has >= P candidates its best P buckets already hold
// k far keys: the cut never falls outside the top P.
__global__ void __launch_bounds__(1024) k_rank_expand(const int64_t *__restrict__ pos, const int32_t *__restrict__ members,
                                                     int32_t *__restrict__ lists, int32_t *__restrict__ lens, int Lmax,
                                                     int k, int sink, int window, int P, int CAP, int TW, IndexWs ws)
{
    extern __shared__ uint64_t rsm[];
    uint64_t *keys = rsm;                                        // [CAP]
    int32_t *wt = reinterpret_cast<int32_t *>(keys + CAP);       // [CAP]
    uint32_t *masks = reinterpret_cast<uint32_t *>(wt + CAP);    // [P][16]
    uint32_t *touched = masks + (size_t)P * 16;                  // [TW]
    int32_t *wrank = reinterpret_cast<int32_t *>(touched + TW);  // [TW]
    int32_t *slot_blk = wrank + TW;                              // [P]
    int32_t *slot_off = slot_blk + P;                            // [P]
    __shared__ int wsum[32];
    __shared__ int hist[256];
    __shared__ int tot_s;

    const int64_t q = blockIdx.x;
    const int t = threadIdx.x;
    const int64_t p = pos[q];
    const int n = min(ws.cnt[q], ws.cap);
    const int64_t w0 = p - window > 0 ? p - window : 0;
    const int64_t s_end = (int64_t)sink < p + 1 ? (int64_t)sink : p + 1;
    if (t == 0) tot_s = 0;
    for (int i = t; i < TW; i += blockDim.x) touched[i] = 0u;
    __syncthreads();
    int my_tot = 0;
    for (int i = t; i < n; i += blockDim.x) {
        const int32_t b = ws.cand_id[q * ws.cap + i];
        keys[i] = rank_key(ws.cand_s[q * ws.cap + i], b);
        const int4 *m4 = reinterpret_cast<const int4 *>(members + (int64_t)b * LSA_NSLOT);
        int nn = 0;
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            const int4 w = __ldg(m4 + v);
            const int mm[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int64_t m = mm[e];  // -1 pads are skipped
                nn += (m >= 0) && !(m < s_end || (m >= w0 && m <= p));
            }
        }
        wt[i] = nn;
        my_tot += nn;
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) my_tot += __shfl_xor_sync(LSA_FULL, my_tot, o);
    if ((t & 31) == 0) atomicAdd(&tot_s, my_tot);
    __syncthreads();
    const int nfar = min(k, tot_s);
    uint64_t cut_key = 0;
    int take = 0;
    if (nfar > 0) block_weighted_select(keys, wt, n, nfar, hist, &cut_key, &take);
    const bool any = nfar > 0;
    for (int i = t; i < n; i += blockDim.x) {
        if (any && keys[i] <= cut_key && wt[i] > 0) {
            const int blk = rank_key_id(keys[i]) / LSA_NBKT;
            atomicOr(&touched[blk >> 5], 1u << (blk & 31));
        }
    }
    __syncthreads();
    for (int i = t; i < TW; i += blockDim.x) wrank[i] = __popc(touched[i]);
    __syncthreads();
    block_inclusive_scan(wrank, TW, wsum);  // wrank[w] = touched blocks in words 0..w
    const int nslots = TW > 0 ? wrank[TW - 1] : 0;
    for (int i = t; i < nslots * 16; i += blockDim.x) masks[i] = 0u;
    __syncthreads();
    for (int i = t; i < n; i += blockDim.x) {
        if (!(any && keys[i] <= cut_key && wt[i] > 0)) continue;
        const int32_t b = rank_key_id(keys[i]);
        const int limit = (keys[i] == cut_key) ? take : 16;
        const int blk = b / LSA_NBKT;
        const uint32_t word = touched[blk >> 5];
        const int slot = wrank[blk >> 5] - __popc(word) + __popc(word & ((1u << (blk & 31)) - 1u));
        slot_blk[slot] = blk;
        const int4 *m4 = reinterpret_cast<const int4 *>(members + (int64_t)b * LSA_NSLOT);
        int idx = 0;
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            const int4 w = __ldg(m4 + v);
            const int mm[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int64_t m = mm[e];
                if (m >= 0 && !(m < s_end || (m >= w0 && m <= p))) {
                    if (idx < limit) atomicOr(&masks[slot * 16 + ((m & 511) >> 5)], 1u << (m & 31));
                    ++idx;
                }
            }
        }
    }
    __syncthreads();
    for (int sl = t; sl < nslots; sl += blockDim.x) {
        int c = 0;
#pragma unroll
        for (int w = 0; w < 16; ++w) c += __popc(masks[sl * 16 + w]);
        slot_off[sl] = c;
    }
    __syncthreads();
    block_inclusive_scan(slot_off, nslots, wsum);
    const int n_sink = (int)min(s_end, w0);
    int32_t *out = lists + q * (int64_t)Lmax;
    {
        const int lane = t & 31, warp = t >> 5, nwarps = blockDim.x >> 5;
        for (int sl = warp; sl < nslots; sl += nwarps) {
            const uint32_t word = lane < 16 ? masks[sl * 16 + lane] : 0u;
            const int c = __popc(word);
            int incl = c;
#pragma unroll
            for (int o = 1; o < 16; o <<= 1) {
                const int y = __shfl_up_sync(LSA_FULL, incl, o);
                if (lane >= o) incl += y;
            }
            int o = n_sink + slot_off[sl] - __shfl_sync(LSA_FULL, incl, 15) + incl - c;
            const int32_t base = slot_blk[sl] * LSA_BLK + lane * 32;
            uint32_t bits = word;
            while (bits) {
                const int bit = __ffs(bits) - 1;
                out[o++] = base + bit;
                bits &= bits - 1;
            }
        }
    }
    const int nwin = (int)(p - w0 + 1);
    const int len = n_sink + nfar + nwin;
    for (int i = t; i < Lmax; i += blockDim.x) {
        if (i < n_sink) out[i] = i;
        else if (i < n_sink + nfar) continue;
        else if (i < len) out[i] = (int32_t)(w0 + (i - n_sink - nfar));
        else out[i] = -1;
    }
    if (t == 0) lens[q] = len;
}

// ---------------------------------------------------------------------------
cudaError_t launch_index(const IndexArgs &a, const IndexWs &ws, const TreeView *tree, cudaStream_t st, int n_sm)
{
    if (a.nq <= 0) return cudaSuccess;
    cudaError_t e;
    {
        int64_t blocks = (a.nq + 7) / 8;
        if (blocks > (int64_t)n_sm * 32) blocks = (int64_t)n_sm * 32;
        k_qnorm<<<(unsigned)blocks, 256, 0, st>>>(a.qidx, a.pos, a.nq, a.n_blocks, ws);
        count_launches(1);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    const int64_t nb_total = a.n_blocks * LSA_NBKT;
    const bool small = a.nq <= SMALL_NQ;
    const int big_block = small ? 1024 : 256;
    if (a.mode == 0 && nb_total > 0) {
        // pass 1 on the tensor cores: group maxima (+ every score for small batches)
        ScoreTcArgs sa;
        sa.nq = a.nq;
        sa.nb_total = nb_total;
        sa.P = a.P;
        sa.mode = 0;
        sa.store = small ? 1 : 0;
        sa.chunk_tiles = 0;
        sa.wait_limit = a.wait_limit;
        sa.extra_tx = a.extra_tx;
        int whole = 0;
        if ((e = launch_score_tc(sa, ws, a.centroid_bf16, st, n_sm, &whole)) != cudaSuccess) return e;
        if (!whole) {  // thresholds from the merged histograms
            k_tau<<<(unsigned)((a.nq + 7) / 8), 256, 0, st>>>(a.nq, a.P, ws);
            count_launches(1);
            if ((e = cudaGetLastError()) != cudaSuccess) return e;
        }
        if (small) {  // pass 2 from the stored scores
            const unsigned blocks = (unsigned)((nb_total + 255) / 256);
            k_dfilter<<<blocks, 256, 0, st>>>(a.nq, ws);
            count_launches(1);
            if ((e = cudaGetLastError()) != cudaSuccess) return e;
        } else {  // pass 2 on the tensor cores: recompute the same scores, keep those >= tau
            sa.mode = 1;
            sa.store = 0;
            sa.extra_tx = 0;
            if ((e = launch_score_tc(sa, ws, a.centroid_bf16, st, n_sm, nullptr)) != cudaSuccess) return e;
        }
        const int64_t fb = small ? a.nq : (a.nq < (int64_t)n_sm * 2 ? a.nq : (int64_t)n_sm * 2);
        k_fallback<<<(unsigned)fb, 256, 0, st>>>(a.nq, a.centroid_bf16, a.P, ws);
        count_launches(1);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    } else if (tree && tree->n_levels > 0) {
        int64_t B1 = ((int64_t)a.P + 1) / 2;
        if (B1 < a.beam) B1 = a.beam;
        const int CM = (int)pow2_ceil64(2 * B1 + LSA_RUN + 2);
        const int KM = a.beam > a.P ? a.beam : a.P;
        const size_t smt = (size_t)CM * (sizeof(uint64_t) + sizeof(int32_t)) + (size_t)KM * sizeof(int32_t);
        cudaFuncSetAttribute(k_tree_beam, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smt);
        k_tree_beam<<<(unsigned)a.nq, 256, smt, st>>>(a.nq, *tree, a.beam, a.P, CM, ws);
        count_launches(1);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    const int TW = (int)((a.n_blocks + 31) / 32) + 1;
    const int nslot_max = a.P;  // touched blocks <= buckets taken <= P (the cut is within any P buckets)
    const size_t smr = (size_t)ws.cap * (8 + 4) + (size_t)nslot_max * (64 + 4 + 4) + (size_t)TW * 8;
    cudaFuncSetAttribute(k_rank_expand, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smr);
    k_rank_expand<<<(unsigned)a.nq, big_block, smr, st>>>(a.pos, a.members, a.lists, a.lens, a.Lmax, a.k, a.sink,
                                                         a.window, nslot_max, ws.cap, TW, ws);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace lsa
