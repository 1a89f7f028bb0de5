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
// P = ceil((k + sink + window) / 4).  Pass 1 scores every bucket and keeps
// only the maximum of each group of g consecutive buckets (g a power of two
// giving 4P..8P groups).  The P-th largest group maximum is a score of P
// distinct buckets, so it is <= the P-th largest score: every bucket scoring
// at least that value is kept by pass 2, which recomputes the same scores
// bit for bit and appends the passing (score, id) pairs.  A query whose
// candidates overflow their slots is redone exactly (radix select on the
// recomputed scores) by the fallback kernel.  The candidates are then ranked
// by (score desc, id asc) and expanded.
#include "lsa_common.cuh"
#include "lsa_kernels.h"

namespace lsa {

constexpr int SQ = 64;    // queries per score CTA
constexpr int SB = 128;   // buckets per score tile
constexpr int QS = 65;    // padded row (floats)
constexpr int SS = 129;   // padded score row
constexpr int MODE_GMAX = 0;
constexpr int MODE_FILTER = 1;

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
    }
}

// Score of one bucket: fp32 FMA chain over d = 0..63 of the bf16 operands.
// k_score, k_fallback and k_tree_beam all use this exact order.
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

// ---------------------------------------------------------------------------
// Flat passes 1 and 2.  CTA = 64 queries x a chunk of buckets, 128-bucket
// tiles, 256 threads each computing 4 queries x 8 buckets.
template <int MODE>
__global__ void __launch_bounds__(256) k_score(int64_t nq, int64_t nb_total, const uint16_t *__restrict__ cbf,
                                               int64_t chunk, int P, IndexWs ws)
{
    extern __shared__ float sm[];
    float *qf = sm;                    // [64][65]
    float *cf = qf + SQ * QS;          // [128][65]
    float *S = cf + SB * QS;           // [64][129] (pass 1 only)
    __shared__ int Nq[SQ];
    __shared__ int gq[SQ];
    __shared__ float tq[SQ];
    __shared__ int nmax_s;

    const int t = threadIdx.x;
    const int64_t q0 = (int64_t)blockIdx.x * SQ;
    if (t == 0) nmax_s = 0;
    __syncthreads();
    if (t < SQ) {
        int64_t q = q0 + t;
        int N = (q < nq) ? ws.horizon[q] * LSA_NBKT : 0;
        Nq[t] = N;
        gq[t] = group_width(N, P);
        tq[t] = (MODE == MODE_FILTER && q < nq) ? ws.tau[q] : 0.0f;
        atomicMax(&nmax_s, N);
    }
    for (int i = t; i < SQ * LSA_D; i += 256) {
        int r = i >> 6, d = i & 63;
        int64_t q = q0 + r;
        qf[r * QS + d] = (q < nq) ? bf_bits2f(ws.qhat[q * LSA_D + d]) : 0.0f;
    }
    __syncthreads();
    const int64_t b_begin = (int64_t)blockIdx.y * chunk;
    const int64_t b_end = min(b_begin + chunk, (int64_t)nmax_s);
    const int ty = t >> 4, tx = t & 15;

    for (int64_t tile = b_begin; tile < b_end; tile += SB) {
        // centroid tile -> float smem (bf16 rows of 128 B, uint4 loads)
        for (int i = t; i < SB * 8; i += 256) {
            int r = i >> 3, v = i & 7;
            int64_t b = tile + r;
            uint4 w = make_uint4(0, 0, 0, 0);
            if (b < nb_total) w = __ldg(reinterpret_cast<const uint4 *>(cbf + b * LSA_D) + v);
            uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                cf[r * QS + v * 8 + 2 * h] = __uint_as_float(ww[h] << 16);
                cf[r * QS + v * 8 + 2 * h + 1] = __uint_as_float(ww[h] & 0xffff0000u);
            }
        }
        __syncthreads();
        float acc[4][8];
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[r][i] = 0.0f;
#pragma unroll 4
        for (int d = 0; d < LSA_D; ++d) {
            float qv[4], cv[8];
#pragma unroll
            for (int r = 0; r < 4; ++r) qv[r] = qf[(ty * 4 + r) * QS + d];
#pragma unroll
            for (int i = 0; i < 8; ++i) cv[i] = cf[(tx + 16 * i) * QS + d];
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int i = 0; i < 8; ++i) acc[r][i] = fmaf(qv[r], cv[i], acc[r][i]);
        }
        if (MODE == MODE_GMAX) {
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int i = 0; i < 8; ++i) S[(ty * 4 + r) * SS + tx + 16 * i] = acc[r][i];
            __syncthreads();
            const int warp = t >> 5, lane = t & 31;
            for (int qi = warp * 8; qi < warp * 8 + 8; ++qi) {
                const int N = Nq[qi];
                if (tile >= N) continue;  // warp-uniform
                const int g = gq[qi];
                const float NEG = __int_as_float(0xff800000);
                float v[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    int64_t b = tile + lane * 4 + e;
                    v[e] = (b < N) ? S[qi * SS + lane * 4 + e] : NEG;
                }
                float *gm = ws.gmax + (q0 + qi) * ws.gmax_stride;
                if (g == 1) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        int64_t b = tile + lane * 4 + e;
                        if (b < N) gm[b] = v[e];
                    }
                } else if (g == 2) {
#pragma unroll
                    for (int e = 0; e < 4; e += 2) {
                        int64_t b = tile + lane * 4 + e;
                        if (b < N) gm[b >> 1] = fmaxf(v[e], v[e + 1]);
                    }
                } else {
                    float m = fmaxf(fmaxf(v[0], v[1]), fmaxf(v[2], v[3]));
                    for (int s = 1; s < (g >> 2); s <<= 1) m = fmaxf(m, __shfl_xor_sync(LSA_FULL, m, s));
                    int64_t b = tile + lane * 4;
                    if ((lane & ((g >> 2) - 1)) == 0 && b < N) gm[b / g] = m;
                }
            }
        } else {
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const int qi = ty * 4 + r;
                const int N = Nq[qi];
                const float tau = tq[qi];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    int64_t b = tile + tx + 16 * i;
                    if (b < N && acc[r][i] >= tau) {
                        int slot = atomicAdd(ws.cnt + q0 + qi, 1);
                        if (slot < ws.cap) {
                            ws.cand_s[(q0 + qi) * ws.cap + slot] = acc[r][i];
                            ws.cand_id[(q0 + qi) * ws.cap + slot] = (int32_t)b;
                        }
                    }
                }
            }
        }
        __syncthreads();
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
        for (int64_t i = threadIdx.x; i < n; i += blockDim.x) {
            uint32_t u = f2ord(get(i));
            if ((u & mask) == prefix) atomicAdd(&hist[(u >> shift) & 255], 1);
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            int64_t acc = 0;
            int digit = 0;
            for (int d = 255; d >= 0; --d) {
                if (acc + hist[d] >= rem) {
                    digit = d;
                    break;
                }
                acc += hist[d];
            }
            sh[0] = digit;
            sh[1] = (int)(rem - acc);
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
__global__ void __launch_bounds__(256) k_select(int64_t nq, int P, IndexWs ws)
{
    __shared__ int hist[256];
    __shared__ int sh[2];
    const int64_t q = blockIdx.x;
    const int64_t N = (int64_t)ws.horizon[q] * LSA_NBKT;
    const int64_t G = n_groups(N, P);
    if (G <= P) {
        if (threadIdx.x == 0) ws.tau[q] = __int_as_float(0xff800000);
        return;
    }
    const float *gm = ws.gmax + q * ws.gmax_stride;
    uint32_t u = block_select_kth_largest(G, P, [&](int64_t i) { return gm[i]; }, hist, sh);
    if (threadIdx.x == 0) ws.tau[q] = ord2f(u);
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
                keys[i] = rank_key(dot_bf16_row(qf, tv.centroid_bf16 + (off + u) * LSA_D), u);
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

// Rank the candidates of one query and expand them into its index list.
__global__ void __launch_bounds__(256) k_rank_expand(const int64_t *__restrict__ pos, const int32_t *__restrict__ members,
                                                     const int32_t *__restrict__ count, int32_t *__restrict__ lists,
                                                     int32_t *__restrict__ lens, int Lmax, int k, int sink,
                                                     int window, int P, int SM, int FM, IndexWs ws)
{
    extern __shared__ uint64_t rsm[];
    uint64_t *keys = rsm;                                 // [SM]
    int32_t *cum = reinterpret_cast<int32_t *>(keys + SM);  // [P]
    int32_t *far = cum + P;                               // [FM]
    __shared__ int wsum[8];

    const int64_t q = blockIdx.x;
    const int t = threadIdx.x;
    const int64_t p = pos[q];
    const int n = min(ws.cnt[q], ws.cap);
    const int S = (int)pow2_ceil64(n > 0 ? n : 1);
    for (int i = t; i < S; i += blockDim.x)
        keys[i] = (i < n) ? rank_key(ws.cand_s[q * ws.cap + i], ws.cand_id[q * ws.cap + i]) : ~0ull;
    __syncthreads();
    block_bitonic_sort(keys, S);
    const int n_take = min(n, P);
    const int64_t w0 = p - window > 0 ? p - window : 0;
    const int64_t s_end = (int64_t)sink < p + 1 ? (int64_t)sink : p + 1;
    for (int r = t; r < n_take; r += blockDim.x) {
        const int32_t b = rank_key_id(keys[r]);
        const int c = count[b];
        int nn = 0;
        for (int e = 0; e < c; ++e) {
            int64_t m = members[(int64_t)b * LSA_NSLOT + e];
            nn += !(m < s_end || (m >= w0 && m <= p));
        }
        cum[r] = nn;
    }
    __syncthreads();
    block_inclusive_scan(cum, n_take, wsum);
    const int total = n_take > 0 ? cum[n_take - 1] : 0;
    const int nfar = min(k, total);
    for (int r = t; r < n_take; r += blockDim.x) {
        const int prev = r > 0 ? cum[r - 1] : 0;
        if (prev >= nfar) continue;
        const int32_t b = rank_key_id(keys[r]);
        const int c = count[b];
        int idx = prev;
        for (int e = 0; e < c && idx < nfar; ++e) {
            int64_t m = members[(int64_t)b * LSA_NSLOT + e];
            if (!(m < s_end || (m >= w0 && m <= p))) far[idx++] = (int32_t)m;
        }
    }
    const int F = (int)pow2_ceil64(nfar > 0 ? nfar : 1);
    for (int i = nfar + t; i < F; i += blockDim.x) far[i] = 0x7fffffff;
    __syncthreads();
    block_bitonic_sort(far, F);
    const int n_sink = (int)min(s_end, w0);
    const int nwin = (int)(p - w0 + 1);
    const int len = n_sink + nfar + nwin;
    int32_t *out = lists + q * (int64_t)Lmax;
    for (int i = t; i < Lmax; i += blockDim.x) {
        int32_t v;
        if (i < n_sink) v = i;
        else if (i < n_sink + nfar) v = far[i - n_sink];
        else if (i < len) v = (int32_t)(w0 + (i - n_sink - nfar));
        else v = -1;
        out[i] = v;
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
    if (a.mode == 0) {
        if (nb_total > 0) {
            const int64_t qtiles = (a.nq + SQ - 1) / SQ;
            const int64_t tiles = (nb_total + SB - 1) / SB;
            int64_t chunks = ((int64_t)n_sm * 8 + qtiles - 1) / qtiles;
            if (chunks > tiles) chunks = tiles;
            if (chunks < 1) chunks = 1;
            if (chunks > 65535) chunks = 65535;
            const int64_t chunk = ((tiles + chunks - 1) / chunks) * SB;
            chunks = (nb_total + chunk - 1) / chunk;
            const size_t sm1 = sizeof(float) * (SQ * QS + SB * QS + SQ * SS);
            const size_t sm2 = sizeof(float) * (SQ * QS + SB * QS);
            cudaFuncSetAttribute(k_score<MODE_GMAX>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm1);
            cudaFuncSetAttribute(k_score<MODE_FILTER>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm2);
            dim3 grid((unsigned)qtiles, (unsigned)chunks);
            k_score<MODE_GMAX><<<grid, 256, sm1, st>>>(a.nq, nb_total, a.centroid_bf16, chunk, a.P, ws);
            count_launches(1);
            if ((e = cudaGetLastError()) != cudaSuccess) return e;
            k_select<<<(unsigned)a.nq, 256, 0, st>>>(a.nq, a.P, ws);
            count_launches(1);
            if ((e = cudaGetLastError()) != cudaSuccess) return e;
            k_score<MODE_FILTER><<<grid, 256, sm2, st>>>(a.nq, nb_total, a.centroid_bf16, chunk, a.P, ws);
            count_launches(1);
            if ((e = cudaGetLastError()) != cudaSuccess) return e;
            int64_t fb = a.nq < (int64_t)n_sm * 2 ? a.nq : (int64_t)n_sm * 2;
            k_fallback<<<(unsigned)fb, 256, 0, st>>>(a.nq, a.centroid_bf16, a.P, ws);
            count_launches(1);
            if ((e = cudaGetLastError()) != cudaSuccess) return e;
        }
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
    const int SMK = (int)pow2_ceil64(ws.cap);
    const int FM = (int)pow2_ceil64(a.k > 0 ? a.k : 1);
    const size_t smr = (size_t)SMK * sizeof(uint64_t) + (size_t)a.P * sizeof(int32_t) + (size_t)FM * sizeof(int32_t);
    cudaFuncSetAttribute(k_rank_expand, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smr);
    k_rank_expand<<<(unsigned)a.nq, 256, smr, st>>>(a.pos, a.members, a.count, a.lists, a.lens, a.Lmax, a.k, a.sink,
                                                   a.window, a.P, SMK, FM, ws);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace lsa
