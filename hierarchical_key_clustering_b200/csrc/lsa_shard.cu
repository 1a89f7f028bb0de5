// Context-parallel pieces of the LSA path: the KV cache and the bucket cache
// split by token range over ranks, as the pages' end-to-end runs do with
// decode context parallelism over 8 GPUs (zhichai forum post, "Reported
// numbers"; sotaaz blog, "Why 72x in one layer becomes 9x").
//
// Rank s holds the complete blocks [b0_s, b1_s) and their K/V rows.  Every
// query is replicated.  Index: each rank finds a local candidate set that
// holds its own top P buckets (the Flat passes and merge of lsa_index.cu over
// its blocks), the sets are exchanged, and every rank takes the same global
// top P from their union: a bucket among the global top P is among the top P
// of the rank that owns it, so the union holds it with its exact score.  The
// same expansion then gives every rank the identical list.  Attention: each
// rank attends over the list entries it owns and the partial results are
// combined by log-sum-exp.
#include "lsa_common.cuh"
#include "lsa_kernels.h"

namespace lsa {

// ---------------------------------------------------------------------------
// A rank's merged local set (one-bucket entries, local bucket ids) into its
// exchange block with global bucket ids (g0 = 64 x the rank's first block).
__global__ void k_shard_pack(IndexWs m, int64_t nq, int64_t g0, int32_t *__restrict__ xcnt,
                             int2 *__restrict__ xent)
{
    pdl_wait();
    pdl_release();
    const int64_t q = blockIdx.x;
    const int n = m.cnt[q];
    if (threadIdx.x == 0) xcnt[q] = n;
    const float4 *c4 = reinterpret_cast<const float4 *>(m.cand4) + q * m.cap;
    const int32_t *cg = m.cand_g + q * m.cap;
    for (int i = threadIdx.x; i < n; i += blockDim.x)
        xent[q * m.cap + i] = make_int2(__float_as_int(c4[i].x), (int32_t)(cg[i] + g0));
}

cudaError_t launch_shard_pack(const IndexWs &m, int64_t nq, int64_t g0, void *xchg, cudaStream_t st)
{
    if (nq <= 0) return cudaSuccess;
    int32_t *xcnt = reinterpret_cast<int32_t *>(xchg);
    int2 *xent = reinterpret_cast<int2 *>(reinterpret_cast<char *>(xchg) + ((nq * 4 + 255) / 256) * 256);
    const int kt = kt_begin("k_shard_pack", st);
    k_shard_pack<<<(unsigned)nq, 256, 0, st>>>(m, nq, g0, xcnt, xent);
    kt_end(kt, st);
    count_launches(1);
    return cudaGetLastError();
}

// Histogram bin of a value over [lo, lo + 256 / scale] (monotone in v): the
// same rounded operations in the counting and the keeping pass.
__device__ __forceinline__ int merge_bin_shard(float v, float lo, float scale)
{
    return min(255, max(0, __float2int_rz(__fmul_rn(__fsub_rn(v, lo), scale))));
}

// ---------------------------------------------------------------------------
// Global top P of the union of the shards' sets (disjoint bucket ids, exact
// scores).  One CTA per query stages the union in shared memory when it fits
// (up to cap_smem entries; every access otherwise goes to the exchange
// blocks in global memory); all of it is kept when it fits the expansion's
// slots, else every bucket from the histogram bin holding the P-th best
// value up when those fit, else the buckets above the P-th score and, at
// that score, the ties with the lowest ids up to P.
constexpr int SM_THREADS = 512;
constexpr int SM_MAX_SHARDS = 32;
constexpr int64_t SM_SMEM_MAX = 200 * 1024;  // staged union, bytes

__global__ void __launch_bounds__(SM_THREADS) k_shard_merge(const int32_t *__restrict__ xcnt_all,
                                                            const int2 *__restrict__ xent_all, int n_shards,
                                                            int64_t nq, int64_t xstride, int slots, int P,
                                                            int cap_smem, IndexWs m)
{
    pdl_wait();
    pdl_release();
    extern __shared__ uint2 um[];  // [cap_smem] (ordered score, bucket id)
    __shared__ int hist[256];
    __shared__ int sh[4];
    __shared__ int s_off[SM_MAX_SHARDS + 1];
    __shared__ int s_out, s_bstar, s_keep;
    __shared__ uint32_t s_vmin, s_vmax;
    const int64_t q = blockIdx.x;
    const int t = threadIdx.x;
    const float NEG = __int_as_float(0xff800000);
    const int KC = m.cap;
    if (t == 0) {
        int o = 0;
        for (int s = 0; s < n_shards; ++s) {
            s_off[s] = o;
            o += min(xcnt_all[s * xstride / 4 + q], slots);
        }
        s_off[n_shards] = o;
        s_out = 0;
    }
    __syncthreads();
    const int n = s_off[n_shards];
    const bool staged = n <= cap_smem;  // block-uniform
    auto from_global = [&](int i) {
        int s = 0;
        while (i >= s_off[s + 1]) ++s;
        const int2 e = *reinterpret_cast<const int2 *>(reinterpret_cast<const char *>(xent_all) + s * xstride +
                                                       (q * slots + (i - s_off[s])) * 8);
        return make_uint2(f2ord(__int_as_float(e.x)), (uint32_t)e.y);
    };
    auto entry = [&](int i) { return staged ? um[i] : from_global(i); };
    if (staged) {
        for (int i = t; i < n; i += SM_THREADS) um[i] = from_global(i);
        __syncthreads();
    }
    float4 *o4 = reinterpret_cast<float4 *>(m.cand4) + q * KC;
    int32_t *og = m.cand_g + q * KC;
    if (n <= KC) {  // everything fits: the expansion ranks it
        for (int i = t; i < n; i += SM_THREADS) {
            const uint2 u = entry(i);
            o4[i] = make_float4(ord2f(u.x), NEG, NEG, NEG);
            og[i] = (int32_t)u.y;
        }
        if (t == 0) s_out = n;
    } else {
        // one 256-bin histogram over the union's [min, max]: every bucket
        // from the bin holding the P-th best value up holds the top P, and
        // is kept when it fits the expansion's slots
        uint32_t vmin = ~0u, vmax = 0u;
        for (int i = t; i < n; i += SM_THREADS) {
            const uint32_t v = entry(i).x;
            vmin = min(vmin, v);
            vmax = max(vmax, v);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            vmin = min(vmin, __shfl_xor_sync(LSA_FULL, vmin, o));
            vmax = max(vmax, __shfl_xor_sync(LSA_FULL, vmax, o));
        }
        if (t == 0) s_vmin = ~0u, s_vmax = 0u;
        for (int i = t; i < 256; i += SM_THREADS) hist[i] = 0;
        __syncthreads();
        if ((t & 31) == 0) {
            atomicMin(&s_vmin, vmin);
            atomicMax(&s_vmax, vmax);
        }
        __syncthreads();
        const float lo = ord2f(s_vmin), hi = ord2f(s_vmax);
        const float scale = hi > lo ? 256.0f / (hi - lo) : 0.0f;
        const int n_round = (n + SM_THREADS - 1) / SM_THREADS * SM_THREADS;
        for (int i = t; i < n_round; i += SM_THREADS) {
            const int bin = i < n ? merge_bin_shard(ord2f(entry(i).x), lo, scale) : -1;
            const unsigned peers = __match_any_sync(LSA_FULL, bin);
            if (bin >= 0 && (t & 31) == __ffs(peers) - 1) atomicAdd(&hist[bin], __popc(peers));
        }
        __syncthreads();
        if (t == 0) {
            int acc = 0, d = 255;
            for (; d > 0; --d) {
                if (acc + hist[d] >= P) break;
                acc += hist[d];
            }
            s_bstar = d;
            s_keep = acc + hist[d];
        }
        __syncthreads();
        if (s_keep <= KC) {  // block-uniform
            const int bstar = s_bstar;
            for (int i = t; i < n; i += SM_THREADS) {
                const uint2 u = entry(i);
                if (merge_bin_shard(ord2f(u.x), lo, scale) >= bstar) {
                    const int j = atomicAdd(&s_out, 1);
                    o4[j] = make_float4(ord2f(u.x), NEG, NEG, NEG);
                    og[j] = (int32_t)u.y;
                }
            }
            __syncthreads();
            if (t == 0) {
                m.cnt[q] = s_out;
                m.tau[q] = NEG;
                m.horizon[q] = 0;
            }
            return;
        }
        const uint32_t cut = block_select_ord(n, P, [&](int64_t i) { return entry((int)i).x; }, hist, sh);
        int above = 0, ties = 0;
        for (int i = t; i < n; i += SM_THREADS) {
            const uint32_t v = entry(i).x;
            above += v > cut;
            ties += v == cut;
        }
        __syncthreads();
        if (t == 0) sh[2] = 0, sh[3] = 0;
        __syncthreads();
        atomicAdd(&sh[2], above);
        atomicAdd(&sh[3], ties);
        __syncthreads();
        const int n_above = sh[2], n_ties = sh[3];
        // ties at the cut: all of them when they fit, else the lowest ids
        uint32_t idcut = 0xffffffffu;
        if (n_above + n_ties > KC) {
            const int need = P - n_above;
            // the need-th smallest id among the ties = the need-th largest of ~id
            idcut = ~block_select_ord(n, need, [&](int64_t i) {
                const uint2 u = entry((int)i);
                return u.x == cut ? ~u.y : 0u;
            }, hist, sh);
        }
        for (int i = t; i < n; i += SM_THREADS) {
            const uint2 u = entry(i);
            if (u.x > cut || (u.x == cut && u.y <= idcut)) {
                const int j = atomicAdd(&s_out, 1);
                o4[j] = make_float4(ord2f(u.x), NEG, NEG, NEG);
                og[j] = (int32_t)u.y;
            }
        }
    }
    __syncthreads();
    if (t == 0) {
        m.cnt[q] = s_out;
        m.tau[q] = NEG;
        m.horizon[q] = 0;  // read only by the expansion's exact path, which a merged set never takes
    }
}

cudaError_t launch_shard_merge(const void *xchg_all, int n_shards, int64_t nq, int slots, int P, const IndexWs &m,
                               cudaStream_t st)
{
    if (nq <= 0) return cudaSuccess;
    const int64_t cnt_bytes = ((nq * 4 + 255) / 256) * 256;
    const int64_t xstride = cnt_bytes + nq * slots * 8;  // one rank's exchange block
    const int32_t *xcnt = reinterpret_cast<const int32_t *>(xchg_all);
    const int2 *xent = reinterpret_cast<const int2 *>(reinterpret_cast<const char *>(xchg_all) + cnt_bytes);
    // the union staged in shared memory when it fits (each shard lists about
    // 1.1 P of its slots), else read from the exchange blocks
    const int cap_smem = (int)min((int64_t)n_shards * slots, (int64_t)(SM_SMEM_MAX / 8));
    const size_t smem = (size_t)cap_smem * 8;
    cudaFuncSetAttribute(k_shard_merge, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    const int kt = kt_begin("k_shard_merge", st);
    k_shard_merge<<<(unsigned)nq, SM_THREADS, smem, st>>>(xcnt, xent, n_shards, nq, xstride, slots, P, cap_smem, m);
    kt_end(kt, st);
    count_launches(1);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// The entries of each list in [t0, t1), shifted to the rank's K/V rows.  One
// warp per query; the order is kept, the rest of the row is not written.
__global__ void __launch_bounds__(256) k_local_lists(const int32_t *__restrict__ lists,
                                                     const int32_t *__restrict__ lens, int64_t nq, int32_t Lmax,
                                                     int64_t t0, int64_t t1, int32_t *__restrict__ out_lists,
                                                     int32_t *__restrict__ out_lens)
{
    pdl_wait();
    pdl_release();
    const int lane = threadIdx.x & 31;
    const int64_t q = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (q >= nq) return;
    const int32_t *in = lists + q * Lmax;
    int32_t *out = out_lists + q * Lmax;
    const int len = min(lens[q], Lmax);
    int n = 0;
    for (int i0 = 0; i0 < len; i0 += 32) {
        const int i = i0 + lane;
        const int64_t v = i < len ? in[i] : -1;
        const bool keep = v >= t0 && v < t1;
        const unsigned bal = __ballot_sync(LSA_FULL, keep);
        if (keep) out[n + __popc(bal & ((1u << lane) - 1u))] = (int32_t)(v - t0);
        n += __popc(bal);
    }
    if (lane == 0) out_lens[q] = n;
}

cudaError_t launch_local_lists(const int32_t *lists, const int32_t *lens, int64_t nq, int32_t Lmax, int64_t t0,
                               int64_t t1, int32_t *out_lists, int32_t *out_lens, cudaStream_t st)
{
    if (nq <= 0) return cudaSuccess;
    const int kt = kt_begin("k_local_lists", st);
    k_local_lists<<<(unsigned)((nq + 7) / 8), 256, 0, st>>>(lists, lens, nq, Lmax, t0, t1, out_lists, out_lens);
    kt_end(kt, st);
    count_launches(1);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// A rank's member table and counts into the replicated global tables: bucket
// g of the rank is global bucket g0 + g, its member positions move by pos0.
__global__ void k_publish_members(const int32_t *__restrict__ members, const int32_t *__restrict__ count, int64_t nb,
                                  int64_t g0, int64_t pos0, int32_t *__restrict__ members_out,
                                  int32_t *__restrict__ count_out)
{
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= nb * LSA_NSLOT) return;
    const int32_t m = members[i];
    members_out[g0 * LSA_NSLOT + i] = m >= 0 ? (int32_t)(m + pos0) : -1;
    if (i % LSA_NSLOT == 0) count_out[g0 + i / LSA_NSLOT] = count[i / LSA_NSLOT];
}

cudaError_t launch_publish_members(const int32_t *members, const int32_t *count, int64_t nb, int64_t g0,
                                   int64_t pos0, int32_t *members_out, int32_t *count_out, cudaStream_t st)
{
    if (nb <= 0) return cudaSuccess;
    const int kt = kt_begin("k_publish_members", st);
    k_publish_members<<<(unsigned)((nb * LSA_NSLOT + 255) / 256), 256, 0, st>>>(members, count, nb, g0, pos0,
                                                                               members_out, count_out);
    kt_end(kt, st);
    count_launches(1);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Log-sum-exp combination of the ranks' attention outputs: O_s normalised
// over rank s's keys with log-sum-exp lse_s (-inf for a rank with none), so
// O = sum_s exp(lse_s - M) O_s / sum_s exp(lse_s - M), lse = M + log(that sum).
// One warp per (query, head), 4 dims per lane.
__global__ void __launch_bounds__(256) k_combine_parts(const uint16_t *__restrict__ O_parts,
                                                       const float *__restrict__ lse_parts, int n_parts, int64_t units,
                                                       uint16_t *__restrict__ O, float *__restrict__ lse)
{
    pdl_wait();
    pdl_release();
    const int lane = threadIdx.x & 31;
    const int64_t u = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (u >= units) return;
    const float NEG = __int_as_float(0xff800000);
    float M = NEG;
    for (int s = 0; s < n_parts; ++s) M = fmaxf(M, lse_parts[s * units + u]);
    float acc[4] = {0.f, 0.f, 0.f, 0.f}, L = 0.0f;
    for (int s = 0; s < n_parts; ++s) {
        const float ls = lse_parts[s * units + u];
        if (!(ls > NEG)) continue;  // no keys on this rank
        const float w = expf(ls - M);
        L += w;
        const uint2 v = *reinterpret_cast<const uint2 *>(O_parts + (s * units + u) * LSA_HEAD + lane * 4);
        acc[0] += w * __uint_as_float(v.x << 16);
        acc[1] += w * __uint_as_float(v.x & 0xffff0000u);
        acc[2] += w * __uint_as_float(v.y << 16);
        acc[3] += w * __uint_as_float(v.y & 0xffff0000u);
    }
    const float inv = L > 0.0f ? 1.0f / L : 0.0f;
    __nv_bfloat16 b[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) b[e] = __float2bfloat16_rn(acc[e] * inv);
    uint2 w;
    w.x = (uint32_t)*reinterpret_cast<uint16_t *>(&b[0]) | ((uint32_t)*reinterpret_cast<uint16_t *>(&b[1]) << 16);
    w.y = (uint32_t)*reinterpret_cast<uint16_t *>(&b[2]) | ((uint32_t)*reinterpret_cast<uint16_t *>(&b[3]) << 16);
    *reinterpret_cast<uint2 *>(O + u * LSA_HEAD + lane * 4) = w;
    if (lane == 0 && lse) lse[u] = L > 0.0f ? M + logf(L) : NEG;
}

cudaError_t launch_combine_parts(const uint16_t *O_parts, const float *lse_parts, int n_parts, int64_t nq, int Hq,
                                 uint16_t *O, float *lse, cudaStream_t st)
{
    const int64_t units = nq * Hq;
    if (units <= 0) return cudaSuccess;
    const int kt = kt_begin("k_combine_parts", st);
    k_combine_parts<<<(unsigned)((units + 7) / 8), 256, 0, st>>>(O_parts, lse_parts, n_parts, units, O, lse);
    kt_end(kt, st);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace lsa
