// Near-set attention tiles on the 5th-generation tensor cores (sm_100a).
//
// Method: Latent Sparse Attention pages -- learnaivisually explainer, "What
// one query actually does": every head of a query attends, with a plain
// softmax, over the query's list (sink, selected keys, window).  The window
// [p - 512, p] and the sinks of consecutive queries are almost the same
// keys, so a tile of NEAR_ROWS / G consecutive queries takes the union of
// their near keys once per KV head (plans from k_near_plan) and k_attn merges
// the partial result with the rest of each list.
//
// One CTA per (tile, KV head); the tile's 128 query-head rows (query r / G,
// head r % G) are the MMA M, so one pass reads each key once for all of them:
//   warp 0     TMA producer: the Q rows once (two 64-dim boxes, 128-byte
//              swizzle), then per 64-key chunk K and V (2-stage rings each);
//              in a chunk with fewer than 64 keys it zeroes the V rows past
//              them once they land (they are not the tile's keys);
//   warp 1     allocates 256 TMEM columns (two 64-column score buffers, 128
//              columns of O); one thread issues S = Q K^T (M 128, N 64, K 128)
//              per chunk and, one chunk behind, O += P V (M 128, N 128, K 64)
//              with P read from tensor memory and V in place from shared
//              memory as an MN-major operand;
//   warps 2-5  one row each (its TMEM lane): the row's keys masked, the
//              online softmax in log2 units, P (bf16 pairs) written over the
//              first 32 columns of the row's score buffer.  O is rescaled in
//              TMEM only when a row's maximum rises more than 8 (2^8) above
//              the one its O and sum refer to, so P stays <= 256 and the
//              rescale is rare.
// Output: per row the unnormalised O, its reference maximum and the sum, as
// the warp-level near kernel writes them.  Every wait is bounded: one that
// runs out sets the device error word and the CTA's abort flag, the producer
// waits (bounded) for its copies in flight and TMEM is freed.
#include <cuda_bf16.h>

#include "lsa_common.cuh"
#include "lsa_kernels.h"
#include "lsa_tc.cuh"

namespace lsa {

namespace {

constexpr int NT_KC = 64;                               // keys per chunk
constexpr int NT_KST = 2;                               // K and V ring stages
constexpr int NT_THREADS = 192;
constexpr uint32_t NT_Q_BYTES = NEAR_ROWS * 128 * 2;    // 32 KB: two 64-dim blocks of 128 rows
constexpr uint32_t NT_K_BYTES = NT_KC * 128 * 2;        // 16 KB: two 64-dim blocks of 64 key rows
constexpr uint32_t NT_V_BYTES = NT_KC * 128 * 2;        // 16 KB: same layout
constexpr uint32_t NT_TMEM_COLS = 256;
constexpr uint32_t NT_IDESC_S = tc::idesc_bf16(NEAR_ROWS, NT_KC);
constexpr uint32_t NT_IDESC_PV = tc::idesc_bf16(NEAR_ROWS, 128) | (1u << 16);  // B (V) MN-major
constexpr float NT_RESCALE = 8.0f;                      // log2 units a row's max may rise before O is rescaled
constexpr float NT_LOG2E = 1.4426950408889634f;

struct NearTcCtl {
    uint64_t q_full, pv_ready, pv_done, o_full, mma_done;
    uint64_t k_full[NT_KST], k_empty[NT_KST], v_full[NT_KST], v_ready[NT_KST], v_empty[NT_KST], s_full[2], s_empty[2];
    uint32_t tmem_base;
    int abort;
};
constexpr size_t NT_SMEM = NT_Q_BYTES + NT_KST * (NT_K_BYTES + NT_V_BYTES) + sizeof(NearTcCtl) + 1024;

__device__ int g_near_error = 0;

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

__global__ void __launch_bounds__(NT_THREADS, 2)
    k_attn_near_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, AttnArgs a)
{
    extern __shared__ __align__(1024) uint8_t nt_raw[];
    uint8_t *sQ = nt_raw + ((1024u - (tc::smem_u32(nt_raw) & 1023u)) & 1023u);
    uint8_t *sK = sQ + NT_Q_BYTES;
    uint8_t *sV = sK + NT_KST * NT_K_BYTES;
    NearTcCtl *cs = reinterpret_cast<NearTcCtl *>(sV + NT_KST * NT_V_BYTES);
    const int4 tile = a.near_tile[blockIdx.x];
    if (!tile.x) return;  // uniform, before any barrier or allocation
    const int G = a.Hq / a.Hkv;
    const int QT = near_tile_queries(G);
    const int g = blockIdx.y;
    const int64_t q0 = (int64_t)blockIdx.x * QT;
    const int nt_q = (int)min((int64_t)QT, a.nq - q0);
    const int lo = tile.z, smax = tile.w, hi = tile.y + nt_q - 1;
    const int nband = (hi - lo + NT_KC) / NT_KC;
    const int nch = (smax > 0 ? 1 : 0) + nband;  // the sink chunk first, then the band
    auto chunk_first = [&](int ch) { return smax > 0 ? (ch == 0 ? 0 : lo + (ch - 1) * NT_KC) : lo + ch * NT_KC; };
    auto chunk_last = [&](int ch) {
        return (smax > 0 && ch == 0) ? smax - 1 : min(hi, chunk_first(ch) + NT_KC - 1);
    };
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    auto bar = [&](uint64_t &b) { return tc::smem_u32(&b); };

    if (threadIdx.x == 0) {
        cs->abort = 0;
        tc::mbar_init(bar(cs->q_full), 1);
        tc::mbar_init(bar(cs->pv_ready), 4);
        tc::mbar_init(bar(cs->pv_done), 1);
        tc::mbar_init(bar(cs->o_full), 1);
        tc::mbar_init(bar(cs->mma_done), 1);
        for (int s = 0; s < NT_KST; ++s) {
            tc::mbar_init(bar(cs->k_full[s]), 1);
            tc::mbar_init(bar(cs->k_empty[s]), 1);
            tc::mbar_init(bar(cs->v_full[s]), 1);
            tc::mbar_init(bar(cs->v_ready[s]), 1);
            tc::mbar_init(bar(cs->v_empty[s]), 1);
        }
        for (int b = 0; b < 2; ++b) {
            tc::mbar_init(bar(cs->s_full[b]), 1);
            tc::mbar_init(bar(cs->s_empty[b]), 1);
        }
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    __syncthreads();
    if (warp == 1) tc::tmem_alloc(tc::smem_u32(&cs->tmem_base), NT_TMEM_COLS);
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = cs->tmem_base;
    volatile int *abort = &cs->abort;
    const uint32_t wl = a.wait_limit;
    int *err = &g_near_error;
    const float NEG = __int_as_float(0xff800000);

    int k_issued = 0, v_issued = 0;  // the producer's copies, for the abort drain
    if (warp == 0) {  // lane 0 issues the copies; the warp zeroes V rows past a chunk's keys
        if (lane == 0) {
            asm volatile("prefetch.tensormap [%0];\n" ::"l"(&tmQ) : "memory");
            asm volatile("prefetch.tensormap [%0];\n" ::"l"(&tmK) : "memory");
            asm volatile("prefetch.tensormap [%0];\n" ::"l"(&tmV) : "memory");
            tc::mbar_expect_tx(bar(cs->q_full), NT_Q_BYTES);
            tc::tma_load_3d(tc::smem_u32(sQ), &tmQ, 0, g * G, (int)q0, bar(cs->q_full));
            tc::tma_load_3d(tc::smem_u32(sQ + NT_Q_BYTES / 2), &tmQ, 64, g * G, (int)q0, bar(cs->q_full));
        }
        // K of chunk j once the S of chunk j - 2 has read its stage, V of
        // chunk j once the P V of chunk j - 2 has read its stage
        auto load_k = [&](int j) {
            const int s = j % NT_KST;
            if (j >= NT_KST && !tc::wait_bounded_sleep(bar(cs->k_empty[s]), (uint32_t)(((j / NT_KST) - 1) & 1), wl, abort, err))
                return false;
            const uint32_t dk = tc::smem_u32(sK + s * NT_K_BYTES);
            tc::mbar_expect_tx(bar(cs->k_full[s]), NT_K_BYTES);
            tc::tma_load_3d(dk, &tmK, 0, g, chunk_first(j), bar(cs->k_full[s]));
            tc::tma_load_3d(dk + NT_K_BYTES / 2, &tmK, 64, g, chunk_first(j), bar(cs->k_full[s]));
            ++k_issued;
            return true;
        };
        auto load_v = [&](int j) {
            const int s = j % NT_KST;
            if (j >= NT_KST && !tc::wait_bounded_sleep(bar(cs->v_empty[s]), (uint32_t)(((j / NT_KST) - 1) & 1), wl, abort, err))
                return false;
            const uint32_t dv = tc::smem_u32(sV + s * NT_V_BYTES);
            tc::mbar_expect_tx(bar(cs->v_full[s]), NT_V_BYTES);
            tc::tma_load_3d(dv, &tmV, 0, g, chunk_first(j), bar(cs->v_full[s]));
            tc::tma_load_3d(dv + NT_V_BYTES / 2, &tmV, 64, g, chunk_first(j), bar(cs->v_full[s]));
            ++v_issued;
            return true;
        };
        // chunk j's copies are issued before chunk j - 1's tail is handled, so
        // that the wait for those rows to land does not hold back the next copies
        for (int j = 0; j <= nch; ++j) {
            if (j < nch) {
                int okl = 1;
                if (lane == 0) okl = load_k(j) && load_v(j);
                if (!__shfl_sync(LSA_FULL, okl, 0)) break;
            }
            if (j == 0) continue;
            const int c = j - 1, s = c % NT_KST, nvalid = chunk_last(c) - chunk_first(c) + 1;
            if (nvalid < NT_KC) {
                // The box also brought the rows past the chunk's last key: not
                // the tile's keys, possibly rows nothing has written yet.  Their
                // scores are masked, but P = 0 times a NaN row is still NaN, so
                // the V rows are zeroed once they land (the stage's next copy is
                // not issued yet, so the phase waited for is unambiguous).
                int okw = 1;
                if (lane == 0)
                    okw = tc::wait_bounded_sleep(bar(cs->v_full[s]), (uint32_t)((c / NT_KST) & 1), wl, abort, err);
                if (!__shfl_sync(LSA_FULL, okw, 0)) break;
                uint8_t *dv = sV + s * NT_V_BYTES;
                const int n16 = (NT_KC - nvalid) * 8;  // 16-byte pieces of the tail rows per 64-dim box
                for (int t = lane; t < 2 * n16; t += 32) {
                    const int box = t / n16, piece = t - box * n16;
                    *reinterpret_cast<uint4 *>(dv + box * (NT_V_BYTES / 2) + nvalid * 128 + piece * 16) =
                        make_uint4(0u, 0u, 0u, 0u);
                }
                tc::fence_proxy_async_smem();
                __syncwarp();
            }
            if (lane == 0) tc::mbar_arrive(bar(cs->v_ready[s]));
        }
    } else if (warp == 1 && lane == 0) {
        auto issue_pv = [&](int c) {
            const int s = c % NT_KST, b = c & 1;
            if (!tc::wait_bounded_sleep(bar(cs->pv_ready), (uint32_t)(c & 1), wl, abort, err)) return false;
            if (!tc::wait_bounded_sleep(bar(cs->v_full[s]), (uint32_t)((c / NT_KST) & 1), wl, abort, err)) return false;
            if (!tc::wait_bounded_sleep(bar(cs->v_ready[s]), (uint32_t)((c / NT_KST) & 1), wl, abort, err)) return false;
            tc::fence_after();
            // P from the first 32 columns of score buffer b (16 keys = 8 columns per
            // instruction); the V chunk as the MN-major B operand: 64-dim halves
            // 8 KB apart (the two TMA boxes), 8-key groups 1 KB apart
            const uint32_t vb = tc::smem_u32(sV + s * NT_V_BYTES);
#pragma unroll
            for (int kk = 0; kk < NT_KC / 16; ++kk)
                tc::mma_bf16_ts(tmem + 128, tmem + b * NT_KC + kk * 8, tc::smem_desc_mn(vb + kk * 2048, NT_V_BYTES / 2, 1024),
                                NT_IDESC_PV, (c > 0 || kk > 0) ? 1u : 0u);
            tc::mma_commit(bar(cs->v_empty[s]));
            tc::mma_commit(bar(cs->s_empty[b]));  // score buffer b (and the P in it) free again
            tc::mma_commit(bar(cs->pv_done));
            return true;
        };
        bool ok = tc::wait_bounded_sleep(bar(cs->q_full), 0, wl, abort, err);
        for (int i = 0; ok && i < nch; ++i) {
            const int s = i % NT_KST, b = i & 1;
            if (!tc::wait_bounded_sleep(bar(cs->k_full[s]), (uint32_t)((i / NT_KST) & 1), wl, abort, err)) {
                ok = false;
                break;
            }
            if (i >= 2 && !tc::wait_bounded_sleep(bar(cs->s_empty[b]), (uint32_t)(((i >> 1) - 1) & 1), wl, abort, err)) {
                ok = false;
                break;
            }
            tc::fence_after();
            const uint32_t ka = tc::smem_u32(sQ), kbase = tc::smem_u32(sK + s * NT_K_BYTES);
#pragma unroll
            for (int kb = 0; kb < 2; ++kb)
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    tc::mma_bf16(tmem + b * NT_KC, tc::smem_desc(ka + kb * (NT_Q_BYTES / 2) + kk * 32),
                                 tc::smem_desc(kbase + kb * (NT_K_BYTES / 2) + kk * 32), NT_IDESC_S,
                                 (kb | kk) ? 1u : 0u);
            tc::mma_commit(bar(cs->k_empty[s]));
            tc::mma_commit(bar(cs->s_full[b]));
            // the previous chunk's P V after this chunk's S, so that its softmax overlaps this MMA
            if (i >= 1 && !issue_pv(i - 1)) {
                ok = false;
                break;
            }
        }
        if (ok && issue_pv(nch - 1)) tc::mma_commit(bar(cs->o_full));
    } else if (warp >= 2) {
        const int quad = warp & 3, r = quad * 32 + lane;
        const uint32_t trow = tmem + ((uint32_t)(quad * 32) << 16);
        const int qi = r / G, h = r % G;
        const bool valid = qi < nt_q;
        const int2 pl = valid ? a.near_plan[q0 + qi] : make_int2(0, 0);
        const int pr = tile.y + qi, lr = pr - pl.y + 1, sr = pl.x;  // the row's band [lr, pr] and sinks [0, sr)
        const float sl2 = a.scale * NT_LOG2E;
        float m = NEG, l = 0.0f;  // the reference maximum of O and l, and the sum
        bool ok = true;
        for (int i = 0; i < nch; ++i) {
            const int b = i & 1;
            ok = __all_sync(LSA_FULL, tc::wait_bounded_sleep(bar(cs->s_full[b]), (uint32_t)((i >> 1) & 1), wl, abort, err));
            if (!ok) break;
            tc::fence_after();
            float v[NT_KC];
            tc::tmem_ld32_nowait(trow + b * NT_KC, v);
            tc::tmem_ld32_nowait(trow + b * NT_KC + 32, v + 32);
            tc::tmem_wait_ld();
            // the row's keys in this chunk as a column range [ca, cb]
            const int k0 = chunk_first(i), k1 = chunk_last(i);
            int ca = 1, cb = 0;  // empty
            if (valid) {
                if (smax > 0 && i == 0) {
                    ca = 0;
                    cb = min(sr - 1, k1) - k0;
                } else {
                    ca = max(lr, k0) - k0;
                    cb = min(pr, k1) - k0;
                }
            }
            if (!__all_sync(LSA_FULL, ca == 0 && cb >= NT_KC - 1)) {  // some row has masked columns
#pragma unroll
                for (int j = 0; j < NT_KC; ++j) v[j] = (j >= ca && j <= cb) ? v[j] : NEG;
            }
            // row maximum of the raw scores by a tree (the scale is positive)
            float t[NT_KC / 2];
#pragma unroll
            for (int j = 0; j < NT_KC / 2; ++j) t[j] = fmaxf(v[j], v[j + NT_KC / 2]);
#pragma unroll
            for (int w = NT_KC / 4; w >= 1; w >>= 1)
#pragma unroll
                for (int j = 0; j < w; ++j) t[j] = fmaxf(t[j], t[j + w]);
            const float mx = t[0] > NEG ? t[0] * sl2 : NEG;
            // the reference moves to a new maximum only when the row had none
            // yet or it rose more than NT_RESCALE; then O and l are scaled
            float alpha = 1.0f;
            if (mx > NEG && (m == NEG || mx > m + NT_RESCALE)) {
                if (m != NEG) alpha = exp2f(m - mx);
                m = mx;
            }
            float pk[NT_KC / 2];  // bf16 pairs, as 32-bit columns
            float rs4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
            const float mneg = m > NEG ? -m : 0.0f;
#pragma unroll
            for (int j = 0; j < NT_KC; j += 2) {
                // masked columns hold -inf, so exp2 gives 0 there
                const float p0 = exp2f(fmaf(v[j], sl2, mneg));
                const float p1 = exp2f(fmaf(v[j + 1], sl2, mneg));
                rs4[(j >> 1) & 3] += p0 + p1;
                pk[j >> 1] = __uint_as_float(pack_bf16x2(p0, p1));
            }
            const float rs = (rs4[0] + rs4[1]) + (rs4[2] + rs4[3]);
            l = l * alpha + rs;
            // the previous P V is waited for at every chunk, not only before a
            // rescale: a waiter that skipped phases could no longer tell them
            // apart by parity.  Rare: a row's reference maximum moved, and this
            // warp's O rows are rescaled in TMEM.
            if (i >= 1) {
                ok = __all_sync(LSA_FULL, tc::wait_bounded_sleep(bar(cs->pv_done), (uint32_t)((i - 1) & 1), wl, abort, err));
                if (!ok) break;
                tc::fence_after();
            }
            if (i >= 1 && __any_sync(LSA_FULL, alpha != 1.0f)) {
#pragma unroll
                for (int cb = 0; cb < 4; ++cb) {
                    float o[32];
                    tc::tmem_ld32_nowait(trow + 128 + cb * 32, o);
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 32; ++j) o[j] *= alpha;
                    tc::tmem_st32(trow + 128 + cb * 32, o);
                }
            }
            tc::tmem_st32(trow + b * NT_KC, pk);  // P over the scores just read
            tc::tmem_wait_st();
            tc::fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(bar(cs->pv_ready));
        }
        if (ok) ok = __all_sync(LSA_FULL, tc::wait_bounded_sleep(bar(cs->o_full), 0, wl, abort, err));
        if (ok) {
            tc::fence_after();
            const int64_t row = (q0 + qi) * a.Hq + (int64_t)g * G + h;
            float *po = a.near_o + row * LSA_HEAD;
#pragma unroll
            for (int cb = 0; cb < 4; ++cb) {
                float o[32];
                tc::tmem_ld32_nowait(trow + 128 + cb * 32, o);
                tc::tmem_wait_ld();
                if (valid)
#pragma unroll
                    for (int j = 0; j < 32; j += 4)
                        *reinterpret_cast<float4 *>(po + cb * 32 + j) = make_float4(o[j], o[j + 1], o[j + 2], o[j + 3]);
            }
            if (valid) *reinterpret_cast<float2 *>(a.near_ml + row * 2) = make_float2(m, l);
        }
    }
    if (warp == 0 && lane == 0 && *abort) {
        // copies that may still be in flight: the last NT_KST K and V chunks
        volatile int dummy = 0;
        for (int i = max(0, k_issued - NT_KST); i < k_issued; ++i)
            tc::wait_bounded(bar(cs->k_full[i % NT_KST]), (uint32_t)((i / NT_KST) & 1), wl, &dummy, err);
        for (int i = max(0, v_issued - NT_KST); i < v_issued; ++i)
            tc::wait_bounded(bar(cs->v_full[i % NT_KST]), (uint32_t)((i / NT_KST) & 1), wl, &dummy, err);
        tc::wait_bounded(bar(cs->q_full), 0, wl, &dummy, err);
    }
    if (warp == 1 && lane == 0) {  // every MMA issued has finished before TMEM is freed
        volatile int dummy = 0;
        tc::mma_commit(bar(cs->mma_done));
        tc::wait_bounded(bar(cs->mma_done), 0, wl, &dummy, err);
    }
    tc::fence_before();
    __syncthreads();
    if (warp == 1) {
        tc::fence_after();
        tc::tmem_dealloc(tmem, NT_TMEM_COLS);
    }
}

// Rows of 128 bf16 ([outer][mid][128], 256-byte rows), 128B swizzle, box
// {64, box_mid, box_outer}; coordinates past the ends read as zero.
bool make_map_3d(CUtensorMap *m, const void *base, int64_t mid, int64_t outer, int box_mid, int box_outer)
{
    EncodeTiledFn fn = tensor_map_encoder();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)LSA_HEAD, (cuuint64_t)mid, (cuuint64_t)outer};
    cuuint64_t strides[2] = {(cuuint64_t)LSA_HEAD * 2, (cuuint64_t)(mid * LSA_HEAD * 2)};
    cuuint32_t box[3] = {64, (cuuint32_t)box_mid, (cuuint32_t)box_outer};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

// The near-set tiles of one attention call (plans already written by
// k_near_plan): grid (tiles, Hkv), two CTAs per SM.
cudaError_t launch_attention_near_tc(const AttnArgs &a, int tiles, cudaStream_t st)
{
    const int G = a.Hq / a.Hkv;
    const int QT = near_tile_queries(G);
    CUtensorMap tmQ, tmK, tmV;
    if (!make_map_3d(&tmQ, a.Q, a.Hq, a.nq, G, QT) || !make_map_3d(&tmK, a.K, a.Hkv, a.Tk, 1, NT_KC) ||
        !make_map_3d(&tmV, a.V, a.Hkv, a.Tk, 1, NT_KC))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(k_attn_near_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)NT_SMEM);
    if (e != cudaSuccess) return e;
    k_attn_near_tc<<<dim3((unsigned)tiles, (unsigned)a.Hkv), NT_THREADS, NT_SMEM, st>>>(tmQ, tmK, tmV, a);
    return cudaGetLastError();
}

int read_near_error(int clear)
{
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_near_error, sizeof(int)) != cudaSuccess) return -1;
    if (clear && v) {
        int z = 0;
        cudaMemcpyToSymbol(g_near_error, &z, sizeof(int));
    }
    return v;
}

}  // namespace lsa
