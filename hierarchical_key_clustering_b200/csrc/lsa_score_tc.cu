// Flat search scores on the 5th-generation tensor cores (tcgen05 + TMEM).
//
// Method: Latent Sparse Attention pages -- learnaivisually explainer, "What
// one query actually does" (the normalised query is scored against every
// bucket centroid of the earlier cluster blocks); zhichai forum post, "Key
// points" (Flat search scores all bucket centroids, ~T/8 per query).
//
// S = Q^ C^T is a dense 64-deep contraction.  A CTA owns two tiles of 128
// queries (two MMA M operands) and streams 128-centroid tiles (the MMA N) of
// its bucket range; each centroid tile feeds both query tiles, which halves
// the centroid bytes per score the CTA pulls from L2.
//   warp 0        TMA producer: both query tiles once (one 256-row box),
//                 centroid tiles into a ring of 4 (threshold pass) or 8
//                 (filter pass) stages, 128B-swizzled, K-major;
//   warp 1        allocates 512 TMEM columns = [query tile][2 buffers] x 128
//                 fp32 columns; one thread issues tcgen05.mma.kind::f16
//                 (bf16 x bf16 -> fp32, 4 x K=16 per query tile) and commits
//                 to the stage's "empty" barrier and the buffer's "full" one;
//   warps 2..9    epilogue, two warps per TMEM lane quadrant: warp w reads
//                 lanes 32 (w % 4) .. +31 of query tile (w - 2) / 4, so each
//                 thread owns one query row; it copies its 128 scores out of
//                 TMEM (4 loads, one wait), frees the buffer for the next MMA
//                 and then works on registers.
// The epilogue is fused with the pass's work, so the score matrix is never
// stored:
//   GMAX    the maximum of each group of g consecutive buckets goes into the
//           row's 256-bin histogram over [-1.0625, 1.0625] in shared memory.
//           A CTA that covers the query's whole bucket range turns the
//           histogram into the threshold tau itself: tau = lower edge of the
//           bin that holds the P-th largest group maximum, a value <= the
//           P-th largest group maximum <= the P-th largest score.  Otherwise
//           the rows are added into a global per-query histogram and k_tau
//           finishes;
//   FILTER  every aligned group of 4 buckets whose best score is >= tau is
//           appended as one entry (first bucket id, its 4 scores); the
//           expansion kernel keeps the scores >= tau.
// Causal masking: bucket b counts for query q only if b < 64 * H(q); N =
// 64 * H is a multiple of 64, so every 64-column half tile is wholly inside
// or outside a query's range.
// Every mbarrier wait is bounded: a wait that runs out sets the library's
// device error word and the CTA leaves its loops, waits (bounded) for the
// copies it issued, frees its TMEM and exits.
#include <cuda.h>

#include <climits>

#include "lsa_common.cuh"
#include "lsa_kernels.h"
#include "lsa_tc.cuh"

namespace lsa {

__device__ int g_device_error = 0;

namespace {

constexpr int TQ = 128;             // queries per tile (MMA M)
constexpr int QT = 2;               // query tiles per CTA
constexpr int TB = 128;             // centroids per tile (MMA N)
constexpr int NST_GMAX = 4;         // centroid stages, threshold pass (its histograms take the rest)
constexpr int NST_FILTER = 8;       // centroid stages, filter pass
constexpr int NST_MAX = 8;
constexpr uint32_t A_BYTES = QT * TQ * LSA_D * 2;  // 32 KB
constexpr uint32_t B_BYTES = TB * LSA_D * 2;       // 16 KB
constexpr int TMEM_COLS = 512;      // [query tile][buffer] x 128 fp32 columns
constexpr int SAMPLE_G = 8;         // group width of the sampled threshold pass
constexpr int EPI_WARPS = 8 * QT;   // 16: TMEM lane quadrant x query tile x column half
constexpr int THREADS = 64 + 32 * EPI_WARPS;  // 576
constexpr int HSTRIDE = HIST_BINS / 2 + 1;   // 32-bit words per row histogram (2 x u16 bins per word, +1 pad)
constexpr uint32_t HIST_BYTES = QT * TQ * HSTRIDE * 4;
constexpr uint32_t ROWCNT_BYTES = QT * TQ * 4;  // per-row entry counters of the filter pass

using tc::mbar_arrive;
using tc::mbar_expect_tx;
using tc::mbar_init;
using tc::smem_desc;
using tc::smem_u32;
using tc::tma_load_2d;
using tc::tmem_ld32_nowait;
using tc::tmem_wait_ld;
using tc::mma_commit;

// Bounded wait; on expiry sets the device error word and the CTA abort flag.
// Waiting threads sleep on the barrier instead of spinning, so that the
// epilogue warps' spins do not take the issue slots of the working ones.
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, uint32_t limit, volatile int *abort)
{
    return tc::wait_bounded_sleep(bar, parity, limit, abort, &g_device_error);
}

// kind::f16: D fp32, A and B bf16, both K-major, N = 128, M = 128.
constexpr uint32_t IDESC = tc::idesc_bf16(TQ, TB);

__device__ __forceinline__ void mma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t accumulate)
{
    tc::mma_bf16(tmem_d, adesc, bdesc, IDESC, accumulate);
}

__device__ __forceinline__ void tc_fence_before() { tc::fence_before(); }
__device__ __forceinline__ void tc_fence_after() { tc::fence_after(); }

__device__ __forceinline__ float max3f(float a, float b, float c)
{
    float d;
    asm("max.f32 %0, %1, %2, %3;\n" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

__device__ __forceinline__ float max4f(const float *v)
{
    return fmaxf(max3f(v[0], v[1], v[2]), v[3]);
}

__device__ __forceinline__ float max8f(const float *v)
{
    return max3f(max3f(v[0], v[1], v[2]), max3f(v[3], v[4], v[5]), fmaxf(v[6], v[7]));
}

struct TcSmem {
    uint64_t full[NST_MAX];
    uint64_t empty[NST_MAX];
    uint64_t tfull[2];
    uint64_t tempty[2];
    uint64_t a_full;
    uint64_t mma_done;
    uint32_t tmem_base;
    int abort;
    int nmax;
    int nmin;
};

}  // namespace

// grid: x = pair of query tiles, y = bucket-tile chunk.  block = 320 threads.
__global__ void __launch_bounds__(THREADS, 1)
    k_score_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, ScoreTcArgs a,
               IndexWs ws)
{
    extern __shared__ __align__(1024) uint8_t tsm_raw[];
    // tiles first (1024-aligned for the 128B swizzle), control block after
    uint8_t *tsm = tsm_raw + ((1024u - (smem_u32(tsm_raw) & 1023u)) & 1023u);
    const int nst = a.mode == 0 ? NST_GMAX : NST_FILTER;
    uint8_t *sA = tsm;
    uint8_t *sB = tsm + A_BYTES;
    uint32_t *hist = reinterpret_cast<uint32_t *>(tsm + A_BYTES + nst * B_BYTES);  // [QT*TQ][HSTRIDE], GMAX only
    int *rowcnt = reinterpret_cast<int *>(tsm + A_BYTES + nst * B_BYTES);           // [QT*TQ], FILTER only
    TcSmem *cs = reinterpret_cast<TcSmem *>(tsm + A_BYTES + nst * B_BYTES + (a.mode == 0 ? HIST_BYTES : ROWCNT_BYTES));

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t q0 = (int64_t)blockIdx.x * (QT * TQ);
    // epilogue identity of this thread (meaningful for warps >= 2)
    const int ep_quad = warp & 3, ep_sel = (warp - 2) >> 2;
    const int ep_qt = ep_sel & 1, ep_half = ep_sel >> 1;
    const int ep_r = ep_quad * 32 + lane;
    const int64_t ep_q = q0 + ep_qt * TQ + ep_r;
    const int ep_N = (warp >= 2 && ep_q < a.nq) ? ws.horizon[ep_q] * LSA_NBKT : 0;
    if (a.mode == 0)
        for (int i = threadIdx.x; i < QT * TQ * HSTRIDE; i += THREADS) hist[i] = 0u;
    else
        for (int i = threadIdx.x; i < QT * TQ; i += THREADS) rowcnt[i] = 0;

    if (threadIdx.x == 0) {
        cs->nmax = 0;
        cs->nmin = INT_MAX;
        cs->abort = 0;
        for (int s = 0; s < nst; ++s) {
            mbar_init(smem_u32(&cs->full[s]), 1);
            mbar_init(smem_u32(&cs->empty[s]), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&cs->tfull[b]), 1);
            mbar_init(smem_u32(&cs->tempty[b]), EPI_WARPS);
        }
        mbar_init(smem_u32(&cs->a_full), 1);
        mbar_init(smem_u32(&cs->mma_done), 1);
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    __syncthreads();
    if (threadIdx.x < QT * TQ) {
        const int64_t q = q0 + threadIdx.x;
        const int N = (q < a.nq) ? ws.horizon[q] * LSA_NBKT : 0;
        atomicMax(&cs->nmax, N);
        if (q < a.nq) atomicMin(&cs->nmin, N);
    }
    __syncthreads();
    // the sampled threshold pass (block-uniform): every S-th centroid tile,
    // while a query's sampled groups of 8 stay below 2^16 (the bin counters)
    const bool sampled = a.mode == 0 && a.sample > 1 && a.whole_range && (int64_t)cs->nmin >= a.sample_min_n &&
                         (int64_t)cs->nmax <= (int64_t)a.sample * 500000;
    const int S = sampled ? a.sample : 1;
    const int64_t tiles_all = ((int64_t)cs->nmax + TB - 1) / TB;
    const int64_t j0 = (int64_t)blockIdx.y * a.chunk_tiles;
    const int64_t j1 = min(j0 + a.chunk_tiles, tiles_all);
    const int ntiles = j1 > j0 ? (int)((j1 - j0 + S - 1) / S) : 0;
    if (ntiles == 0) return;  // uniform: nothing allocated yet
    // CTAs start their walk at evenly spread tiles of the range (and wrap), so
    // that at any moment they read different centroid tiles instead of all
    // pulling the same lines from the same L2 slices
    const int rot = (int)(((int64_t)blockIdx.x * ntiles) / gridDim.x);
    auto tile_of = [&](int it) {
        const int r = it + rot;
        return j0 + (int64_t)(r >= ntiles ? r - ntiles : r) * S;
    };

    volatile int *abort = &cs->abort;
    if (warp == 1) {  // whole warp: TMEM allocation
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(
                         smem_u32(&cs->tmem_base)),
                     "r"(TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = cs->tmem_base;

    int issued = 0;  // producer: centroid tiles issued
    if (warp == 0 && lane == 0) {
        asm volatile("prefetch.tensormap [%0];\n" ::"l"(&tmA) : "memory");
        asm volatile("prefetch.tensormap [%0];\n" ::"l"(&tmB) : "memory");
        const uint32_t abar = smem_u32(&cs->a_full);
        mbar_expect_tx(abar, A_BYTES);
        if (a.extra_tx == 0) tma_load_2d(smem_u32(sA), &tmA, 0, (int)q0, abar);  // test hook: never arrives
        int s = 0, ph = 0;
        for (int it = 0; it < ntiles; ++it) {
            if (it >= nst && !wait_bounded(smem_u32(&cs->empty[s]), (uint32_t)(ph ^ 1), a.wait_limit, abort)) break;
            const uint32_t bar = smem_u32(&cs->full[s]);
            mbar_expect_tx(bar, B_BYTES);
            tma_load_2d(smem_u32(sB + s * B_BYTES), &tmB, 0, (int)(tile_of(it) * TB), bar);
            ++issued;
            if (++s == nst) {
                s = 0;
                ph ^= 1;
            }
        }
    } else if (warp == 1 && lane == 0) {
        if (wait_bounded(smem_u32(&cs->a_full), 0, a.wait_limit, abort)) {
            tc_fence_after();
            const uint32_t a_addr = smem_u32(sA);
            int s = 0, ph = 0;
            for (int it = 0; it < ntiles; ++it) {
                const int buf = it & 1;
                if (!wait_bounded(smem_u32(&cs->full[s]), (uint32_t)ph, a.wait_limit, abort)) break;
                if (it >= 2 &&
                    !wait_bounded(smem_u32(&cs->tempty[buf]), (uint32_t)(((it >> 1) - 1) & 1), a.wait_limit, abort))
                    break;
                tc_fence_after();
                const uint32_t b_addr = smem_u32(sB + s * B_BYTES);
#pragma unroll
                for (int qt = 0; qt < QT; ++qt) {
                    const uint32_t d = tmem + (uint32_t)((qt * 2 + buf) * TB);
                    const uint32_t aq = a_addr + (uint32_t)(qt * TQ * LSA_D * 2);
#pragma unroll
                    for (int k = 0; k < LSA_D / 16; ++k)
                        mma_bf16(d, smem_desc(aq + k * 32), smem_desc(b_addr + k * 32), k > 0 ? 1u : 0u);
                }
                mma_commit(smem_u32(&cs->empty[s]));
                mma_commit(smem_u32(&cs->tfull[buf]));
                if (++s == nst) {
                    s = 0;
                    ph ^= 1;
                }
            }
        }
    } else if (warp >= 2) {
        // epilogue: warp w reads TMEM lanes 32 (w % 4) .. + 31 (rows of query
        // tile qt) and one 64-column half of each 128-column accumulator, 32
        // columns at a time; the row's two halves go to two warps
        const float NEG = __int_as_float(0xff800000);
        // <= 64: a group never spans two halves; a sampled pass counts the
        // maxima of groups of 8 (its targets lie far in the tail, where a
        // group rarely holds two buckets above them)
        const int g = sampled ? SAMPLE_G : (ep_N > 0 ? group_width(ep_N, a.P) : 1);
        const float tau = (a.mode == 1 && ep_q < a.nq) ? ws.tau[ep_q] : 0.0f;
        uint32_t *hrow = hist + (ep_qt * TQ + ep_r) * HSTRIDE;
        auto count = [&](float m) {  // counts per bin stay below 2^16 (at most 2^16 - 1 groups per query)
            const int bin = hist_bin(m);
            atomicAdd(&hrow[bin >> 1], 1u << ((bin & 1) * 16));
        };
        float4 *c4 = reinterpret_cast<float4 *>(ws.cand4) + ep_q * ws.cap;
        int32_t *cg = ws.cand_g + ep_q * ws.cap;
        const uint32_t lane_base = tmem + ((uint32_t)(ep_quad * 32) << 16) + (uint32_t)(ep_qt * 2 * TB + ep_half * 64);
        for (int it = 0; it < ntiles; ++it) {
            const int buf = it & 1;
            const bool ok = wait_bounded(smem_u32(&cs->tfull[buf]), (uint32_t)((it >> 1) & 1), a.wait_limit, abort);
            if (!__all_sync(LSA_FULL, ok)) break;  // warp-uniform: tcgen05.ld needs the whole warp
            tc_fence_after();
            const int64_t bh = tile_of(it) * TB + 64 * ep_half;  // first bucket of this half
            float run = NEG;                                     // g = 64: maximum over the half
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                float x[32];
                tmem_ld32_nowait(lane_base + (uint32_t)(buf * TB + 32 * c), x);
                tmem_wait_ld();
                if (c == 1) {  // this warp has read its half: the MMA may refill the buffer
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(smem_u32(&cs->tempty[buf]));
                }
                const int64_t b0 = bh + 32 * c;
                const bool in = bh < ep_N;  // N is a multiple of 64: the half is wholly in or out
                if (a.mode == 0) {
                    if (!in) continue;  // nothing warp-wide below in this pass
                    if (g >= 8) {
                        float m8[4];
#pragma unroll
                        for (int j = 0; j < 4; ++j) m8[j] = max8f(x + 8 * j);
                        if (g == 8) {
#pragma unroll
                            for (int j = 0; j < 4; ++j) count(m8[j]);
                        } else if (g == 16) {
                            count(fmaxf(m8[0], m8[1]));
                            count(fmaxf(m8[2], m8[3]));
                        } else {
                            const float m32 = max4f(m8);
                            if (g == 32) {
                                count(m32);
                            } else {  // g == 64: both 32-column parts
                                run = fmaxf(run, m32);
                                if (c == 1) count(run);
                            }
                        }
                    } else if (g == 4) {
#pragma unroll
                        for (int j = 0; j < 8; ++j) count(max4f(x + 4 * j));
                    } else if (g == 2) {
#pragma unroll
                        for (int j = 0; j < 16; ++j) count(fmaxf(x[2 * j], x[2 * j + 1]));
                    } else {
#pragma unroll
                        for (int j = 0; j < 32; ++j) count(x[j]);
                    }
                } else {
                    float m4[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) m4[j] = max4f(x + 4 * j);
                    const float m32 = fmaxf(max4f(m4), max4f(m4 + 4));
                    const bool hit = in && m32 >= tau;
                    if (!__any_sync(LSA_FULL, hit)) continue;  // every lane votes
                    if (hit) {
                        // one bit per 4-bucket group at or above tau; entries are
                        // written only for those (usually one per hit lane)
                        unsigned mask = 0;
#pragma unroll
                        for (int j = 0; j < 8; ++j) mask |= (m4[j] >= tau ? 1u : 0u) << j;
                        const int n = __popc(mask);
                        int slot = a.whole_range ? atomicAdd(&rowcnt[ep_qt * TQ + ep_r], n) : atomicAdd(ws.cnt + ep_q, n);
                        while (mask) {
                            const int j = __ffs(mask) - 1;
                            mask &= mask - 1;
                            // x[4j .. 4j+3] for a runtime j: select on its bits
                            float4 v[4];
#pragma unroll
                            for (int i = 0; i < 4; ++i)
                                v[i] = (j & 1) ? make_float4(x[8 * i + 4], x[8 * i + 5], x[8 * i + 6], x[8 * i + 7])
                                               : make_float4(x[8 * i], x[8 * i + 1], x[8 * i + 2], x[8 * i + 3]);
                            const float4 w0 = (j & 2) ? v[1] : v[0], w1 = (j & 2) ? v[3] : v[2];
                            const float4 e = (j & 4) ? w1 : w0;
                            if (slot < ws.cap) {
                                c4[slot] = e;
                                cg[slot] = (int32_t)(b0 + 4 * j);
                            }
                            ++slot;
                        }
                    }
                }
            }
        }
    }
    __syncthreads();
    // per-row results, once both halves of every row are in: one thread per row
    if (warp >= 2 && ep_half == 0 && ep_q < a.nq && ep_N > 0 && !*abort) {
        uint32_t *hrow = hist + (ep_qt * TQ + ep_r) * HSTRIDE;
        if (a.mode == 1) {
            if (a.whole_range) ws.cnt[ep_q] = rowcnt[ep_qt * TQ + ep_r];
        } else if (a.whole_range) {
            // this CTA saw every bucket of the query (or every S-th tile of
            // them): threshold from the histogram.  Exact pass: the P-th
            // largest group maximum, so >= P buckets score >= tau.  Sampled
            // pass: the score above which margin x P x (sampled / visible)
            // sampled scores lie -- about margin x P buckets in all, checked
            // by the expansion
            int64_t count = n_groups(ep_N, a.P), target = a.P;
            if (sampled) {
                const int64_t full = ep_N / TB;  // N is a multiple of 64: at most one half tile
                const int64_t ns = ((full + S - 1) / S) * TB + ((ep_N % TB) != 0 && full % S == 0 ? ep_N % TB : 0);
                count = ns / SAMPLE_G;
                target = (int64_t)ceilf(a.sample_margin * (float)a.P * (float)ns / (float)ep_N);
            }
            float t = __int_as_float(0xff800000);
            if (count > target) {
                int64_t acc = 0;
                for (int bin = HIST_BINS - 1; bin > 0; --bin) {
                    acc += (hrow[bin >> 1] >> ((bin & 1) * 16)) & 0xffffu;
                    if (acc >= target) {
                        t = hist_edge(bin);
                        break;
                    }
                }
            }
            ws.tau[ep_q] = t;
        } else {
            uint32_t *gh = ws.ghist + ep_q * HIST_BINS;
            for (int bin = 0; bin < HIST_BINS; ++bin) {
                const uint32_t c = (hrow[bin >> 1] >> ((bin & 1) * 16)) & 0xffffu;
                if (c) atomicAdd(gh + bin, c);
            }
        }
    }
    if (warp == 0 && lane == 0 && *abort) {
        // copies that may still be in flight (the producer reused a stage only
        // after the MMA had consumed its previous copy): wait for the last
        // nst of them (bounded) before exit
        volatile int dummy = 0;
        for (int it = max(0, issued - nst); it < issued; ++it)
            wait_bounded(smem_u32(&cs->full[it % nst]), (uint32_t)((it / nst) & 1), a.wait_limit, &dummy);
        // and the query tile: the wait that ran out may have been the MMA
        // thread's wait on it, with the copy slow rather than lost
        if (a.extra_tx == 0) wait_bounded(smem_u32(&cs->a_full), 0, a.wait_limit, &dummy);
    }
    if (warp == 1 && lane == 0) {
        // every MMA this thread issued has finished before its TMEM is freed
        volatile int dummy = 0;
        mma_commit(smem_u32(&cs->mma_done));
        wait_bounded(smem_u32(&cs->mma_done), 0, a.wait_limit, &dummy);
    }
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(TMEM_COLS)
                     : "memory");
    }
}

// ---------------------------------------------------------------------------
// Host side: tensor maps and launch.

EncodeTiledFn tensor_map_encoder()
{
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// Rows of 64 bf16 (128 B), box = box_rows x 64, 128B swizzle; rows past the
// end read as zero.
static bool make_map(CUtensorMap *m, const void *base, int64_t rows, int box_rows)
{
    EncodeTiledFn fn = tensor_map_encoder();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)LSA_D, (cuuint64_t)(rows > 0 ? rows : 1)};
    cuuint64_t strides[1] = {(cuuint64_t)LSA_D * 2};
    cuuint32_t box[2] = {(cuuint32_t)LSA_D, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t launch_score_tc(const ScoreTcArgs &a, const IndexWs &ws, const uint16_t *centroid_bf16, cudaStream_t st,
                            int n_sm, int *whole_range)
{
    if (a.nq <= 0 || a.nb_total <= 0) return cudaSuccess;
    CUtensorMap tmA, tmB;
    if (!make_map(&tmA, ws.qhat, a.nq, QT * TQ) || !make_map(&tmB, centroid_bf16, a.nb_total, TB))
        return cudaErrorInvalidValue;
    const int64_t qpairs = (a.nq + QT * TQ - 1) / (QT * TQ);
    const int64_t tiles = (a.nb_total + TB - 1) / TB;
    // One CTA per pair of query tiles over its whole bucket range when that
    // fills most SMs (no atomics, threshold set in place); otherwise split the
    // range so that about four waves of CTAs balance the SMs.  (Splitting to
    // even out the waves of 256 pairs on 148 SMs measured slower: the filter
    // pass then counts every row's entries with global atomics.)
    int64_t chunks = 1;
    if (qpairs * 4 < (int64_t)n_sm * 3) chunks = (4LL * n_sm + qpairs - 1) / qpairs;
    if (chunks > tiles) chunks = tiles;
    if (chunks < 1) chunks = 1;
    if (chunks > 65535) chunks = 65535;
    ScoreTcArgs b = a;
    b.chunk_tiles = (tiles + chunks - 1) / chunks;
    chunks = (tiles + b.chunk_tiles - 1) / b.chunk_tiles;
    b.whole_range = (chunks == 1) ? 1 : 0;
    if (whole_range) *whole_range = b.whole_range;
    const size_t smem = A_BYTES + (size_t)(a.mode == 0 ? NST_GMAX : NST_FILTER) * B_BYTES +
                        (a.mode == 0 ? HIST_BYTES : ROWCNT_BYTES) + sizeof(TcSmem) + 1024;
    cudaError_t e = cudaFuncSetAttribute(k_score_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int kt = kt_begin(a.mode == 0 ? (a.sample > 1 && b.whole_range ? "k_score_tc:sampled" : "k_score_tc:threshold")
                                        : "k_score_tc:filter",
                            st);
    k_score_tc<<<dim3((unsigned)qpairs, (unsigned)chunks), THREADS, smem, st>>>(tmA, tmB, b, ws);
    kt_end(kt, st);
    count_launches(1);
    return cudaGetLastError();
}

int read_device_error(int clear)
{
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof(int)) != cudaSuccess) return -1;
    if (clear && v) {
        int z = 0;
        cudaMemcpyToSymbol(g_device_error, &z, sizeof(int));
    }
    const int w = read_shrink_error(clear);  // the projection kernel's own word
    if (w < 0) return -1;
    const int wn = read_near_error(clear);  // the near-set tensor-core attention's word
    if (wn < 0) return -1;
    const int ba = read_bounds_error_attn(clear), bi = read_bounds_error_index(clear);  // debug build only
    if (ba < 0 || bi < 0) return -1;
    return v | w | wn | ba | bi;
}

}  // namespace lsa
