// Step 1 of the indexer, "Shrink" (sotaaz blog, "The same steps in general",
// step 1; zhichai forum post, "Key points"): before anything is clustered,
// a position's key is mapped linearly to a 64-dim vector that serves only the
// selection of keys, never the attention itself.  The D-LSA variant trains
// that map per layer; the forum post reports that a map taken from principal
// components works about as well.  x_t = W v_t, with v_t the row of a
// position (e.g. its key over all KV heads, D = Hkv x 128) and W [64, D].
//
// A dense contraction on the tensor cores, bound by reading V from HBM: one
// CTA per 128 positions (the MMA M), N = 64, K = D in 64-wide stages:
//   warp 0     TMA: the 128 x 64 tile of V and the 64 x 64 tile of W of each
//              stage (128-byte swizzle, K-major) into a ring;
//   warp 1     64 TMEM columns; one thread issues tcgen05.mma.kind::f16
//              (bf16 x bf16 -> fp32) four K=16 steps per stage;
//   warps 2-5  one position each (its TMEM lane): the fp32 key, written out
//              if asked; normalised exactly as the cache build normalises a
//              key (the same fixed-order sum of squares, sqrt and divide),
//              staged in shared memory (the drained ring) and summed 4 at a
//              time into pooled items in the cache build's order.
// Three CTAs per SM overlap one tile's ring fill with the others' streams
// (one CTA per SM with 6 stages reached 3.2 TB/s, three with 3 stages 6.2
// TB/s over 4M rows of D = 1024).
// Every wait is bounded (the kernel's device error word, abort flag).
#include <cuda.h>

#include "lsa_common.cuh"
#include "lsa_kernels.h"
#include "lsa_tc.cuh"

namespace lsa {

__device__ int g_shrink_error = 0;

namespace {
constexpr int SH_M = 128;                          // positions per tile (MMA M)
constexpr int SH_KB = 64;                          // K per stage: one 128-byte swizzle row
constexpr int SH_NST = 3;                          // ring stages (three CTAs per SM)
constexpr uint32_t SH_A_BYTES = SH_M * SH_KB * 2;  // 16 KB of V
constexpr uint32_t SH_B_BYTES = 64 * SH_KB * 2;    // 8 KB of W
constexpr int SH_THREADS = 192;
constexpr int SH_NS = 65;  // floats per staged row (conflict-free)
constexpr uint32_t SH_IDESC = tc::idesc_bf16(SH_M, 64);
struct ShCtl {
    uint64_t full[SH_NST], empty[SH_NST], acc, mma_done;
    uint32_t tmem;
    int abort;
};
// the epilogue's staged rows reuse the ring, drained once the accumulator is complete
static_assert(SH_M * SH_NS * 4 <= SH_NST * (SH_A_BYTES + SH_B_BYTES), "staged rows must fit in the ring");
constexpr size_t SH_SMEM = SH_NST * (SH_A_BYTES + SH_B_BYTES) + sizeof(ShCtl) + 1024;
}  // namespace

__global__ void __launch_bounds__(SH_THREADS, 3)
    k_shrink(const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmW, ShrinkArgs a)
{
    extern __shared__ __align__(1024) uint8_t sh_raw[];
    uint8_t *sA = sh_raw + ((1024u - (tc::smem_u32(sh_raw) & 1023u)) & 1023u);
    uint8_t *sB = sA + SH_NST * SH_A_BYTES;
    float *rows = reinterpret_cast<float *>(sA);  // after the last MMA only
    ShCtl *cs = reinterpret_cast<ShCtl *>(sB + SH_NST * SH_B_BYTES);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t t0 = a.t_begin + (int64_t)blockIdx.x * SH_M;
    const int nk = (int)(a.D / SH_KB);
    auto bar = [&](uint64_t &b) { return tc::smem_u32(&b); };
    if (threadIdx.x == 0) {
        cs->abort = 0;
        for (int s = 0; s < SH_NST; ++s) {
            tc::mbar_init(bar(cs->full[s]), 1);
            tc::mbar_init(bar(cs->empty[s]), 1);
        }
        tc::mbar_init(bar(cs->acc), 1);
        tc::mbar_init(bar(cs->mma_done), 1);
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    __syncthreads();
    if (warp == 1) tc::tmem_alloc(tc::smem_u32(&cs->tmem), 64);
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = cs->tmem;
    volatile int *abort = &cs->abort;
    int *err = &g_shrink_error;
    const uint32_t wl = a.wait_limit;

    int issued = 0;
    if (warp == 0 && lane == 0) {
        asm volatile("prefetch.tensormap [%0];\n" ::"l"(&tmV) : "memory");
        asm volatile("prefetch.tensormap [%0];\n" ::"l"(&tmW) : "memory");
        for (int k = 0; k < nk && !*abort; ++k) {
            const int s = k % SH_NST;
            if (k >= SH_NST && !tc::wait_bounded_sleep(bar(cs->empty[s]), (uint32_t)(((k / SH_NST) - 1) & 1), wl, abort, err))
                break;
            tc::mbar_expect_tx(bar(cs->full[s]), SH_A_BYTES + SH_B_BYTES);
            tc::tma_load_2d(tc::smem_u32(sA + s * SH_A_BYTES), &tmV, k * SH_KB, (int)t0, bar(cs->full[s]));
            tc::tma_load_2d(tc::smem_u32(sB + s * SH_B_BYTES), &tmW, k * SH_KB, 0, bar(cs->full[s]));
            ++issued;
        }
    } else if (warp == 1 && lane == 0) {
        bool ok = true;
        for (int k = 0; k < nk; ++k) {
            const int s = k % SH_NST;
            if (!tc::wait_bounded_sleep(bar(cs->full[s]), (uint32_t)((k / SH_NST) & 1), wl, abort, err)) {
                ok = false;
                break;
            }
            tc::fence_after();
#pragma unroll
            for (int kk = 0; kk < SH_KB / 16; ++kk)
                tc::mma_bf16(tmem, tc::smem_desc(tc::smem_u32(sA + s * SH_A_BYTES) + kk * 32),
                             tc::smem_desc(tc::smem_u32(sB + s * SH_B_BYTES) + kk * 32), SH_IDESC,
                             (k | kk) ? 1u : 0u);
            tc::mma_commit(bar(cs->empty[s]));
        }
        if (ok) tc::mma_commit(bar(cs->acc));
    } else if (warp >= 2) {
        const int quad = warp & 3, r = quad * 32 + lane;
        const uint32_t trow = tmem + ((uint32_t)(quad * 32) << 16);
        const bool ok = __all_sync(LSA_FULL, tc::wait_bounded_sleep(bar(cs->acc), 0, wl, abort, err));
        if (ok) {
            tc::fence_after();
            float x[64];
            tc::tmem_ld32_nowait(trow, x);
            tc::tmem_ld32_nowait(trow + 32, x + 32);
            tc::tmem_wait_ld();
            const int64_t t = t0 + r;
            if (a.keys && t < a.t_end) {
                float4 *out = reinterpret_cast<float4 *>(a.keys + t * LSA_D);
#pragma unroll
                for (int d = 0; d < 16; ++d) out[d] = make_float4(x[4 * d], x[4 * d + 1], x[4 * d + 2], x[4 * d + 3]);
            }
            if (a.pooled) {  // normalise as the cache build does (warp_normalize's order, one thread)
                float sq[32];
#pragma unroll
                for (int l = 0; l < 32; ++l) sq[l] = __fadd_rn(__fmul_rn(x[l], x[l]), __fmul_rn(x[l + 32], x[l + 32]));
                const float n = __fsqrt_rn(thread_tree32(sq));
#pragma unroll
                for (int d = 0; d < 64; ++d) rows[r * SH_NS + d] = n > 0.0f ? __fdiv_rn(x[d], n) : 0.0f;
            }
        }
        asm volatile("bar.sync 1, 128;\n" ::: "memory");  // the 4 epilogue warps
        if (ok && a.pooled) {
            // 32 pooled items per tile: thread e takes item e / 4, dims 16 (e % 4) ..
            const int e = (int)threadIdx.x - 64, j = e >> 2, m = e & 3;
            const int64_t tj = t0 + 4 * j;
            if (tj + 3 < a.t_end) {
                float *out = a.pooled + (tj / LSA_NP) * LSA_D + 16 * m;
                const float *y = rows + (4 * j) * SH_NS + 16 * m;
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    float v = y[i];
                    v = __fadd_rn(v, y[SH_NS + i]);
                    v = __fadd_rn(v, y[2 * SH_NS + i]);
                    v = __fadd_rn(v, y[3 * SH_NS + i]);
                    out[i] = v;
                }
            }
        }
    }
    if (warp == 0 && lane == 0 && *abort) {  // copies that may still be in flight
        volatile int dummy = 0;
        for (int k = max(0, issued - SH_NST); k < issued; ++k)
            tc::wait_bounded(bar(cs->full[k % SH_NST]), (uint32_t)((k / SH_NST) & 1), wl, &dummy, err);
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
        tc::tmem_dealloc(tmem, 64);
    }
}

// 2D map over rows of `cols` bf16 (row stride cols x 2 bytes), box
// 64 x box_rows, 128B swizzle; rows past `rows` read as zero.
static bool make_map_rows(CUtensorMap *m, const void *base, int64_t cols, int64_t rows, int box_rows)
{
    EncodeTiledFn fn = tensor_map_encoder();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    cuuint32_t box[2] = {(cuuint32_t)SH_KB, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t launch_shrink(const uint16_t *V, const uint16_t *W, const ShrinkArgs &a, cudaStream_t st)
{
    if (a.t_end <= a.t_begin) return cudaSuccess;
    CUtensorMap tmV, tmW;
    if (!make_map_rows(&tmV, V, a.D, a.t_end, SH_M) || !make_map_rows(&tmW, W, a.D, 64, 64))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(k_shrink, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SH_SMEM);
    if (e != cudaSuccess) return e;
    const int64_t tiles = (a.t_end - a.t_begin + SH_M - 1) / SH_M;
    for (int64_t s = 0; s < tiles; s += 2147483647LL) {
        ShrinkArgs b = a;
        b.t_begin = a.t_begin + s * SH_M;
        const int64_t n = min(tiles - s, (int64_t)2147483647LL);
        const int kt = kt_begin("k_shrink", st);
        k_shrink<<<(unsigned)n, SH_THREADS, SH_SMEM, st>>>(tmV, tmW, b);
        kt_end(kt, st);
        count_launches(1);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

int read_shrink_error(int clear)
{
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_shrink_error, sizeof(int)) != cudaSuccess) return -1;
    if (clear && v) {
        int z = 0;
        cudaMemcpyToSymbol(g_shrink_error, &z, sizeof(int));
    }
    return v;
}

}  // namespace lsa
