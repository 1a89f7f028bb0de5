// Device helpers shared by the LSA kernels (sm_100a).
//
// Build-path arithmetic (normalise, pool, Ward costs, tree costs, centroids)
// uses the IEEE-rounded intrinsics __fadd_rn / __fmul_rn / __fsub_rn /
// __fdiv_rn / __fsqrt_rn so that nvcc never contracts a multiply and an add
// into an FMA: every value is reproducible bit for bit.  64-term sums of
// squares follow one fixed order: lane l holds terms l and l+32, adds them,
// then an xor butterfly over offsets 16, 8, 4, 2, 1 (IEEE addition is
// commutative, so all lanes end with the same bits).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#define LSA_D 64
#define LSA_BLK 512
#define LSA_NP 4
#define LSA_NITEMS 128
#define LSA_NBKT 64
#define LSA_NSLOT 16
#define LSA_RUN 128
#define LSA_HEAD 128
#define LSA_MAXHEADS 16  /* index heads per token (multi-head Flat search) */
#define LSA_FULL 0xffffffffu

namespace lsa {

__device__ __forceinline__ float warp_sum_pairs(float t)
{
#pragma unroll
    for (int s = 16; s >= 1; s >>= 1) t = __fadd_rn(t, __shfl_xor_sync(LSA_FULL, t, s));
    return t;
}

// Sum of squares of a 64-vector held as (a = x[lane], b = x[lane + 32]).
__device__ __forceinline__ float warp_sumsq(float a, float b)
{
    return warp_sum_pairs(__fadd_rn(__fmul_rn(a, a), __fmul_rn(b, b)));
}

// Squared distance of two 64-vectors held lane-wise.
__device__ __forceinline__ float warp_sqdist(float a0, float a1, float b0, float b1)
{
    float e0 = __fsub_rn(a0, b0), e1 = __fsub_rn(a1, b1);
    return warp_sum_pairs(__fadd_rn(__fmul_rn(e0, e0), __fmul_rn(e1, e1)));
}

// The same fixed-order reduction done by one thread over 32 partial terms.
__device__ __forceinline__ float thread_tree32(float *t)
{
#pragma unroll
    for (int s = 16; s >= 1; s >>= 1)
#pragma unroll
        for (int l = 0; l < s; ++l) t[l] = __fadd_rn(t[l], t[l + s]);
    return t[0];
}

// Normalise one lane-wise 64-vector: x / sqrt(sum x^2); zero stays zero.
__device__ __forceinline__ void warp_normalize(float &a, float &b)
{
    float n = __fsqrt_rn(warp_sumsq(a, b));
    if (n > 0.0f) {
        a = __fdiv_rn(a, n);
        b = __fdiv_rn(b, n);
    } else {
        a = 0.0f;
        b = 0.0f;
    }
}

__device__ __forceinline__ uint16_t f2bf_bits(float f)
{
    __nv_bfloat16 h = __float2bfloat16_rn(f);
    return *reinterpret_cast<uint16_t *>(&h);
}

__device__ __forceinline__ float bf_bits2f(uint16_t b)
{
    return __uint_as_float(((uint32_t)b) << 16);
}

// Monotone map float -> uint32 (larger float -> larger key).
__device__ __forceinline__ uint32_t f2ord(float f)
{
    uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float ord2f(uint32_t k)
{
    uint32_t u = (k & 0x80000000u) ? (k & 0x7fffffffu) : ~k;
    return __uint_as_float(u);
}

// Radix select: the P-th largest of the ordered keys get(i), i in [0, n)
// (8 bits per round, most significant first); all threads of the block call
// it and get the same key.
template <typename Get>
__device__ uint32_t block_select_ord(int64_t n, int64_t P, Get get, int *hist, int *sh)
{
    uint32_t prefix = 0, mask = 0;
    int64_t rem = P;
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int i = threadIdx.x; i < 256; i += blockDim.x) hist[i] = 0;
        __syncthreads();
        const int64_t n_round = ((n + blockDim.x - 1) / blockDim.x) * blockDim.x;
        for (int64_t i = threadIdx.x; i < n_round; i += blockDim.x) {
            const bool valid = i < n;
            const uint32_t u = valid ? get(i) : 0u;
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

// Rank key for buckets: ascending order = (score desc, id asc).
__device__ __forceinline__ uint64_t rank_key(float s, int32_t id)
{
    s = __fadd_rn(s, 0.0f);  // -0 ranks as +0 (they compare equal)
    return ((uint64_t)(~f2ord(s)) << 32) | (uint32_t)id;
}

__device__ __forceinline__ float rank_key_score(uint64_t k)
{
    return ord2f(~(uint32_t)(k >> 32));
}

__device__ __forceinline__ int32_t rank_key_id(uint64_t k)
{
    return (int32_t)(uint32_t)(k & 0xffffffffu);
}

// Programmatic dependent launch.  pdl_wait: block until the grids this one
// depends on have completed and their writes are visible (a no-op for an
// ordinary launch); pdl_release: let the next kernel of the stream start
// launching, so that its launch and prologue overlap this grid's tail.
__device__ __forceinline__ void pdl_wait()
{
    asm volatile("griddepcontrol.wait;\n" ::: "memory");
}
__device__ __forceinline__ void pdl_release()
{
    asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
}

__host__ __device__ __forceinline__ int64_t pow2_ceil64(int64_t x)
{
    int64_t p = 1;
    while (p < x) p <<= 1;
    return p;
}

__host__ __device__ __forceinline__ int64_t pow2_floor64(int64_t x)
{
    int64_t p = 1;
    while ((p << 1) <= x) p <<= 1;
    return p;
}

// Group width of the Flat threshold pass for a query that sees N buckets:
// the largest power of two <= N / (4P), clamped to [1, 64], so a query has
// between 4P and 8P group maxima (or N of them when N is small).
__host__ __device__ __forceinline__ int group_width(int64_t N, int64_t P)
{
    int64_t g = (N >= 4 * P) ? pow2_floor64(N / (4 * P)) : 1;
    if (g > 64) g = 64;
    return (int)g;
}

__host__ __device__ __forceinline__ int64_t n_groups(int64_t N, int64_t P)
{
    int g = group_width(N, P);
    return (N + g - 1) / g;
}

// Bounds checks of the debug build (built with -DLSA_BOUNDS_CHECKS=1, the
// library liblsa_debug.so): the gather indices kernels read from memory --
// the list entries the attention gathers K/V rows with, the bucket ids and
// member positions the expansion reads, the child ids the tree search
// follows -- and every list length are checked before use.  A
// failed check ORs its code into this translation unit's g_bounds_error and
// the access is skipped; nothing traps.  lsa_check_device_errors() reads and
// clears the words of every translation unit.  In the release build
// LSA_IN_BOUNDS(cond, code) is the constant true and costs nothing.
#ifndef LSA_BOUNDS_CHECKS
#define LSA_BOUNDS_CHECKS 0
#endif
enum : int {
    BOUNDS_LIST = 2,    // an index-list entry outside [0, Tk) or not increasing, or a length above Lmax
    BOUNDS_BUCKET = 4,  // a bucket id outside the query's visible buckets, or a member position out of range
    BOUNDS_NODE = 8,    // a tree-node id outside its level
};

static __device__ int g_bounds_error = 0;  // one per translation unit

__device__ __forceinline__ bool bounds_check(bool ok, int code)
{
    if (!ok) atomicOr(&g_bounds_error, code);
    return ok;
}

#if LSA_BOUNDS_CHECKS
#define LSA_IN_BOUNDS(cond, code) (::lsa::bounds_check((cond), (code)))
#else
#define LSA_IN_BOUNDS(cond, code) (true)
#endif

// Defines `int name(int clear)`: this translation unit's bounds word (read,
// and cleared when clear != 0), or -1 if it cannot be read.
#define LSA_BOUNDS_READER(name)                                                           \
    int name(int clear)                                                                   \
    {                                                                                     \
        int v = 0;                                                                        \
        if (cudaMemcpyFromSymbol(&v, ::lsa::g_bounds_error, sizeof(int)) != cudaSuccess) \
            return -1;                                                                    \
        if (clear && v) {                                                                 \
            int z = 0;                                                                    \
            if (cudaMemcpyToSymbol(::lsa::g_bounds_error, &z, sizeof(int)) != cudaSuccess) \
                return -1;                                                                \
        }                                                                                 \
        return v;                                                                         \
    }

}  // namespace lsa
