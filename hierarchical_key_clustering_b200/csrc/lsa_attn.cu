// Exact sparse attention over LSA index lists on sm_100a.
//
// Method: Latent Sparse Attention pages -- learnaivisually explainer, "What
// one query actually does": one index list per query, shared by all of its
// attention heads, then ordinary (softmax) attention over sink, selected keys
// and window.
//
// Each list is private to one query, so the work is a gather: per (query,
// KV head) the listed K and V rows (256 B each) stream in once and are used
// by the Hq/Hkv query heads of that group.  One warp owns one (query, KV
// head[, key split]) unit: its G = Hq/Hkv heads form the rows of a 16-row
// mma.sync tile (rows >= G are zero), 16 gathered keys form a chunk, and an
// fp32 online softmax carries the running max and sum.  K/V rows are
// gathered with cp.async (16 B per lane) into a 2-stage ring of swizzled
// 256-byte rows in shared memory (2 stages leave room for 12 warps per SM,
// which hides the gather latency better than deeper rings with 8 warps); each warp loads the list indices of the next chunk one issue ahead,
// so a gather never waits on a dependent index load.  The warps of a CTA are
// independent (no CTA barrier), which keeps many gathers in flight per SM.
// Units run head-major (all queries of KV head 0, then head 1, ...): the K/V
// rows of one head are 1/Hkv of the cache, so at 128K tokens (67 MB per
// head) the rows that queries share stay in L2.
// A decode query (few queries, long list) splits its list over many warps
// and a second kernel merges the partial results by log-sum-exp.
//
// Measured alternative (kept out): one CTA per query fetching each 2 KB
// position row of all 8 KV heads with cp.async.bulk into an mbarrier ring was
// 1.5x slower on the 128K workload -- one pipeline per SM hides latency worse
// than eight independent warp pipelines.
#include <cuda_bf16.h>

#include <array>
#include <vector>

#include "lsa_common.cuh"
#include "lsa_kernels.h"

namespace lsa {

constexpr int KCH = 16;                          // keys per chunk
constexpr int ROWB = 128;                        // bf16 per smem row (256 B, 16-byte segments XOR-swizzled)
constexpr int NST = 2;                           // pipeline stages (2 x 8 KB per warp: 3 CTAs of 4 warps per SM)
constexpr int NST_SPLIT = 4;                     // stages of split lists (few warps: one CTA per SM, deeper rings)
constexpr int STAGE_BYTES = 2 * KCH * ROWB * 2;  // K + V
constexpr int AWARPS = 4;
constexpr float LOG2E = 1.4426950408889634f;
constexpr float LN2 = 0.6931471805599453f;

// Byte offset of the 16-byte segment `seg` (dims 8 seg .. 8 seg + 7) of row
// `row` in a staged K or V tile.  Rows are 256 B, so every 32-byte sector of
// a gathered row lands in one aligned 32-byte piece of shared memory (the XOR
// keeps segment pairs 2k, 2k + 1 together), and the XOR with row & 7 puts the
// 8 rows an ldmatrix reads at one logical segment in 8 different bank groups.
__device__ __forceinline__ uint32_t tile_off(int row, int seg)
{
    return (uint32_t)(row * (ROWB * 2) + ((seg ^ (row & 7)) << 4));
}

__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], uint32_t addr)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, int bytes)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(bytes));
}

__device__ __forceinline__ void cp_async16_hint(uint32_t dst, const void *src, int bytes, uint64_t pol)
{
    asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2, %3;\n" ::"r"(dst), "l"(src),
                 "r"(bytes), "l"(pol));
}

__device__ __forceinline__ float ld_f_hint(const float *p, uint64_t pol)
{
    float v;
    asm volatile("ld.global.L2::cache_hint.f32 %0, [%1], %2;\n" : "=f"(v) : "l"(p), "l"(pol));
    return v;
}

__device__ __forceinline__ float2 ld_f2_hint(const float *p, uint64_t pol)
{
    float2 v;
    asm volatile("ld.global.L2::cache_hint.v2.f32 {%0, %1}, [%2], %3;\n" : "=f"(v.x), "=f"(v.y) : "l"(p), "l"(pol));
    return v;
}

__device__ __forceinline__ void st_f_hint(float *p, float v, uint64_t pol)
{
    asm volatile("st.global.L2::cache_hint.f32 [%0], %1, %2;\n" ::"l"(p), "f"(v), "l"(pol) : "memory");
}

__device__ __forceinline__ void st_f2_hint(float *p, float2 v, uint64_t pol)
{
    asm volatile("st.global.L2::cache_hint.v2.f32 [%0], {%1, %2}, %3;\n" ::"l"(p), "f"(v.x), "f"(v.y), "l"(pol)
                 : "memory");
}

__device__ __forceinline__ void cp_commit()
{
    asm volatile("cp.async.commit_group;\n" ::);
}

template <int N>
__device__ __forceinline__ void cp_wait()
{
    asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

__device__ __forceinline__ uint32_t ld_u32(const uint16_t *p)
{
    return *reinterpret_cast<const uint32_t *>(p);
}

// 8x8 b16 transpose across the warp (fragment layout of mma.m16n8k16).
__device__ __forceinline__ uint32_t movmatrix_t(uint32_t x)
{
    uint32_t y;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(y) : "r"(x));
    return y;
}

// One warp per (query, KV head[, key split]).  Scores are computed
// transposed, S^T = K Q^T: the 16 keys of a chunk are the MMA rows and the
// G query heads the columns (NT tiles of 8), so a chunk takes 8 MMAs per
// column tile for S^T and 8 for O^T += V^T P^T, with no rows wasted on
// padding heads.  Lane (r0 = lane / 4, c = lane % 4) holds keys r0, r0 + 8 of
// heads 2c, 2c + 1 of each column tile, and keeps the running max / sum of
// those two heads; P^T turns into the B operand of the PV product by one
// movmatrix transpose per 8 x 8 block.
//
// PH (position-range phases, AttnArgs::state_o set): the launch runs one KV
// head phase_g and one key range phase_r for every query (one warp per
// query): the query's list entries in that range, starting from the running
// result the earlier ranges left in state_o / state_ml (nothing yet when the
// running max is -inf).  The warp whose range holds the query's last entry
// writes the normalised output and lse; the others write the running result
// back.  K/V rows are fetched with an L2 evict-last policy and the
// per-query data with evict-first, so the range's rows stay in L2 while
// every query reads them.
template <int NT, bool PH, int NS>
__global__ void __launch_bounds__(AWARPS * 32) k_attn(AttnArgs a, int keys_per_split)
{
    extern __shared__ __align__(128) uint8_t asmem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t unit = (int64_t)blockIdx.x * AWARPS + warp;
    const int64_t total = PH ? a.nq : a.nq * a.Hkv * a.nsplit;
    if (unit >= total) return;
    // head-major order: the warps in flight all read one KV head, whose rows
    // (Tk x 512 B of K+V) stay resident in L2 while its queries run
    const int split = PH ? 0 : (int)(unit % a.nsplit);
    const int64_t qg = PH ? unit : unit / a.nsplit;
    const int g = PH ? a.phase_g : (int)(qg / a.nq);
    const int64_t q = PH ? unit : qg % a.nq;
    const int G = a.Hq / a.Hkv;
    const int r0 = lane >> 2, c = lane & 3;
    // B operand Q^T: dims 2c, 2c + 1 (and + 8) of dim block kk, head 8 nt + r0.
    // Q is not written by the kernels this one waits for (the index lists),
    // so it is loaded before the wait.
    const uint16_t *Qb = a.Q + ((q * a.Hq) + (int64_t)g * G) * LSA_HEAD;
    uint32_t qb[NT][8][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int h = nt * 8 + r0;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            qb[nt][kk][0] = h < G ? ld_u32(Qb + h * LSA_HEAD + kk * 16 + 2 * c) : 0u;
            qb[nt][kk][1] = h < G ? ld_u32(Qb + h * LSA_HEAD + kk * 16 + 8 + 2 * c) : 0u;
        }
    }
    pdl_wait();
    pdl_release();
    const int len = min(a.lens[q], a.Lmax);
    if (lane == 0 && split == 0 && (!PH || (a.phase_g == 0 && a.phase_r == 0)))
        (void)LSA_IN_BOUNDS(a.lens[q] >= 0 && a.lens[q] <= a.Lmax, BOUNDS_LIST);
    // with a near-set plan the sink prefix and window suffix were done densely
    const int2 plan = (!PH && a.near_plan) ? a.near_plan[q] : make_int2(0, 0);
    const int lend = max(plan.x, len - plan.y);
    int begin, end;
    bool last = true;  // this warp writes the query's output
    if (PH) {
        const int32_t *ro = a.range_off + q * (int64_t)(a.n_ranges + 1) + a.phase_r;
        begin = ro[0];
        end = min(ro[1], len);
        last = (begin < end && end == len) || (len <= 0 && a.phase_r == 0);
        if (begin >= end && !last) return;  // nothing of this query in the range
    } else {
        begin = plan.x + split * keys_per_split;
        end = min(lend, begin + keys_per_split);
    }
    const int nch = end > begin ? (end - begin + KCH - 1) / KCH : 0;
    uint64_t pol_kv = 0, pol_q = 0;
    if (PH) {
        asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;\n" : "=l"(pol_kv));
        asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;\n" : "=l"(pol_q));
    }
    const uint32_t sbase = smem_u32(asmem + warp * NS * STAGE_BYTES);
    const int32_t *lst = a.lists + q * (int64_t)a.Lmax;

    auto fetch_idx = [&](int ch) {
        const int base = begin + ch * KCH;
        int v = -1;
        if (lane < KCH && ch < nch && base + lane < end) {
            v = lst[base + lane];
            // debug build: entries of a list lie in [0, Tk) and strictly increase
            if (!LSA_IN_BOUNDS(v >= 0 && v < a.Tk && (base + lane == 0 || lst[base + lane - 1] < v), BOUNDS_LIST))
                v = -1;
        }
        return v;
    };
    // lane's list entry in each of the next NS - 1 chunks to issue: the
    // entries of a chunk are loaded NS - 1 issues ahead of its rows
    int pre[NS - 1];
#pragma unroll
    for (int j = 0; j < NS - 1; ++j) pre[j] = fetch_idx(j);
    auto load = [&](int ch, int st) {
        int my = pre[0];
#pragma unroll
        for (int j = 0; j < NS - 2; ++j) pre[j] = pre[j + 1];
        pre[NS - 2] = fetch_idx(ch + NS - 1);
        if (my >= a.Tk) my = -1;  // out-of-range entries are read as zeros, never fetched
        const uint32_t sK = sbase + st * STAGE_BYTES;
        const uint32_t sV = sK + KCH * ROWB * 2;
#pragma unroll
        for (int it = 0; it < 8; ++it) {
            const int lin = it * 32 + lane;
            const int row = lin >> 4, seg = lin & 15;
            const int idx = __shfl_sync(LSA_FULL, my, row);
            const int64_t off = ((int64_t)(idx < 0 ? 0 : idx) * a.Hkv + g) * LSA_HEAD + seg * 8;
            const int bytes = idx < 0 ? 0 : 16;
            const uint32_t so = tile_off(row, seg);
            if (PH) {
                cp_async16_hint(sK + so, a.K + off, bytes, pol_kv);
                cp_async16_hint(sV + so, a.V + off, bytes, pol_kv);
            } else {
                cp_async16(sK + so, a.K + off, bytes);
                cp_async16(sV + so, a.V + off, bytes);
            }
        }
        cp_commit();
    };

    float o[NT][8][4];  // O^T: dims 16 mt + r0 (+ 8) x heads 8 nt + 2c (+ 1)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int mt = 0; mt < 8; ++mt)
#pragma unroll
            for (int j = 0; j < 4; ++j) o[nt][mt][j] = 0.0f;
    const float NEG = __int_as_float(0xff800000);
    float m[NT][2], l[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) m[nt][0] = m[nt][1] = NEG, l[nt][0] = l[nt][1] = 0.0f;
    const float sl2 = a.scale * LOG2E;
#pragma unroll
    for (int s = 0; s < NS - 1; ++s) {
        if (s < nch) load(s, s);
        else cp_commit();
    }
    if (PH) {  // the running result of the earlier ranges, if any (read while the first rows are in flight)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int h = nt * 8 + 2 * c + e;
                if (h >= G) continue;
                const int64_t row = (q * a.Hq) + (int64_t)g * G + h;
                const float2 ml = ld_f2_hint(a.state_ml + row * 2, pol_q);
                if (ml.x == NEG) continue;
                m[nt][e] = ml.x;
                l[nt][e] = ml.y;
                const float *so = a.state_o + row * LSA_HEAD;
#pragma unroll
                for (int mt = 0; mt < 8; ++mt) {
                    o[nt][mt][e] = ld_f_hint(so + mt * 16 + r0, pol_q);
                    o[nt][mt][2 + e] = ld_f_hint(so + mt * 16 + 8 + r0, pol_q);
                }
            }
    }

    for (int ch = 0; ch < nch; ++ch) {
        const int nxt = ch + NS - 1;
        if (nxt < nch) load(nxt, nxt % NS);
        else cp_commit();
        cp_wait<NS - 1>();
        __syncwarp();
        const uint32_t sK = sbase + (ch % NS) * STAGE_BYTES;
        const uint32_t sV = sK + KCH * ROWB * 2;
        float s[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int j = 0; j < 4; ++j) s[nt][j] = 0.0f;
        {
            // A = K chunk (16 keys x 16 dims): matrix mm = lane / 8 is keys
            // 8 (mm & 1) .., dims 8 (mm >> 1) ..
            const int key = (lane & 7) + (((lane >> 3) & 1) << 3);
            const int dsub = (lane >> 4) << 3;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                uint32_t ka[4];
                ldsm_x4(ka, sK + tile_off(key, 2 * kk + (dsub >> 3)));
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) mma16816(s[nt], ka, qb[nt][kk][0], qb[nt][kk][1]);
            }
        }
        const int base = begin + ch * KCH;
        const bool v0 = base + r0 < end, v1 = base + r0 + 8 < end;
        uint32_t pb[NT][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            s[nt][0] = v0 ? s[nt][0] * sl2 : NEG;
            s[nt][1] = v0 ? s[nt][1] * sl2 : NEG;
            s[nt][2] = v1 ? s[nt][2] * sl2 : NEG;
            s[nt][3] = v1 ? s[nt][3] * sl2 : NEG;
            // column (head) maxima over the 16 keys: lanes with equal c
            float mx0 = fmaxf(s[nt][0], s[nt][2]), mx1 = fmaxf(s[nt][1], s[nt][3]);
#pragma unroll
            for (int o2 = 4; o2 < 32; o2 <<= 1) {
                mx0 = fmaxf(mx0, __shfl_xor_sync(LSA_FULL, mx0, o2));
                mx1 = fmaxf(mx1, __shfl_xor_sync(LSA_FULL, mx1, o2));
            }
            const float mn0 = fmaxf(m[nt][0], mx0), mn1 = fmaxf(m[nt][1], mx1);
            const float al0 = exp2f(m[nt][0] - mn0), al1 = exp2f(m[nt][1] - mn1);
            s[nt][0] = exp2f(s[nt][0] - mn0);
            s[nt][1] = exp2f(s[nt][1] - mn1);
            s[nt][2] = exp2f(s[nt][2] - mn0);
            s[nt][3] = exp2f(s[nt][3] - mn1);
            float rs0 = s[nt][0] + s[nt][2], rs1 = s[nt][1] + s[nt][3];
#pragma unroll
            for (int o2 = 4; o2 < 32; o2 <<= 1) {
                rs0 += __shfl_xor_sync(LSA_FULL, rs0, o2);
                rs1 += __shfl_xor_sync(LSA_FULL, rs1, o2);
            }
            l[nt][0] = l[nt][0] * al0 + rs0;
            l[nt][1] = l[nt][1] * al1 + rs1;
            m[nt][0] = mn0;
            m[nt][1] = mn1;
            if (al0 != 1.0f || al1 != 1.0f) {  // the running max moved: rescale O^T
#pragma unroll
                for (int mt = 0; mt < 8; ++mt) {
                    o[nt][mt][0] *= al0;
                    o[nt][mt][1] *= al1;
                    o[nt][mt][2] *= al0;
                    o[nt][mt][3] *= al1;
                }
            }
            // P^T blocks (keys r0 / r0 + 8, heads 2c, 2c + 1) -> B fragments
            pb[nt][0] = movmatrix_t(pack_bf16(s[nt][0], s[nt][1]));
            pb[nt][1] = movmatrix_t(pack_bf16(s[nt][2], s[nt][3]));
        }
        {
            // A = V^T (16 dims x 16 keys) by transposing loads of V rows:
            // matrix mm = lane / 8 is dims 8 (mm & 1) .., keys 8 (mm >> 1) ..
            const int key = (lane & 7) + ((lane >> 4) << 3);
            const int dsub = ((lane >> 3) & 1) << 3;
#pragma unroll
            for (int mt = 0; mt < 8; ++mt) {
                uint32_t va[4];
                ldsm_x4_t(va, sV + tile_off(key, 2 * mt + (dsub >> 3)));
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) mma16816(o[nt][mt], va, pb[nt][0], pb[nt][1]);
            }
        }
        __syncwarp();
    }
    cp_wait<0>();

    if (PH && !last) {  // the running result goes back for the next range
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int h = nt * 8 + 2 * c + e;
                if (h >= G) continue;
                const int64_t row = (q * a.Hq) + (int64_t)g * G + h;
                float *so = a.state_o + row * LSA_HEAD;
#pragma unroll
                for (int mt = 0; mt < 8; ++mt) {
                    st_f_hint(so + mt * 16 + r0, o[nt][mt][e], pol_q);
                    st_f_hint(so + mt * 16 + 8 + r0, o[nt][mt][2 + e], pol_q);
                }
                if (r0 == 0) st_f2_hint(a.state_ml + row * 2, make_float2(m[nt][e], l[nt][e]), pol_q);
            }
    } else if (a.nsplit == 1) {
        if (plan.x | plan.y) {  // merge the near-set partial results
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int h = nt * 8 + 2 * c + e;
                    if (h >= G) continue;
                    const int64_t row = (q * a.Hq) + (int64_t)g * G + h;
                    const float2 ml = *reinterpret_cast<const float2 *>(a.near_ml + row * 2);
                    const float M = fmaxf(m[nt][e], ml.x);
                    const float ws_ = m[nt][e] == NEG ? 0.0f : exp2f(m[nt][e] - M);
                    const float wd = ml.x == NEG ? 0.0f : exp2f(ml.x - M);
                    l[nt][e] = l[nt][e] * ws_ + ml.y * wd;
                    m[nt][e] = M;
                    const float *po = a.near_o + row * LSA_HEAD;
#pragma unroll
                    for (int mt = 0; mt < 8; ++mt) {
                        o[nt][mt][e] = o[nt][mt][e] * ws_ + po[mt * 16 + r0] * wd;
                        o[nt][mt][2 + e] = o[nt][mt][2 + e] * ws_ + po[mt * 16 + 8 + r0] * wd;
                    }
                }
        }
        uint16_t *Ob = a.O + ((q * a.Hq) + (int64_t)g * G) * LSA_HEAD;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const float i0 = l[nt][0] > 0.0f ? 1.0f / l[nt][0] : 0.0f;
            const float i1 = l[nt][1] > 0.0f ? 1.0f / l[nt][1] : 0.0f;
            const int h = nt * 8 + r0;  // after the transpose: head row r0, dims 2c, 2c + 1
#pragma unroll
            for (int mt = 0; mt < 8; ++mt) {
                const uint32_t lo = movmatrix_t(pack_bf16(o[nt][mt][0] * i0, o[nt][mt][1] * i1));
                const uint32_t hi = movmatrix_t(pack_bf16(o[nt][mt][2] * i0, o[nt][mt][3] * i1));
                if (h < G) {
                    *reinterpret_cast<uint32_t *>(Ob + h * LSA_HEAD + mt * 16 + 2 * c) = lo;
                    *reinterpret_cast<uint32_t *>(Ob + h * LSA_HEAD + mt * 16 + 8 + 2 * c) = hi;
                }
            }
            if (r0 == 0 && a.lse) {
                if (nt * 8 + 2 * c < G) a.lse[q * a.Hq + g * G + nt * 8 + 2 * c] = m[nt][0] * LN2 + logf(l[nt][0]);
                if (nt * 8 + 2 * c + 1 < G)
                    a.lse[q * a.Hq + g * G + nt * 8 + 2 * c + 1] = m[nt][1] * LN2 + logf(l[nt][1]);
            }
        }
    } else {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int h = nt * 8 + 2 * c + e;
                if (h >= G) continue;
                const int64_t pidx = ((q * a.Hq) + (int64_t)g * G + h) * a.nsplit + split;
                float *po = a.part_o + pidx * LSA_HEAD;
#pragma unroll
                for (int mt = 0; mt < 8; ++mt) {
                    po[mt * 16 + r0] = o[nt][mt][e];
                    po[mt * 16 + 8 + r0] = o[nt][mt][2 + e];
                }
                if (r0 == 0) {
                    a.part_ml[pidx * 2] = m[nt][e];
                    a.part_ml[pidx * 2 + 1] = l[nt][e];
                }
            }
    }
}

// Merge the partial results of the key splits of one (query, head): one
// 256-thread CTA.  Warp w takes the splits w, w + 8, .. in batches of
// CB_BATCH; lane i loads dims 4i .. 4i + 3 of each of its splits'
// unnormalised outputs (16-byte loads) and the splits' (max, sum) records
// before the maximum M over all splits is known, so the partials arrive in
// one round trip; the weights 2^(m_s - M) then scale them (a split with no
// key weighs 0), and the warps' sums are added in shared memory.
constexpr int CB_THREADS = 256;
constexpr int CB_WARPS = CB_THREADS / 32;
constexpr int CB_BATCH = 8;
__global__ void __launch_bounds__(CB_THREADS) k_attn_combine(AttnArgs a)
{
    pdl_wait();
    pdl_release();
    __shared__ float red[2][CB_WARPS];
    __shared__ float4 part[CB_WARPS][32];
    const int64_t unit = blockIdx.x;
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const float NEG = __int_as_float(0xff800000);
    const int ns = a.nsplit;
    const float2 *ml = reinterpret_cast<const float2 *>(a.part_ml + unit * ns * 2);
    const float4 *po = reinterpret_cast<const float4 *>(a.part_o + unit * ns * LSA_HEAD) + lane;
    float4 x[CB_BATCH];
    float2 r[CB_BATCH];
    auto fetch = [&](int b0) {
#pragma unroll
        for (int j = 0; j < CB_BATCH; ++j) {
            const int sp = b0 + warp + j * CB_WARPS;
            r[j] = sp < ns ? ml[sp] : make_float2(NEG, 0.0f);
            x[j] = sp < ns ? po[(int64_t)sp * (LSA_HEAD / 4)] : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        }
    };
    fetch(0);
    float M = NEG;
    for (int sp = t; sp < ns; sp += CB_THREADS) {
        const float2 v = ml[sp];
        if (v.y > 0.0f) M = fmaxf(M, v.x);
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) M = fmaxf(M, __shfl_xor_sync(LSA_FULL, M, o));
    if (lane == 0) red[0][warp] = M;
    __syncthreads();
    M = red[0][0];
#pragma unroll
    for (int w = 1; w < CB_WARPS; ++w) M = fmaxf(M, red[0][w]);
    float L = 0.0f;
    for (int sp = t; sp < ns; sp += CB_THREADS) {
        const float2 v = ml[sp];
        if (v.y > 0.0f) L += v.y * exp2f(v.x - M);
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) L += __shfl_xor_sync(LSA_FULL, L, o);
    if (lane == 0) red[1][warp] = L;
    float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    for (int b0 = 0;;) {  // warp-uniform
#pragma unroll
        for (int j = 0; j < CB_BATCH; ++j) {
            if (r[j].y > 0.0f) {
                const float w = exp2f(r[j].x - M);
                acc.x += x[j].x * w;
                acc.y += x[j].y * w;
                acc.z += x[j].z * w;
                acc.w += x[j].w * w;
            }
        }
        b0 += CB_BATCH * CB_WARPS;
        if (b0 >= ns) break;
        fetch(b0);
    }
    part[warp][lane] = acc;
    __syncthreads();
    if (warp == 0) {
        acc = part[0][lane];
        L = red[1][0];
#pragma unroll
        for (int w = 1; w < CB_WARPS; ++w) {
            const float4 y = part[w][lane];
            acc.x += y.x;
            acc.y += y.y;
            acc.z += y.z;
            acc.w += y.w;
            L += red[1][w];
        }
        const float inv = L > 0.0f ? 1.0f / L : 0.0f;
        const uint32_t lo = pack_bf16(acc.x * inv, acc.y * inv), hi = pack_bf16(acc.z * inv, acc.w * inv);
        *reinterpret_cast<uint2 *>(a.O + unit * LSA_HEAD + lane * 4) = make_uint2(lo, hi);
        if (lane == 0 && a.lse) a.lse[unit] = M * LN2 + logf(L);
    }
}

// ---------------------------------------------------------------------------
// Near set, shared by consecutive queries.  A list written by the indexer
// ends with the window [p - window, p] and starts with the sink keys
// 0 .. sink - 1; consecutive queries (positions p, p + 1, ...) read almost
// the same window rows.  The near-set kernel takes, per query, the longest run of
// consecutive positions that ends the list (at most NEAR_DMAX keys, the last
// being p) and the run 0, 1, .. that starts it (at most NEAR_SMAX keys,
// disjoint from the first), read from the list itself, so any strictly
// increasing list is handled.  A CTA takes a tile of NEAR_ROWS / G
// consecutive queries and one KV head: the union of the tile's near keys
// streams through shared memory once, 64 keys at a time, and every query
// head of the tile is a row of a 128 x 64 score tile on the tensor cores
// (k_attn_near_tc, lsa_near_tc.cu: tcgen05 with TMEM accumulators, fp32
// online softmax masked per row to the query's own keys).  The partial
// results (unnormalised O, reference max, sum) go to the workspace; k_attn
// then reads only the rest of each list and merges.  A tile
// whose queries do not sit at consecutive positions gets an empty plan and
// k_attn reads those lists whole.
constexpr int NEAR_DMAX = 1024;  // longest window suffix taken densely
constexpr int NEAR_SMAX = 16;    // longest sink prefix taken densely

// Plan of one tile (one CTA of NEAR_ROWS threads): per query p = its last
// listed position, d = the run of consecutive positions that ends the list,
// s = the run 0, 1, .. that starts it, disjoint from the first (binary
// searches: lists strictly increase).  The tile is usable when its queries
// sit at consecutive positions; otherwise every plan is (0, 0).
__global__ void __launch_bounds__(NEAR_ROWS) k_near_plan(AttnArgs a)
{
    __shared__ int t_p[NEAR_ROWS], t_d[NEAR_ROWS], t_s[NEAR_ROWS];
    __shared__ int t_ok;
    const int QT = near_tile_queries(a.Hq / a.Hkv);
    const int64_t q0 = (int64_t)blockIdx.x * QT;
    const int nt_q = (int)min((int64_t)QT, a.nq - q0);
    const int t = threadIdx.x;
    if (t == 0) t_ok = 1;
    __syncthreads();
    if (t < nt_q) {
        const int64_t q = q0 + t;
        const int32_t *lst = a.lists + q * (int64_t)a.Lmax;
        const int len = min(a.lens[q], a.Lmax);
        (void)LSA_IN_BOUNDS(a.lens[q] >= 0 && a.lens[q] <= a.Lmax, BOUNDS_LIST);
        int p = -1, d = 0, s = 0;
        if (len >= 1) {
            p = lst[len - 1];
            int lo = 1, hi = min(len, NEAR_DMAX);
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (lst[len - mid] == p - mid + 1) lo = mid;
                else hi = mid - 1;
            }
            d = lo;
            int slo = 0, shi = min(len - d, NEAR_SMAX);
            while (slo < shi) {
                const int mid = (slo + shi + 1) >> 1;
                if (lst[mid - 1] == mid - 1) slo = mid;
                else shi = mid - 1;
            }
            s = slo;
        }
        t_p[t] = p;
        t_d[t] = d;
        t_s[t] = s;
        if (len < 1 || p - d + 1 < 0 || (int64_t)p >= a.Tk) t_ok = 0;
    }
    __syncthreads();
    if (t < nt_q && t_p[t] != t_p[0] + t) t_ok = 0;
    __syncthreads();
    const bool ok = t_ok != 0;
    if (t < nt_q) a.near_plan[q0 + t] = ok ? make_int2(t_s[t], t_d[t]) : make_int2(0, 0);
    if (t == 0) {
        int lo = t_p[0], smax = 0;
        for (int i = 0; i < nt_q; ++i) {
            lo = min(lo, t_p[i] - t_d[i] + 1);
            smax = max(smax, t_s[i]);
        }
        a.near_tile[blockIdx.x] = make_int4(ok ? 1 : 0, t_p[0], lo, smax);
    }
}


int attention_list_cap()
{
    return 1 << 30;  // the list is streamed, not staged: any length
}

// Plan of the phased gather: per query, the index of its first list entry at
// or past each range start (a lower bound in the ascending list; the last
// bound is the list length), and its running results set to "nothing yet".
// One warp per query, one lane per range bound.
__global__ void __launch_bounds__(256) k_range_plan(AttnArgs a)
{
    pdl_wait();
    pdl_release();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t q = (int64_t)blockIdx.x * 8 + warp;
    if (q >= a.nq) return;
    const int len = max(0, min(a.lens[q], a.Lmax));
    const int32_t *lst = a.lists + q * (int64_t)a.Lmax;
    int32_t *ro = a.range_off + q * (int64_t)(a.n_ranges + 1);
    for (int r = lane; r <= a.n_ranges; r += 32) {
        int lo = len;
        if (r < a.n_ranges) {
            const int64_t b = (int64_t)r * a.range_rows;
            int hi = len;
            lo = 0;
            while (lo < hi) {
                const int mid = (lo + hi) >> 1;
                if ((int64_t)lst[mid] < b) lo = mid + 1;
                else hi = mid;
            }
        }
        ro[r] = lo;
    }
    float2 *ml = reinterpret_cast<float2 *>(a.state_ml) + q * a.Hq;
    for (int h = lane; h < a.Hq; h += 32) ml[h] = make_float2(__int_as_float(0xff800000), 0.0f);
}

cudaError_t launch_attention(const AttnArgs &a, cudaStream_t st, int n_sm)
{
    (void)n_sm;
    if (a.nq <= 0) return cudaSuccess;
    const int smem = AWARPS * NST * STAGE_BYTES;
    const int G = a.Hq / a.Hkv;
    cudaError_t e;
    if (a.state_o) {  // position-range phases: one launch per (KV head, range)
        auto kph = G <= 8 ? k_attn<1, true, NST> : k_attn<2, true, NST>;
        if ((e = cudaFuncSetAttribute(kph, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) != cudaSuccess)
            return e;
        int kt = kt_begin("k_range_plan", st);
        k_range_plan<<<(unsigned)((a.nq + 7) / 8), 256, 0, st>>>(a);
        kt_end(kt, st);
        count_launches(1);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        kt = kt_begin("k_attn", st);
        AttnArgs b = a;
        const unsigned blocks = (unsigned)((a.nq + AWARPS - 1) / AWARPS);
        for (int g = 0; g < a.Hkv; ++g)
            for (int r = 0; r < a.n_ranges; ++r) {
                b.phase_g = g;
                b.phase_r = r;
                // each launch waits for the previous one's results (griddepcontrol.wait) but its launch
                // overlaps the previous one's tail
                e = launch_k(true, kph, dim3(blocks), dim3(AWARPS * 32), (size_t)smem, st, b, 0);
                if (e != cudaSuccess) {
                    kt_end(kt, st);
                    return e;
                }
            }
        kt_end(kt, st);
        count_launches(a.Hkv * a.n_ranges);
        return cudaSuccess;
    }
    // split lists (few queries): few warps, so deeper rings (one CTA per SM)
    const bool split = a.nsplit > 1;
    auto kern = split ? (G <= 8 ? k_attn<1, false, NST_SPLIT> : k_attn<2, false, NST_SPLIT>)
                      : (G <= 8 ? k_attn<1, false, NST> : k_attn<2, false, NST>);
    const int smem_g = AWARPS * (split ? NST_SPLIT : NST) * STAGE_BYTES;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_g);
    if (e != cudaSuccess) return e;
    int kps = (a.Lmax + a.nsplit - 1) / a.nsplit;
    kps = ((kps + KCH - 1) / KCH) * KCH;
    if (a.near_plan) {  // near sets of consecutive queries first (plans + partials)
        const int QT = near_tile_queries(G);
        const unsigned tiles = (unsigned)((a.nq + QT - 1) / QT);
        int kt = kt_begin("k_near_plan", st);
        k_near_plan<<<tiles, NEAR_ROWS, 0, st>>>(a);
        kt_end(kt, st);
        kt = kt_begin("k_attn_near_tc", st);
        e = launch_attention_near_tc(a, (int)tiles, st);
        kt_end(kt, st);
        if (e != cudaSuccess) return e;
        count_launches(2);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    const int64_t units = a.nq * a.Hkv * a.nsplit;
    const int64_t blocks = (units + AWARPS - 1) / AWARPS;
    // split lists (few queries, decode): short kernels, launched back to back
    int kt = kt_begin("k_attn", st);
    e = launch_k(split, kern, dim3((unsigned)blocks), dim3(AWARPS * 32), (size_t)smem_g, st, a, kps);
    kt_end(kt, st);
    if (e != cudaSuccess) return e;
    count_launches(1);
    if (a.nsplit > 1) {
        kt = kt_begin("k_attn_combine", st);
        e = launch_k(true, k_attn_combine, dim3((unsigned)(a.nq * a.Hq)), dim3(CB_THREADS), 0, st, a);
        kt_end(kt, st);
        count_launches(1);
    }
    return e;
}

// this file's bounds-check word (debug build; always 0 in the release build)
LSA_BOUNDS_READER(read_bounds_error_attn)

}  // namespace lsa
