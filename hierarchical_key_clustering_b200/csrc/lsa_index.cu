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
// P = ceil((k + sink + window) / 4).  Pass 1 scores every bucket and
// histograms the maximum of each group of g consecutive buckets (g a power of
// two giving 4P..8P groups).  The P-th largest group maximum is a score of P
// distinct buckets, so it is <= the P-th largest score, and so is tau, the
// lower edge of its histogram bin: every bucket scoring at least tau is a
// candidate.  Pass 2 recomputes the same scores bit for bit on the tensor
// cores (lsa_score_tc.cu) or, for <= 16 queries, reads the scores pass 1
// stored (k_dscore streams the centroids once on the CUDA cores), and appends
// every aligned group of 4 buckets whose best score is >= tau as one entry.
// The expansion kernel keeps the scores >= tau, ranks them by (score desc,
// id asc) and expands them; a query whose entries or candidates overflow
// their slots is redone exactly there (radix select on recomputed scores).
//
// Several index heads per token (N-LSA's selection by the best head score):
// the Flat passes run over one row per (query, head), and k_heads_merge
// turns each query's rows into one candidate set for the same expansion.
#include "lsa_common.cuh"
#include "lsa_kernels.h"

namespace lsa {


// ---------------------------------------------------------------------------
// One warp per row; a row is one index query, `heads` consecutive rows per
// token (all with that token's horizon).
__global__ void __launch_bounds__(256) k_qnorm(const float *__restrict__ qidx, const int64_t *__restrict__ pos,
                                               int64_t nq, int heads, int64_t pos_shift, int64_t n_blocks, IndexWs ws)
{
    pdl_wait();
    pdl_release();
    const int lane = threadIdx.x & 31;
    const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t q = warp; q < nq; q += nwarps) {
        float a = qidx[q * LSA_D + lane], b = qidx[q * LSA_D + lane + 32];
        warp_normalize(a, b);
        ws.qhat[q * LSA_D + lane] = f2bf_bits(a);
        ws.qhat[q * LSA_D + lane + 32] = f2bf_bits(b);
        if (lane == 0) {
            int64_t p = pos[q / heads] - pos_shift;  // shift: first position of a shard's cache
            int64_t H = p < 0 ? 0 : p / LSA_BLK;
            if (H > n_blocks) H = n_blocks;
            ws.horizon[q] = (int32_t)H;
            ws.cnt[q] = 0;
        }
        for (int i = lane; i < HIST_BINS; i += 32) ws.ghist[q * HIST_BINS + i] = 0u;
    }
}

// Score of one bucket on the CUDA cores: fp32 FMA chain over d = 0..63 of the
// bf16 operands (the exact selections of a query whose candidates overflowed
// or whose sampled threshold kept too little).  It can differ from the tensor
// cores' sum of the same products in the last bit, which only matters for
// scores within ~1e-6 of each other, at the one cut a Flat search makes.
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
// Radix select over scores: the P-th largest f2ord(get(i)), i in [0, n).
template <typename Get>
__device__ uint32_t block_select_kth_largest(int64_t n, int64_t P, Get get, int *hist, int *sh)
{
    return block_select_ord(n, P, [&](int64_t i) { return f2ord(get(i)); }, hist, sh);
}

// ---------------------------------------------------------------------------
// Tree beam search, level by level from the root, one query per team of TEAM
// warps (teams of a CTA are independent: TEAM = 2 for many queries, 8 for a
// few).  Per level the candidates are gathered, scored and the best B kept.
// Keeping the best B is a selection, not a sort: a 256-bin histogram of the
// scores over their own [min, max] range finds the bin holding the B-th best;
// the bins above it are kept whole, and the boundary bin's members are ranked
// exactly by their rank keys (score desc, id asc): by pairwise counting when
// they are few, by a radix select over the 64-bit keys otherwise.  Rank keys
// are unique, so the kept set is the one a full sort gives; its order is free
// (the expansion ranks the entries itself).
//
// Candidate slots: the children of kept node i sit at slots 2i and 2i + 1 (a
// node with one child leaves a hole, key ~0, skipped everywhere), then the
// visible nodes whose parent is not visible.  Centroid rows are scored from
// shared memory: a warp copies 32 rows with coalesced 16-byte loads (eight
// lanes per row, so one load instruction touches 4 lines, not 32), then each
// lane scores one row.
constexpr int TB_BINS = 256;
constexpr int TB_SMALL = 128;  // boundary members ranked by pairwise counting
constexpr int TB_STAGE = 32 * LSA_D * 2;  // bytes of one warp's staged rows
constexpr uint64_t TB_HOLE = ~0ull;
// many queries: teams of BEAM_TEAM warps, BEAM_MINB CTAs per SM sharing its
// 228 KB of shared memory (1 KB of which each CTA reserves)
constexpr int BEAM_TEAM = 2, BEAM_MINB = 3;
constexpr size_t SM_SMEM = 233472;

// Shared memory of one team: qd double[64] | hist int[256] (later the
// boundary list, uint64[128]) | ctl int[16] | red float[32] (two per warp of
// a team of up to 16) | keys uint64[CM] | kept int32[KM] | staged rows,
// TB_STAGE bytes per warp.
constexpr int TB_KEYS_OFF = 512 + 1024 + 64 + 128;
__host__ __device__ __forceinline__ size_t tree_beam_keys_bytes(int CM) { return (8 * (size_t)CM + 15) & ~(size_t)15; }
__host__ __device__ __forceinline__ size_t tree_beam_kept_bytes(int KM) { return (4 * (size_t)KM + 15) & ~(size_t)15; }
__host__ __device__ __forceinline__ size_t tree_beam_team_bytes(int CM, int KM, int team_warps)
{
    return TB_KEYS_OFF + tree_beam_keys_bytes(CM) + tree_beam_kept_bytes(KM) + (size_t)team_warps * TB_STAGE;
}

// Barrier of one team: a warp barrier for one warp, else the named barrier
// 1 + team over the team's 32 TEAM threads (teams of a CTA never wait on one
// another).
template <int TEAM>
__device__ __forceinline__ void team_sync(int team)
{
    if constexpr (TEAM == 1) __syncwarp();
    else asm volatile("bar.sync %0, %1;\n" ::"r"(team + 1), "r"(TEAM * 32) : "memory");
}

// Team-wide sum of an int; every thread returns it.
template <int TEAM>
__device__ __forceinline__ int team_sum(int x, int *red, int team)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(LSA_FULL, x, o);
    if constexpr (TEAM > 1) {
        const int w = (threadIdx.x >> 5) % TEAM;
        if ((threadIdx.x & 31) == 0) red[w] = x;
        team_sync<TEAM>(team);
        x = 0;
#pragma unroll
        for (int k = 0; k < TEAM; ++k) x += red[k];
        team_sync<TEAM>(team);
    }
    return x;
}

// Team-wide minimum and maximum; every thread returns both.
template <int TEAM>
__device__ __forceinline__ void team_min_max(float &lo, float &hi, float *red, int team)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        lo = fminf(lo, __shfl_xor_sync(LSA_FULL, lo, o));
        hi = fmaxf(hi, __shfl_xor_sync(LSA_FULL, hi, o));
    }
    if constexpr (TEAM > 1) {
        const int w = (threadIdx.x >> 5) % TEAM;
        if ((threadIdx.x & 31) == 0) {
            red[w] = lo;
            red[TEAM + w] = hi;
        }
        team_sync<TEAM>(team);
        lo = red[0];
        hi = red[TEAM];
#pragma unroll
        for (int k = 1; k < TEAM; ++k) {
            lo = fminf(lo, red[k]);
            hi = fmaxf(hi, red[TEAM + k]);
        }
        team_sync<TEAM>(team);
    }
}

// One warp over a 256-bin histogram: the bin at which the count, taken bin by
// bin in scan order (descending bins when desc), first reaches need, and the
// count in the bins scanned before it.  Lane l owns scan positions 8l..8l+7.
__device__ __forceinline__ void warp_hist_pick(const int *h, int need, bool desc, int &sel, int &before)
{
    const int lane = threadIdx.x & 31;
    int c[8], c8 = 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        c[e] = h[desc ? 255 - 8 * lane - e : 8 * lane + e];
        c8 += c[e];
    }
    int incl = c8;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(LSA_FULL, incl, o);
        if (lane >= o) incl += y;
    }
    const int excl = incl - c8;
    int e_hit = -1, acc = excl;
    if (excl < need && need <= incl) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            if (e_hit < 0) {
                if (acc + c[e] >= need) e_hit = e;
                else acc += c[e];
            }
        }
    }
    const unsigned who = __ballot_sync(LSA_FULL, e_hit >= 0);
    const int src = who ? __ffs(who) - 1 : 0;
    e_hit = __shfl_sync(LSA_FULL, e_hit, src);
    acc = __shfl_sync(LSA_FULL, acc, src);
    if (!who) {  // need exceeds the total: cannot happen; keep the index in range
        e_hit = 7;
        acc = 0;
    }
    sel = desc ? 255 - 8 * src - e_hit : 8 * src + e_hit;
    before = acc;
}

// Score of one tree node from its staged row (16-byte segments stored at
// segment ^ sw), rounded once to fp32 from the fp64 sum over d = 0..63 of the
// bf16 products taken in that order.  A product of two bf16 values is exact
// in fp64, so each fused step rounds exactly like a separate add and the
// result is the fp32 value of a plain fp64 dot product written out in index
// order.  A beam search cuts at every level; scoring this way makes those
// cuts independent of the accumulation order.
__device__ __forceinline__ float dot_staged_f64(const double *qd, const uint4 *row, int sw)
{
    double x = 0.0;
#pragma unroll
    for (int v = 0; v < 8; ++v) {
        const uint4 w = row[v ^ sw];
        const uint32_t ua[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            const double2 qq = *reinterpret_cast<const double2 *>(qd + v * 8 + 2 * h);
            x = __fma_rn(qq.x, (double)__uint_as_float(ua[h] << 16), x);
            x = __fma_rn(qq.y, (double)__uint_as_float(ua[h] & 0xffff0000u), x);
        }
    }
    return __double2float_rn(x);
}

// Warp-aggregated append: the lanes with pred get consecutive slots from the
// shared counter *ctr (one atomic per warp); returns the lane's slot.
__device__ __forceinline__ int warp_append(bool pred, int *ctr)
{
    const int lane = threadIdx.x & 31;
    const unsigned m = __ballot_sync(LSA_FULL, pred);
    int base = 0;
    if (lane == 0 && m) base = atomicAdd(ctr, __popc(m));
    base = __shfl_sync(LSA_FULL, base, 0);
    return base + __popc(m & ((1u << lane) - 1u));
}

// TEAM warps per query, MINB CTAs per SM (register budget).
template <int TEAM, int MINB>
__global__ void __launch_bounds__(TEAM >= 8 ? 32 * TEAM : 256, MINB)
    k_tree_beam(int64_t nq, TreeView tv, int W, int P, int CM, int KM, IndexWs ws)
{
    pdl_wait();
    pdl_release();
    extern __shared__ __align__(16) unsigned char tb_smem[];
    const int lane = threadIdx.x & 31;
    static_assert(TEAM >= 1 && TEAM <= 16 && 256 / (32 * TEAM) <= 15, "team reductions hold 2 floats per warp of <= 16; barrier ids 1..15");
    constexpr int TT = TEAM * 32;
    constexpr int RUNP = (LSA_RUN + TT - 1) / TT;
    const int tw = (int)threadIdx.x % TT;
    const int wi = tw >> 5;
    const int team = (int)threadIdx.x / TT;
    const int64_t q = (int64_t)blockIdx.x * (blockDim.x / TT) + team;
    if (q >= nq) return;  // team-uniform; teams synchronise only among themselves
    unsigned char *base = tb_smem + (size_t)team * tree_beam_team_bytes(CM, KM, TEAM);
    double *qd = reinterpret_cast<double *>(base);
    int *hist = reinterpret_cast<int *>(base + 512);
    uint64_t *small = reinterpret_cast<uint64_t *>(base + 512);
    int *ctl = reinterpret_cast<int *>(base + 1536);  // 0 candidates, 1 kept, 2 boundary list, 3.. picks
    float *red = reinterpret_cast<float *>(base + 1536 + 64);
    uint64_t *keys = reinterpret_cast<uint64_t *>(base + TB_KEYS_OFF);
    int32_t *kept = reinterpret_cast<int32_t *>(base + TB_KEYS_OFF + tree_beam_keys_bytes(CM));
    uint4 *stage =
        reinterpret_cast<uint4 *>(base + TB_KEYS_OFF + tree_beam_keys_bytes(CM) + tree_beam_kept_bytes(KM)) +
        wi * (TB_STAGE / 16);
    const float NEG = __int_as_float(0xff800000);
    float4 *c4 = reinterpret_cast<float4 *>(ws.cand4) + q * ws.cap;
    int32_t *cg = ws.cand_g + q * ws.cap;
    const int2 *child2 = reinterpret_cast<const int2 *>(tv.child);

    const int H = ws.horizon[q];
    for (int d = tw; d < LSA_D; d += TT) qd[d] = (double)bf_bits2f(ws.qhat[q * LSA_D + d]);
    int n_kept = 0;
    const int top = tv.n_levels - 1;
    // Visible nodes whose parent is not visible: only the run of 128 nodes
    // holding block H can mix the two (at the top level, every visible node).
    // Each level's flags are loaded while the level above is processed.
    bool run_ok[RUNP];
    int32_t rmb[RUNP], rpar[RUNP];
    {
        const int64_t off = tv.level_offset[top], hi = min(tv.level_size[top], (int64_t)RUNP * TT);
#pragma unroll
        for (int k = 0; k < RUNP; ++k) {
            const int64_t u = k * TT + tw;
            run_ok[k] = u < hi && tv.max_block[off + u] < H;
        }
    }
    for (int l = top; l >= 0; --l) {
        const int64_t off = tv.level_offset[l];
        const int64_t offp = tv.level_offset[l + 1];
        const int nch = min(2 * n_kept, CM);  // children slots
        if (l > 0) {  // the next level's run: visibility and parents
            const int64_t rlo = ((int64_t)H >> l) * LSA_RUN;
            const int64_t rhi = min(min(rlo + LSA_RUN, tv.level_size[l - 1]), rlo + (int64_t)RUNP * TT);
            const int64_t offn = tv.level_offset[l - 1];
#pragma unroll
            for (int k = 0; k < RUNP; ++k) {
                const int64_t u = rlo + k * TT + tw;
                rmb[k] = INT_MAX;
                rpar[k] = 0;
                if (u < rhi) {
                    rmb[k] = tv.max_block[offn + u];
                    rpar[k] = tv.parent[offn + u];
                }
            }
        }
        // children of the kept nodes at fixed slots
        int holes = 0;
        for (int i = tw; i < n_kept; i += TT) {
            int2 c = __ldg(child2 + offp + kept[i]);
            if (!LSA_IN_BOUNDS(c.x < (int)tv.level_size[l], BOUNDS_NODE)) c.x = -1;
            if (!LSA_IN_BOUNDS(c.y < (int)tv.level_size[l], BOUNDS_NODE)) c.y = -1;
            if (2 * i + 1 < CM) {
                keys[2 * i] = c.x >= 0 ? (uint64_t)(uint32_t)c.x : TB_HOLE;
                keys[2 * i + 1] = c.y >= 0 ? (uint64_t)(uint32_t)c.y : TB_HOLE;
            }
            holes += (c.x < 0) + (c.y < 0);
        }
        if (tw == 0) {
            ctl[0] = nch;
            ctl[1] = ctl[2] = 0;
        }
        for (int i = tw; i < TB_BINS; i += TT) hist[i] = 0;
        team_sync<TEAM>(team);
        {
            const int64_t lo = l == top ? 0 : ((int64_t)H >> (l + 1)) * LSA_RUN;
#pragma unroll
            for (int k = 0; k < RUNP; ++k) {
                const int slot = warp_append(run_ok[k], &ctl[0]);
                if (run_ok[k] && slot < CM) keys[slot] = (uint64_t)(lo + k * TT + tw);
            }
        }
        const int nholes = team_sum<TEAM>(holes, reinterpret_cast<int *>(red), team);
        team_sync<TEAM>(team);
        const int ns = min(ctl[0], CM);  // slots
        const int n = ns - nholes;  // valid candidates
        int64_t Bl = ((int64_t)P + ((int64_t)1 << l) - 1) >> l;
        if (Bl < W) Bl = W;
        const int B = (int)min((int64_t)n, Bl);
        float smin = __int_as_float(0x7f800000), smax = NEG;
        if (n > Bl || l == 0) {
            // scores (rank keys in place of the ids), 32 staged rows at a time
            const uint16_t *crow = tv.centroid_bf16 + off * LSA_D;
            for (int c0 = wi * 32; c0 < ns; c0 += TT) {
                const int m = min(32, ns - c0);
                uint4 v[8];
                bool ok[8];
#pragma unroll
                for (int p = 0; p < 8; ++p) {
                    const int r = 4 * p + (lane >> 3);
                    const uint64_t id = r < m ? keys[c0 + r] : TB_HOLE;
                    ok[p] = id != TB_HOLE;
                    v[p] = ok[p] ? __ldg(reinterpret_cast<const uint4 *>(crow + (int64_t)(uint32_t)id * LSA_D) + (lane & 7))
                                 : make_uint4(0, 0, 0, 0);
                }
#pragma unroll
                for (int p = 0; p < 8; ++p) {
                    const int r = 4 * p + (lane >> 3);
                    if (ok[p]) stage[r * 8 + ((lane & 7) ^ (r & 7))] = v[p];
                }
                __syncwarp();
                if (lane < m) {
                    const uint64_t id = keys[c0 + lane];
                    if (id != TB_HOLE) {
                        const float s = dot_staged_f64(qd, stage + lane * 8, lane & 7);
                        keys[c0 + lane] = rank_key(s, (int32_t)(uint32_t)id);
                        smin = fminf(smin, s);
                        smax = fmaxf(smax, s);
                    }
                }
                __syncwarp();
            }
            team_sync<TEAM>(team);
            if (n > Bl) team_min_max<TEAM>(smin, smax, red, team);
        }
        // emit the key as kept (levels above the buckets) or as a candidate
        // entry (bucket level; one bucket per entry)
        auto emit = [&](uint64_t key, int slot) {
            if (l > 0) {
                if (slot < KM) kept[slot] = rank_key_id(key);
            } else if (slot < ws.cap) {
                c4[slot] = make_float4(rank_key_score(key), NEG, NEG, NEG);
                cg[slot] = rank_key_id(key);
            }
        };
        if (n <= Bl) {
            for (int b0 = 0; b0 < ns; b0 += TT) {
                const int i = b0 + tw;
                const uint64_t key = i < ns ? keys[i] : TB_HOLE;
                const int ks = warp_append(key != TB_HOLE, &ctl[1]);
                if (key != TB_HOLE) emit(key, ks);
            }
        } else {
            // monotone bin of a score over [smin, smax]; equal scores share a bin
            float scale = smax > smin ? __fdiv_rn((float)TB_BINS, __fsub_rn(smax, smin)) : 0.0f;
            if (!(scale < 1e30f)) scale = 0.0f;
            auto binof = [&](uint64_t key) -> int {
                if (key == TB_HOLE) return -1;
                const int b = (int)__fmul_rn(__fsub_rn(rank_key_score(key), smin), scale);
                return min(max(b, 0), TB_BINS - 1);
            };
            for (int i = tw; i < ns; i += TT) {
                const int b = binof(keys[i]);
                if (b >= 0) atomicAdd(&hist[b], 1);
            }
            team_sync<TEAM>(team);
            if (tw < 32) {
                int sel, before;
                warp_hist_pick(hist, B, true, sel, before);
                if (lane == 0) {
                    ctl[3] = sel;
                    ctl[4] = B - before;
                    ctl[5] = hist[sel];
                }
            }
            team_sync<TEAM>(team);
            const int bsel = ctl[3], r = ctl[4], m1 = ctl[5];
            if (m1 <= TB_SMALL) {
                // bins above the boundary kept; the boundary bin's members
                // listed, then ranked by counting
                for (int b0 = 0; b0 < ns; b0 += TT) {
                    const int i = b0 + tw;
                    uint64_t key = 0;
                    int bn = -1;
                    if (i < ns) {
                        key = keys[i];
                        bn = binof(key);
                    }
                    const int ks = warp_append(bn > bsel, &ctl[1]);
                    if (bn > bsel) emit(key, ks);
                    const int ss = warp_append(bn == bsel, &ctl[2]);
                    if (bn == bsel && ss < TB_SMALL) small[ss] = key;
                }
                team_sync<TEAM>(team);
                if (tw < 32) {
                    for (int e0 = 0; e0 < m1; e0 += 32) {
                        const int e = e0 + lane;
                        const uint64_t ke = e < m1 ? small[e] : ~0ull;
                        int rank = 0;
                        for (int j = 0; j < m1; ++j) rank += small[j] < ke;
                        const bool keep = e < m1 && rank < r;
                        const int ks = warp_append(keep, &ctl[1]);
                        if (keep) emit(ke, ks);
                    }
                }
            } else {
                // many members share the boundary bin (near-equal scores):
                // radix select of the r-th smallest rank key among them
                uint64_t prefix = 0, mask = 0;
                int rem = r;
                for (int shift = 56; shift >= 0; shift -= 8) {
                    for (int i = tw; i < TB_BINS; i += TT) hist[i] = 0;
                    team_sync<TEAM>(team);
                    for (int i = tw; i < ns; i += TT) {
                        const uint64_t key = keys[i];
                        if (binof(key) == bsel && (key & mask) == prefix)
                            atomicAdd(&hist[(int)((key >> shift) & 255u)], 1);
                    }
                    team_sync<TEAM>(team);
                    if (tw < 32) {
                        int sel, before;
                        warp_hist_pick(hist, rem, false, sel, before);
                        if (lane == 0) {
                            ctl[6] = sel;
                            ctl[7] = before;
                            ctl[8] = hist[sel];
                        }
                    }
                    team_sync<TEAM>(team);
                    prefix |= (uint64_t)ctl[6] << shift;
                    mask |= (uint64_t)255u << shift;
                    rem -= ctl[7];
                    const bool done = ctl[8] == rem;
                    team_sync<TEAM>(team);
                    if (done) break;
                }
                for (int b0 = 0; b0 < ns; b0 += TT) {
                    const int i = b0 + tw;
                    bool keep = false;
                    uint64_t key = 0;
                    if (i < ns) {
                        key = keys[i];
                        const int bn = binof(key);
                        keep = bn > bsel || (bn == bsel && (key & mask) <= prefix);
                    }
                    const int ks = warp_append(keep, &ctl[1]);
                    if (keep) emit(key, ks);
                }
            }
        }
        if (l == 0 && tw == 0) {  // tau = -inf keeps every entry
            ws.cnt[q] = B;
            ws.tau[q] = NEG;
        }
        if (l > 0) {  // parents of the next level's run sit at this level
#pragma unroll
            for (int k = 0; k < RUNP; ++k) run_ok[k] = rmb[k] < H && tv.max_block[off + rpar[k]] >= H;
        }
        n_kept = B;
        team_sync<TEAM>(team);
    }
}

// ---------------------------------------------------------------------------
// Block-wide inclusive scan of a[0..n) in shared memory.  Warp w scans the
// contiguous segment [w * seg, (w + 1) * seg) 32 elements at a time, lane i
// on element i (no bank conflicts), carrying the running total; then the
// segment totals are added in (each warp sums the totals of the warps before
// it with one shuffle reduction).  Any block size up to 1024 threads.
template <typename T>
__device__ void block_inclusive_scan(T *a, int n, T *wsum)
{
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const int seg = (((n + nw - 1) / nw) + 31) & ~31;
    const int lo = min(n, w * seg), hi = min(n, lo + seg);
    T carry = 0;
    for (int base = lo; base < hi; base += 128) {  // warp-uniform; 4 independent 32-element scans per round
        T x[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int i = base + 32 * k + lane;
            x[k] = i < hi ? a[i] : T(0);
        }
#pragma unroll
        for (int o = 1; o < 32; o <<= 1)
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const T y = __shfl_up_sync(LSA_FULL, x[k], o);
                if (lane >= o) x[k] += y;
            }
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int i = base + 32 * k + lane;
            if (i < hi) a[i] = x[k] + carry;
            carry += __shfl_sync(LSA_FULL, x[k], 31);
        }
    }
    if (lane == 0) wsum[w] = carry;
    __syncthreads();
    T before = lane < w ? wsum[lane] : T(0);
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) before += __shfl_xor_sync(LSA_FULL, before, o);
    if (before != T(0))
        for (int i = lo + lane; i < hi; i += 32) a[i] += before;
    __syncthreads();
}

// Threshold of one query from its group-maximum histogram (warp-collective,
// every lane returns it): the lower edge of the bin holding the P-th largest
// group maximum, -inf when the query has <= P groups.
__device__ float tau_from_hist(const uint32_t *h, int64_t N, int P)
{
    const int lane = threadIdx.x & 31;
    const float NEG = __int_as_float(0xff800000);
    if (n_groups(N, P) <= P) return NEG;
    // lane l owns bins 255-8l .. 248-8l (descending)
    int cb[8], c8 = 0;
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
    int bin = -1;
    if (excl < P && P <= incl) {
        int acc = excl;
        bin = HIST_BINS - 1 - 8 * lane;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            acc += cb[e];
            if (acc >= P) {
                bin = HIST_BINS - 1 - 8 * lane - e;
                break;
            }
        }
    }
    const unsigned who = __ballot_sync(LSA_FULL, bin >= 0);
    bin = who ? __shfl_sync(LSA_FULL, bin, __ffs(who) - 1) : 0;
    return bin > 0 ? hist_edge(bin) : NEG;
}

// Threshold per query from its global group-maximum histogram, for queries
// whose buckets were split over several score CTAs.  One warp per query.
__global__ void __launch_bounds__(256) k_tau(int64_t nq, int P, IndexWs ws)
{
    const int64_t q = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (q >= nq) return;
    const float t = tau_from_hist(ws.ghist + q * HIST_BINS, (int64_t)ws.horizon[q] * LSA_NBKT, P);
    if ((threadIdx.x & 31) == 0) ws.tau[q] = t;
}

// ---------------------------------------------------------------------------
// Small batches (<= SMALL_NQ queries, decode), pass 1: every score on the
// CUDA cores, each centroid row streamed once from HBM for all queries of
// the batch, stored for the filter pass, with each query's group maxima
// counted into its global histogram.  A CTA of DS_WARPS warps takes
// DS_WARPS * 128 consecutive buckets; a warp takes an aligned run of 128
// (groups are at most 128 buckets, so none straddles two warps), 32 rows at
// a time: the rows are copied with coalesced 16-byte cp.async (a warp
// instruction moves 4 whole rows) into a padded shared tile, double-buffered,
// and lane i then scores row i from there.
constexpr int DS_WARPS = 4;
constexpr int DS_SPAN = DS_WARPS * 128;
constexpr int DS_ROW = 144;  // bytes per staged row: 128 + 16 (bank-conflict-free 16-byte reads)

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, uint32_t src_bytes)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}

// NQ: the batch rounded up to a power of two (the per-query loops are
// unrolled over it, so a batch of one keeps few registers and many CTAs).
template <int NQ>
__global__ void __launch_bounds__(DS_WARPS * 32) k_dscore(int64_t nq, int64_t nb_total,
                                                          const uint16_t *__restrict__ cbf, int P, IndexWs ws)
{
    // dynamic shared memory: [DS_WARPS][2][32 * DS_ROW] staged rows, then the
    // batch's histograms [nq][HIST_BINS] and queries [nq][LSA_D]
    extern __shared__ __align__(16) uint8_t ds_dyn[];
    uint32_t *hs = reinterpret_cast<uint32_t *>(ds_dyn + DS_WARPS * 2 * 32 * DS_ROW);
    float *qf = reinterpret_cast<float *>(hs + nq * HIST_BINS);
    __shared__ int Nq[NQ], gq[NQ];
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const float NEG = __int_as_float(0xff800000);
    const int64_t wbase = (int64_t)blockIdx.x * DS_SPAN + warp * 128;
    // copy the 32 rows of round r into stage[warp][r & 1]: instruction v moves
    // rows 4v .. 4v + 3, lane l the 16 bytes l % 8 of row 4v + l / 8; rows past
    // the end are zero-filled (source clamped to row 0, nothing read)
    auto issue = [&](int r) {
        const uint32_t dst0 = (uint32_t)__cvta_generic_to_shared(ds_dyn + (warp * 2 + (r & 1)) * 32 * DS_ROW);
#pragma unroll
        for (int v = 0; v < 8; ++v) {
            const int row = 4 * v + (lane >> 3);
            const int64_t b = wbase + r * 32 + row;
            const bool ok = b < nb_total;
            cp_async16(dst0 + row * DS_ROW + (lane & 7) * 16, cbf + (ok ? b : 0) * LSA_D + (lane & 7) * 8,
                       ok ? 16u : 0u);
        }
        asm volatile("cp.async.commit_group;\n" ::: "memory");
    };
    // the centroid rows are not written by the kernel this one waits for (the
    // query normalisation), so the first two rounds are in flight before the wait
    issue(0);
    issue(1);
    pdl_wait();
    pdl_release();
    for (int i = t; i < nq * LSA_D; i += blockDim.x) qf[i] = bf_bits2f(ws.qhat[i]);
    for (int i = t; i < nq * HIST_BINS; i += blockDim.x) hs[i] = 0u;
    if (t < nq) {
        const int N = ws.horizon[t] * LSA_NBKT;
        Nq[t] = N;
        gq[t] = group_width(N, P);
    }
    __syncthreads();
    float run[NQ];
#pragma unroll
    for (int i = 0; i < NQ; ++i) run[i] = NEG;
    for (int r = 0; r < 4; ++r) {
        if (r >= 1 && r + 1 < 4) issue(r + 1);  // rounds 0 and 1 were issued above
        if (r + 1 < 4) asm volatile("cp.async.wait_group 1;\n" ::: "memory");
        else asm volatile("cp.async.wait_group 0;\n" ::: "memory");
        __syncwarp();
        const int64_t b = wbase + r * 32 + lane;
        uint32_t cw[32];
        const uint4 *src = reinterpret_cast<const uint4 *>(ds_dyn + (warp * 2 + (r & 1)) * 32 * DS_ROW + lane * DS_ROW);
#pragma unroll
        for (int v = 0; v < 8; ++v) {
            const uint4 w = src[v];
            cw[4 * v] = w.x;
            cw[4 * v + 1] = w.y;
            cw[4 * v + 2] = w.z;
            cw[4 * v + 3] = w.w;
        }
        __syncwarp();  // this buffer is refilled two rounds later
#pragma unroll
        for (int qi = 0; qi < NQ; ++qi) {
            if (qi >= nq) break;  // uniform
            const float4 *qv = reinterpret_cast<const float4 *>(qf + qi * LSA_D);
            float acc = 0.0f;
#pragma unroll
            for (int v = 0; v < 16; ++v) {
                const float4 x = qv[v];
                acc = fmaf(x.x, __uint_as_float(cw[2 * v] << 16), acc);
                acc = fmaf(x.y, __uint_as_float(cw[2 * v] & 0xffff0000u), acc);
                acc = fmaf(x.z, __uint_as_float(cw[2 * v + 1] << 16), acc);
                acc = fmaf(x.w, __uint_as_float(cw[2 * v + 1] & 0xffff0000u), acc);
            }
            const bool valid = b < Nq[qi];
            if (valid) ws.scores[qi * ws.score_stride + b] = acc;
            const int g = gq[qi];
            float m = valid ? acc : NEG;
            if (g <= 32) {
                for (int o = 1; o < g; o <<= 1) m = fmaxf(m, __shfl_xor_sync(LSA_FULL, m, o));
                if (valid && (lane & (g - 1)) == 0) atomicAdd(&hs[qi * HIST_BINS + hist_bin(m)], 1u);
            } else {
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) m = fmaxf(m, __shfl_xor_sync(LSA_FULL, m, o));
                run[qi] = fmaxf(run[qi], m);
                const int per = g >> 5;  // 2 or 4 rounds per group
                if ((r & (per - 1)) == per - 1) {
                    const int64_t gstart = wbase + (int64_t)(r - per + 1) * 32;
                    if (lane == 0 && gstart < Nq[qi]) atomicAdd(&hs[qi * HIST_BINS + hist_bin(run[qi])], 1u);
                    run[qi] = NEG;
                }
            }
        }
    }
    __syncthreads();
    for (int i = t; i < nq * HIST_BINS; i += blockDim.x) {
        const uint32_t c = hs[i];
        if (c) atomicAdd(ws.ghist + i, c);
    }
}

// Small batches, pass 2: each CTA derives every query's threshold from its
// histogram (CTA 0 also stores it), then one thread per aligned group of 4
// stored scores appends the group as a candidate entry when its best score
// is >= tau.
__global__ void __launch_bounds__(256) k_dfilter(int64_t nq, int P, IndexWs ws)
{
    pdl_wait();
    pdl_release();
    __shared__ float tq[SMALL_NQ];
    __shared__ int Nq[SMALL_NQ];
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    for (int qi = warp; qi < nq; qi += blockDim.x >> 5) {
        const int64_t N = (int64_t)ws.horizon[qi] * LSA_NBKT;
        const float tau = tau_from_hist(ws.ghist + qi * HIST_BINS, N, P);
        if (lane == 0) {
            tq[qi] = tau;
            Nq[qi] = (int)N;
            if (blockIdx.x == 0) ws.tau[qi] = tau;
        }
    }
    __syncthreads();
    const int64_t b4 = ((int64_t)blockIdx.x * blockDim.x + t) * 4;
    for (int qi = 0; qi < nq; ++qi) {
        if (b4 >= Nq[qi]) continue;
        const float4 s = *reinterpret_cast<const float4 *>(ws.scores + qi * ws.score_stride + b4);
        if (fmaxf(fmaxf(s.x, s.y), fmaxf(s.z, s.w)) >= tq[qi]) {
            const int slot = atomicAdd(ws.cnt + qi, 1);
            if (slot < ws.cap) {
                reinterpret_cast<float4 *>(ws.cand4)[qi * ws.cap + slot] = s;
                ws.cand_g[qi * ws.cap + slot] = (int32_t)b4;
            }
        }
    }
}

// ---------------------------------------------------------------------------
// Rank the candidates of one query and expand them into its index list.
//   1. candidates: every listed score >= tau (a Flat query whose entries or
//      candidates overflow, or whose sampled tau keeps fewer than k far keys,
//      is redone exactly here: radix select of the P-th largest score
//      recomputed on the CUDA cores, then every bucket above it and the
//      lowest-id buckets equal to it, P in all);
//   2. each candidate's weight: its members outside near;
//   3. the walk over buckets in (score desc, id asc) order stops at the
//      bucket where the weights reach k: found by histogramming the weights
//      over the candidates' rank keys (1024 or 4096 bins over the remaining
//      key range) and narrowing to the bin where k is reached until it holds
//      at most 32 keys, which one warp ranks -- buckets ranked before the cut
//      are taken whole, their order does not matter;
//   4. the chosen positions are marked in one 512-bit mask per touched block
//      (blocks found through a bitmap over all visible blocks, RX_SLOTS
//      blocks at a time) and emitted block by block in ascending order -- the
//      far keys come out sorted without sorting them; with few queries (1024
//      threads per query) k_rx_emit does this for all touched blocks at once;
//   5. sink, far keys and window are written.
// Every bucket has >= 4 keys and at most sink + window clustered keys are
// near, so the best P buckets already hold k far keys: the cut never falls
// outside the top P.
constexpr int RX_SLOTS = 512;  // touched blocks per emit batch
constexpr int RX_BINS = 4096;  // bins of the cut search at most (aliases the masks)
constexpr int RX_SPLIT = 2048; // touched blocks handed to k_rx_emit at most (16 B of shared memory each)

constexpr int RX_MW = 16;      // words per touched block's mask row; word w sits at w ^ (slot & 15), so
                               // one thread per slot reading word w hits at most 2-way bank conflicts
__device__ __forceinline__ int mword(int slot, int w)
{
    return slot * RX_MW + (w ^ (slot & 15));
}

__host__ __device__ inline size_t rank_expand_smem(int KC, int TW)
{
    return (size_t)KC * 8 + (size_t)RX_SLOTS * RX_MW * 4 + (size_t)TW * 8 + (size_t)RX_SLOTS * 8 + (size_t)KC;
}

template <int NT>
__global__ void __launch_bounds__(NT) k_rank_expand(const int64_t *__restrict__ pos,
                                                      const int32_t *__restrict__ members,
                                                      const int32_t *__restrict__ count,
                                                      const uint16_t *__restrict__ cbf, int32_t *__restrict__ lists,
                                                      int32_t *__restrict__ lens, int Lmax, int k, int sink,
                                                      int window, int P, int KC, int TW, IndexWs ws)
{
    pdl_wait();
    pdl_release();
    extern __shared__ uint64_t rsm[];
    uint64_t *keys = rsm;                                           // [KC]
    uint32_t *masks = reinterpret_cast<uint32_t *>(keys + KC);      // [RX_SLOTS][RX_MW]
    uint32_t *bins = masks;                                         // [RX_BINS] (before the masks are used)
    uint32_t *touched = masks + RX_SLOTS * RX_MW;                   // [TW]
    int32_t *wrank = reinterpret_cast<int32_t *>(touched + TW);     // [TW]
    int32_t *slot_blk = wrank + TW;                                 // [RX_SLOTS]
    int32_t *slot_off = slot_blk + RX_SLOTS;                        // [RX_SLOTS]
    uint8_t *wt = reinterpret_cast<uint8_t *>(slot_off + RX_SLOTS);  // [KC]
    __shared__ int wsum[32];
    __shared__ int hist[256];
    __shared__ int sh[4];
    __shared__ float qf[LSA_D];
    __shared__ int nk_s, fb_s, tot_s, cnt_s, excl_s, ng_s;
    __shared__ unsigned long long lo_s, hi_s, cut_s;

    const int64_t q = blockIdx.x;
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5, nwarps = blockDim.x >> 5;
    const int64_t p = pos[q];
    const int64_t w0 = p - window > 0 ? p - window : 0;
    const int64_t s_end = (int64_t)sink < p + 1 ? (int64_t)sink : p + 1;
    const int64_t N = (int64_t)ws.horizon[q] * LSA_NBKT;
    const float NEG = __int_as_float(0xff800000);
    const int ne = ws.cnt[q];
    if (t == 0) {
        nk_s = 0;
        fb_s = ne > ws.cap;
        tot_s = 0;
        lo_s = ~0ull;
        hi_s = 0ull;
    }
    for (int i = t; i < TW; i += blockDim.x) touched[i] = 0u;
    __syncthreads();

    const float tau = ws.tau[q];
    // Weights: only a block that overlaps the sink or the window can hold near
    // keys; a bucket of any other block weighs its member count.
    auto clear_of_near = [&](int32_t b) {
        const int64_t blo = (int64_t)(b / LSA_NBKT) * LSA_BLK;
        return blo >= s_end && blo + LSA_BLK <= w0;
    };
    auto far_members = [&](int32_t b) {  // members of b outside sink and window
        const int4 *m4 = reinterpret_cast<const int4 *>(members + (int64_t)b * LSA_NSLOT);
        int nn = 0;
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            const int4 w = __ldg(m4 + v);
            const int mm[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                int64_t m = mm[e];  // -1 pads are skipped
                if (m >= 0 && !LSA_IN_BOUNDS(m < N * (LSA_BLK / LSA_NBKT), BOUNDS_BUCKET)) m = -1;
                nn += (m >= 0) && !(m < s_end || (m >= w0 && m <= p));
            }
        }
        return nn;
    };
    int n = 0;
    int my_tot = 0;  // this thread's weights and weighted key range
    unsigned long long my_lo = ~0ull, my_hi = 0ull;
    for (;;) {  // at most twice: a sampled threshold that keeps too little is redone exactly
    // 1. candidates
    if (!fb_s) {
        const float4 *c4 = reinterpret_cast<const float4 *>(ws.cand4) + q * ws.cap;
        const int32_t *cg = ws.cand_g + q * ws.cap;
        // each thread's next entry is loaded before this one's shuffles and
        // shared-memory atomic, so the loads of consecutive rounds overlap
        float4 nx4 = make_float4(NEG, NEG, NEG, NEG);
        int32_t nxg = 0;
        if (t < ne) {
            nx4 = c4[t];
            nxg = cg[t];
        }
        for (int i0 = 0; i0 < ne; i0 += blockDim.x) {  // block-uniform trip count
            float sv[4] = {nx4.x, nx4.y, nx4.z, nx4.w};
            const int32_t g = nxg;
            {
                const int in = i0 + (int)blockDim.x + t;
                nx4 = make_float4(NEG, NEG, NEG, NEG);
                nxg = 0;
                if (in < ne) {
                    nx4 = c4[in];
                    nxg = cg[in];
                }
            }
            int nc = 0;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                if (sv[e] >= tau && sv[e] > NEG && !LSA_IN_BOUNDS(g + e >= 0 && g + e < N, BOUNDS_BUCKET))
                    sv[e] = NEG;  // debug build: a bucket the query cannot see is dropped
                nc += sv[e] >= tau && sv[e] > NEG;
            }
            // one shared-memory atomic per warp
            int incl = nc;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(LSA_FULL, incl, o);
                if (lane >= o) incl += y;
            }
            int base = 0;
            if (lane == 31 && incl > 0) base = atomicAdd(&nk_s, incl);
            int slot = __shfl_sync(LSA_FULL, base, 31) + incl - nc;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                if (sv[e] >= tau && sv[e] > NEG) {
                    if (slot < KC) keys[slot] = rank_key(sv[e], g + e);
                    ++slot;
                }
            }
        }
        __syncthreads();
        if (t == 0 && nk_s > KC) fb_s = 1;
        __syncthreads();
    }
    if (fb_s) {  // block-uniform: exact selection of the top P
        if (t < LSA_D) qf[t] = bf_bits2f(ws.qhat[q * LSA_D + t]);
        if (t == 0) nk_s = 0;
        __syncthreads();
        auto score = [&](int64_t b) { return dot_bf16_row(qf, cbf + b * LSA_D); };
        const float ts = ord2f(block_select_kth_largest(N, P, score, hist, sh));
        for (int64_t b = t; b < N; b += blockDim.x) {
            const float s = score(b);
            if (s > ts) keys[atomicAdd(&nk_s, 1)] = rank_key(s, (int32_t)b);
        }
        __syncthreads();
        // ties at ts in ascending bucket order, up to P candidates in all
        for (int64_t base = 0; base < N; base += blockDim.x) {
            if (nk_s >= P) break;  // block-uniform (read after a barrier)
            const int64_t b = base + t;
            const bool tie = (b < N) && (score(b) == ts);
            const unsigned bal = __ballot_sync(LSA_FULL, tie);
            if (lane == 0) wsum[warp] = __popc(bal);
            __syncthreads();
            int before = nk_s;
            for (int w = 0; w < warp; ++w) before += wsum[w];
            before += __popc(bal & ((1u << lane) - 1u));
            if (tie && before < P) keys[before] = rank_key(ts, (int32_t)b);
            __syncthreads();
            if (t == 0) {
                int tot = 0;
                for (int w = 0; w < nwarps; ++w) tot += wsum[w];
                nk_s = min(P, nk_s + tot);
            }
            __syncthreads();
        }
    }
    n = nk_s;

    // 2. weights of the candidates and the range of their weighted keys
    {
        my_tot = 0;
        my_lo = ~0ull;
        my_hi = 0ull;
        // the next candidate's member count is loaded before this one is used
        int nx_cnt = t < n ? __ldg(count + rank_key_id(keys[t])) : 0;
        for (int i = t; i < n; i += blockDim.x) {
            const int32_t b = rank_key_id(keys[i]);
            const int cnt_b = nx_cnt;
            if (i + (int)blockDim.x < n) nx_cnt = __ldg(count + rank_key_id(keys[i + blockDim.x]));
            const int nn = clear_of_near(b) ? cnt_b : far_members(b);
            wt[i] = (uint8_t)nn;
            my_tot += nn;
            if (nn > 0) {
                my_lo = min(my_lo, (unsigned long long)keys[i]);
                my_hi = max(my_hi, (unsigned long long)keys[i]);
            }
        }
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
        my_tot += __shfl_xor_sync(LSA_FULL, my_tot, o);
        my_lo = min(my_lo, __shfl_xor_sync(LSA_FULL, my_lo, o));
        my_hi = max(my_hi, __shfl_xor_sync(LSA_FULL, my_hi, o));
    }
    if (lane == 0) {
        atomicAdd(&tot_s, my_tot);
        atomicMin(&lo_s, my_lo);
        atomicMax(&hi_s, my_hi);
    }
    __syncthreads();
    // An exact tau sits at or below the P-th best score, and the best P
    // buckets hold k far keys, so fewer than k above it means tau = -inf.
    // A sampled tau can land above the cut: then the query is redone by the
    // exact selection (block-uniform: read after the barrier).
    if (fb_s || tot_s >= k || !(tau > NEG)) break;
    __syncthreads();
    if (t == 0) {
        fb_s = 1;
        tot_s = 0;
        lo_s = ~0ull;
        hi_s = 0ull;
    }
    __syncthreads();
    }
    const int nfar = min(k, tot_s);

    // 3. the cut: smallest key K with (weight of keys <= K) >= nfar, and the
    //    number of K's far keys still needed (take)
    uint64_t cut = 0;
    int take = 0;
    if (nfar > 0) {
        uint64_t lo = lo_s, hi = hi_s;
        int rem = nfar;
        // 1024 bins for up to 2048 candidates (a cut bin then holds a few keys,
        // ranked by one warp below), 4096 for more
        const int nbins = n <= 2048 ? 1024 : RX_BINS, lb = 31 - __clz(nbins);
        for (int round = 0;; ++round) {  // block-uniform
            const uint64_t span = hi - lo;
            const int shift = (span >> lb) == 0 ? 0 : (64 - __clzll((long long)span)) - lb;
            for (int i = t; i < nbins; i += blockDim.x) bins[i] = 0u;
            if (t == 0) cut_s = ~0ull;
            __syncthreads();
            for (int i = t; i < n; i += blockDim.x) {
                const uint64_t key = keys[i];
                if (wt[i] > 0 && key >= lo && key <= hi)
                    atomicAdd(&bins[(key - lo) >> shift], (1u << 18) | (uint32_t)wt[i]);
            }
            __syncthreads();
            block_inclusive_scan(bins, nbins, reinterpret_cast<uint32_t *>(wsum));  // count << 18 | weight
            for (int c = t; c < nbins; c += blockDim.x) {
                const uint32_t inc = bins[c], exc = c > 0 ? bins[c - 1] : 0u;
                if ((int)(exc & 0x3ffffu) < rem && rem <= (int)(inc & 0x3ffffu)) {
                    sh[0] = c;
                    excl_s = (int)(exc & 0x3ffffu);
                    cnt_s = (int)((inc >> 18) - (exc >> 18));
                }
            }
            __syncthreads();
            const int c = sh[0];
            const uint64_t blo = lo + ((uint64_t)c << shift);
            const uint64_t bhi = min(hi, blo + (((uint64_t)1 << shift) - 1));
            rem -= excl_s;
            // one weighted key left in [blo, bhi] (always so once a bin is one
            // key wide, since keys are distinct): it is the cut
            if (cnt_s == 1 || shift == 0 || round == 7) {
                for (int i = t; i < n; i += blockDim.x)
                    if (wt[i] > 0 && keys[i] >= blo && keys[i] <= bhi) atomicMin(&cut_s, (unsigned long long)keys[i]);
                __syncthreads();
                cut = cut_s;
                take = rem;
                break;
            }
            if (cnt_s <= 32) {
                // a few weighted keys left in [blo, bhi]: one warp ranks them
                // by pairwise comparison, each key's weight before it gives the cut
                uint64_t *gk = reinterpret_cast<uint64_t *>(bins);  // [32] (the bins are read by now)
                uint32_t *gw = bins + 64;                            // [32]
                if (t == 0) ng_s = 0;
                __syncthreads();
                for (int i = t; i < n; i += blockDim.x)
                    if (wt[i] > 0 && keys[i] >= blo && keys[i] <= bhi) {
                        const int g = atomicAdd(&ng_s, 1);
                        gk[g] = keys[i];
                        gw[g] = wt[i];
                    }
                __syncthreads();
                if (warp == 0) {
                    const int m = ng_s;
                    const uint64_t mk = lane < m ? gk[lane] : ~0ull;
                    const int mw = lane < m ? (int)gw[lane] : 0;
                    int before = 0;
                    for (int j = 0; j < m; ++j) {
                        const uint64_t kj = __shfl_sync(LSA_FULL, mk, j);
                        const int wj = __shfl_sync(LSA_FULL, mw, j);
                        if (kj < mk) before += wj;
                    }
                    if (lane < m && before < rem && rem <= before + mw) {
                        cut_s = mk;
                        excl_s = before;
                    }
                }
                __syncthreads();
                cut = cut_s;
                take = rem - excl_s;
                break;
            }
            lo = blo;
            hi = bhi;
            __syncthreads();
        }
    }
    const bool any = nfar > 0;

    // 4. touched blocks, then masks and emission RX_SLOTS blocks at a time
    for (int i = t; i < n; i += blockDim.x) {
        if (any && wt[i] > 0 && keys[i] <= cut) {
            const int blk = rank_key_id(keys[i]) / LSA_NBKT;
            atomicOr(&touched[blk >> 5], 1u << (blk & 31));
        }
    }
    __syncthreads();
    for (int i = t; i < TW; i += blockDim.x) wrank[i] = __popc(touched[i]);
    __syncthreads();
    block_inclusive_scan(wrank, TW, wsum);  // wrank[w] = touched blocks in words 0..w
    const int nslots = TW > 0 ? wrank[TW - 1] : 0;
    const int n_sink = (int)min(s_end, w0);
    int32_t *out = lists + q * (int64_t)Lmax;
    int emitted = 0;
    // Wide blocks (few queries): each touched block's chosen buckets (a 64-bit
    // mask) and the list offset of its far keys go to the candidate space
    // (read whole by now), and k_rx_emit emits the blocks in parallel.
    const bool split = NT >= 1024 && any && nslots <= RX_SPLIT && ws.cap >= 3;
    if (split) {
        uint64_t *smask = reinterpret_cast<uint64_t *>(masks);  // [RX_SPLIT]
        int32_t *scnt = reinterpret_cast<int32_t *>(smask + RX_SPLIT);
        int32_t *sblk = scnt + RX_SPLIT;
        for (int i = t; i < nslots; i += blockDim.x) {
            smask[i] = 0ull;
            scnt[i] = 0;
        }
        __syncthreads();
        for (int i = t; i < n; i += blockDim.x) {
            if (wt[i] > 0 && keys[i] <= cut) {
                const int32_t b = rank_key_id(keys[i]);
                const int blk = b / LSA_NBKT;
                const uint32_t word = touched[blk >> 5];
                const int slot = wrank[blk >> 5] - __popc(word) + __popc(word & ((1u << (blk & 31)) - 1u));
                atomicOr(reinterpret_cast<unsigned long long *>(smask + slot), 1ull << (b % LSA_NBKT));
                atomicAdd(scnt + slot, keys[i] == cut ? take : (int)wt[i]);
                sblk[slot] = blk;  // every writer of a slot writes the same block
            }
        }
        __syncthreads();
        block_inclusive_scan(scnt, nslots, wsum);
        int4 *rec = reinterpret_cast<int4 *>(ws.cand4) + q * ws.cap;
        for (int i = t; i < nslots; i += blockDim.x)
            rec[i] = make_int4(sblk[i], i > 0 ? scnt[i - 1] : 0, (int)(uint32_t)smask[i],
                               (int)(uint32_t)(smask[i] >> 32));
        if (t == 0) {
            int32_t *hd = ws.cand_g + q * ws.cap;
            hd[0] = nslots;
            hd[1] = rank_key_id(cut);
            hd[2] = take;
        }
        emitted = scnt[nslots - 1];
    } else if (NT >= 1024 && t == 0 && ws.cap >= 1) {
        ws.cand_g[q * ws.cap] = -1;  // nothing left for k_rx_emit
    }
    // one batch whose far keys fit in the candidate keys' space (free once the
    // marks are set): stage them there and copy the whole list out coalesced
    const bool stage = !split && nslots <= RX_SLOTS && nfar <= 2 * KC;
    int32_t *stg = reinterpret_cast<int32_t *>(keys);
    for (int b0 = 0; b0 < (split ? 0 : nslots); b0 += RX_SLOTS) {
        const int nb = min(RX_SLOTS, nslots - b0);
        for (int i = t; i < nb * RX_MW; i += blockDim.x) masks[i] = 0u;
        __syncthreads();
        // the member row of this thread's next marked candidate is loaded
        // before the current one's atomics
        auto marked = [&](int i) { return i < n && any && wt[i] > 0 && keys[i] <= cut; };
        auto row_of = [&](int i) {
            return reinterpret_cast<const int4 *>(members + (int64_t)rank_key_id(keys[i]) * LSA_NSLOT);
        };
        int nxi = t;
        while (nxi < n && !marked(nxi)) nxi += blockDim.x;
        int4 nxm[4];
        if (nxi < n) {
#pragma unroll
            for (int v = 0; v < 4; ++v) nxm[v] = __ldg(row_of(nxi) + v);
        }
        while (nxi < n) {
            const int i = nxi;
            int4 mrow[4];
#pragma unroll
            for (int v = 0; v < 4; ++v) mrow[v] = nxm[v];
            nxi = i + blockDim.x;
            while (nxi < n && !marked(nxi)) nxi += blockDim.x;
            if (nxi < n) {
#pragma unroll
                for (int v = 0; v < 4; ++v) nxm[v] = __ldg(row_of(nxi) + v);
            }
            const int32_t b = rank_key_id(keys[i]);
            const int blk = b / LSA_NBKT;
            const uint32_t word = touched[blk >> 5];
            const int slot = wrank[blk >> 5] - __popc(word) + __popc(word & ((1u << (blk & 31)) - 1u)) - b0;
            if (slot < 0 || slot >= nb) continue;
            slot_blk[slot] = blk;
            const int64_t blo = (int64_t)blk * LSA_BLK;
            if (keys[i] != cut && blo >= s_end && blo + LSA_BLK <= w0) {
                // a bucket taken whole in a block clear of sink and window: its
                // members are whole pooled items (slots 4v .. 4v + 3 hold the 4
                // consecutive positions of item v), marked 4 bits at a time
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    int m = mrow[v].x;
                    if (m >= 0 && !LSA_IN_BOUNDS(m < N * (LSA_BLK / LSA_NBKT), BOUNDS_BUCKET)) m = -1;
                    if (m >= 0) atomicOr(&masks[mword(slot, (m & 511) >> 5)], 0xFu << (m & 31));
                }
                continue;
            }
            const int limit = (keys[i] == cut) ? take : 16;
            int idx = 0;
#pragma unroll
            for (int v = 0; v < 4; ++v) {
                const int4 w = mrow[v];
                const int mm[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    int64_t m = mm[e];
                    if (m >= 0 && !LSA_IN_BOUNDS(m < N * (LSA_BLK / LSA_NBKT), BOUNDS_BUCKET)) m = -1;
                    if (m >= 0 && !(m < s_end || (m >= w0 && m <= p))) {
                        if (idx < limit) atomicOr(&masks[mword(slot, (int)((m & 511) >> 5))], 1u << (m & 31));
                        ++idx;
                    }
                }
            }
        }
        __syncthreads();
        for (int sl = t; sl < nb; sl += blockDim.x) {
            int c = 0;
#pragma unroll
            for (int w = 0; w < 16; ++w) c += __popc(masks[mword(sl, w)]);
            slot_off[sl] = c;
        }
        __syncthreads();
        block_inclusive_scan(slot_off, nb, wsum);
        // one thread per touched block: its positions in ascending order
        for (int sl = t; sl < nb; sl += blockDim.x) {
            int o = (stage ? 0 : n_sink) + emitted + (sl > 0 ? slot_off[sl - 1] : 0);
            int32_t *dst = stage ? stg : out;
            const int32_t base = slot_blk[sl] * LSA_BLK;
#pragma unroll 4
            for (int w = 0; w < 16; ++w) {
                uint32_t bits = masks[mword(sl, w)];
                while (bits) {
                    const int b = __ffs(bits) - 1;
                    const int32_t pos0 = base + 32 * w + b;
                    if ((b & 3) == 0 && ((bits >> b) & 0xFu) == 0xFu) {  // a whole item: 4 positions at once
                        dst[o] = pos0;
                        dst[o + 1] = pos0 + 1;
                        dst[o + 2] = pos0 + 2;
                        dst[o + 3] = pos0 + 3;
                        o += 4;
                        bits &= ~(0xFu << b);
                    } else {
                        dst[o++] = pos0;
                        bits &= bits - 1;
                    }
                }
            }
        }
        emitted += slot_off[nb - 1];
        __syncthreads();
    }
    // emitted == nfar (the marks add up to the weights before the cut plus
    // take); the list is laid out from what was written either way
    const int nwin = (int)(p - w0 + 1);
    const int len = n_sink + emitted + nwin;
    if (t == 0) (void)LSA_IN_BOUNDS(len <= Lmax, BOUNDS_LIST);
    for (int i = t; i < Lmax; i += blockDim.x) {
        if (i < n_sink) out[i] = i;
        else if (i < n_sink + emitted) {
            if (stage) out[i] = stg[i - n_sink];
        }
        else if (i < len) out[i] = (int32_t)(w0 + (i - n_sink - emitted));
        else out[i] = -1;
    }
    if (t == 0) lens[q] = len;
}

// ---------------------------------------------------------------------------
// The far keys of one query's touched blocks, for the wide (few-query)
// expansion: one warp per touched block.  Its chosen buckets (a 64-bit mask)
// are read two at a time, 16 member slots each; far members (not sink, not
// window) are marked in the warp's 512-bit mask -- of the cut bucket only the
// first `take` in slot order -- and lane w < 16 writes the positions of word
// w in ascending order at the block's offset.
__global__ void __launch_bounds__(256) k_rx_emit(const int64_t *__restrict__ pos,
                                                 const int32_t *__restrict__ members, int32_t *__restrict__ lists,
                                                 int Lmax, int sink, int window, IndexWs ws)
{
    pdl_wait();
    pdl_release();
    __shared__ uint32_t words[8][16];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t q = blockIdx.y;
    const int32_t *hd = ws.cand_g + q * ws.cap;
    const int nslots = hd[0];  // -1: the expansion wrote the list itself
    const int slot = blockIdx.x * 8 + warp;
    if (slot >= nslots) return;
    const int32_t cutb = hd[1];
    const int take = hd[2];
    const int64_t p = pos[q];
    const int64_t w0 = p - window > 0 ? p - window : 0;
    const int64_t s_end = (int64_t)sink < p + 1 ? (int64_t)sink : p + 1;
    const int n_sink = (int)min(s_end, w0);
    const int64_t N = (int64_t)ws.horizon[q] * LSA_NBKT;
    (void)N;  // read by the debug build's bounds checks only
    const int4 r = reinterpret_cast<const int4 *>(ws.cand4)[q * ws.cap + slot];
    const int blk = r.x;
    if (!LSA_IN_BOUNDS(blk >= 0 && (int64_t)blk * LSA_NBKT < N, BOUNDS_BUCKET)) return;
    uint64_t mm = ((uint64_t)(uint32_t)r.w << 32) | (uint32_t)r.z;
    if (lane < 16) words[warp][lane] = 0u;
    __syncwarp();
    const int half = lane >> 4, li = lane & 15;
    while (mm) {  // warp-uniform
        const int j0 = __ffsll((long long)mm) - 1;
        mm &= mm - 1;
        const int j1 = mm ? __ffsll((long long)mm) - 1 : -1;
        if (mm) mm &= mm - 1;
        const int j = half ? j1 : j0;
        const int32_t b = blk * LSA_NBKT + j;
        int m = j >= 0 ? __ldg(members + (int64_t)b * LSA_NSLOT + li) : -1;
        if (m >= 0 && !LSA_IN_BOUNDS(m < N * (LSA_BLK / LSA_NBKT), BOUNDS_BUCKET)) m = -1;
        bool far = m >= 0 && !(m < s_end || (m >= w0 && m <= p));
        const unsigned bal = __ballot_sync(LSA_FULL, far);
        if (far && b == cutb) far = __popc((bal >> (16 * half)) & ((1u << li) - 1u)) < take;
        if (far) atomicOr(&words[warp][(m & (LSA_BLK - 1)) >> 5], 1u << (m & 31));
    }
    __syncwarp();
    uint32_t bits = lane < 16 ? words[warp][lane] : 0u;
    const int c = __popc(bits);
    int incl = c;
#pragma unroll
    for (int o = 1; o < 16; o <<= 1) {
        const int y = __shfl_up_sync(LSA_FULL, incl, o);
        if (lane >= o) incl += y;
    }
    int o = n_sink + r.y + incl - c;
    if (!LSA_IN_BOUNDS(o + c <= Lmax, BOUNDS_LIST)) return;
    int32_t *out = lists + q * (int64_t)Lmax;
    const int32_t base = blk * LSA_BLK + 32 * lane;
    while (bits) {
        const int b = __ffs(bits) - 1;
        out[o++] = base + b;
        bits &= bits - 1;
    }
}

// ---------------------------------------------------------------------------
// Multi-head Flat search (zhichai forum post, "Key points": N-LSA ranks a
// bucket by its best score across the index heads).  Every (query, head) row
// went through the Flat passes above on its own.  A bucket among the top P
// by best score is among the top P of the head that attains that score (a
// bucket ahead of it for that head is ahead of it overall), so that head
// listed it, with that very score.  Keeping every listed bucket once, with
// the largest score any head listed for it, and cutting at the P-th largest
// of those values keeps exactly the top P: a kept value falls short of a
// bucket's best only for buckets outside the top P.  Scores below
// tau* = max over heads of tau_h are dropped first: every head's top P
// scores are at least tau_h, so at least P buckets have a best score
// >= tau_h for every h, and the P-th best is >= tau*.
// The kept buckets go out as one-bucket entries with tau = -inf, for the
// unchanged expansion.  The union is deduplicated in a shared-memory hash
// table with linear probing, sized from the query's entry count (one retry
// at the launch's full size).  A query whose rows overflowed their entry
// slots, whose union does not fit the table, or whose cut keeps more than
// the expansion's slots (ties) is redone exactly: every visible bucket
// scored for every head on the CUDA cores, radix select, ties in ascending
// bucket order.
constexpr int HM_THREADS = 512;
constexpr int HM_MAX_SLOTS = 25600;  // 200 KB of table
constexpr int HM_UNROLL = 4;         // entries a thread loads before using them

// Table slots for a launch: about 2 x heads x P (a head lists ~1.2 P
// buckets at or above tau* on the measured workloads), a multiple of 512, at
// most HM_MAX_SLOTS.
inline int heads_merge_slots(int heads, int P)
{
    const int64_t want = ((int64_t)2 * heads * P + 511) / 512 * 512;
    return (int)(want < HM_MAX_SLOTS ? (want < 512 ? 512 : want) : HM_MAX_SLOTS);
}

// Insert bucket `id` with ordered score v: 1 if the id was new, 0 if it was
// there, -1 if the table is full.
__device__ __forceinline__ int hash_insert(int32_t *hkey, uint32_t *hval, int TS, int32_t id, uint32_t v)
{
    uint32_t s = __umulhi((uint32_t)id * 0x9E3779B1u, (uint32_t)TS);
    for (int n = 0; n < TS; ++n) {
        const int32_t prev = atomicCAS(&hkey[s], -1, id);
        if (prev == -1 || prev == id) {
            atomicMax(&hval[s], v);
            return prev == -1;
        }
        s = (s + 1 == (uint32_t)TS) ? 0u : s + 1;
    }
    return -1;
}

// Histogram bin of a merged value over [lo, lo + 256 / scale]; the same
// rounded operations in the counting and the keeping pass.
__device__ __forceinline__ int merge_bin(float v, float lo, float scale)
{
    return min(255, max(0, __float2int_rz(__fmul_rn(__fsub_rn(v, lo), scale))));
}

__global__ void __launch_bounds__(HM_THREADS, 2) k_heads_merge(int heads, int P, int TSMAX,
                                                              const uint16_t *__restrict__ cbf, IndexWs ws, IndexWs m)
{
    pdl_wait();
    pdl_release();
    extern __shared__ uint32_t hsm[];
    int32_t *hkey = reinterpret_cast<int32_t *>(hsm);  // [TS] bucket id, -1 = empty
    uint32_t *hval = hsm + TSMAX;                      // [TS] f2ord of its best listed score
    __shared__ int hist[256];
    __shared__ int sh[4];
    __shared__ int s_off[LSA_MAXHEADS + 1];  // entry offsets of the heads' rows, flattened
    __shared__ float s_tstar;
    __shared__ int s_over, s_full, s_uniq, s_out, s_exact, s_bstar, s_keep;
    __shared__ uint32_t s_vmin, s_vmax;
    __shared__ uint2 wq[HM_THREADS / 32][64];  // per warp: kept (bucket, value) pairs waiting to be inserted
    const int64_t q = blockIdx.x;
    const int64_t r0 = q * heads;
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const float NEG = __int_as_float(0xff800000);
    const int KC = m.cap;
    float4 *o4 = reinterpret_cast<float4 *>(m.cand4) + q * KC;
    int32_t *og = m.cand_g + q * KC;
    if (t < 32) {  // warp 0, lane h: head h's entry count and threshold
        const int ne = lane < heads ? ws.cnt[r0 + lane] : 0;
        float ts = lane < heads ? ws.tau[r0 + lane] : NEG;
        const unsigned over = __ballot_sync(LSA_FULL, ne > ws.cap);  // a row lost entries: exact path
        int incl = min(ne, ws.cap);
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(LSA_FULL, incl, o);
            if (lane >= o) incl += y;
            ts = fmaxf(ts, __shfl_xor_sync(LSA_FULL, ts, o));
        }
        if (lane < heads) s_off[lane + 1] = incl;
        if (lane == 0) {
            s_off[0] = 0;
            s_tstar = ts;
            s_over = over != 0u;
            s_out = 0;
        }
    }
    __syncthreads();
    const int E = s_off[heads];
    const float tstar = s_tstar;
    // a query's table: 1.5 slots per entry for several heads (their union
    // has about 0.7 buckets per entry), 2 for one row (about 1.4 kept
    // scores per entry when a shard holds few blocks); one that fills is
    // redone once with all of the launch's slots, and a union that fills
    // those takes the exact path.  One row (a shard's own candidates) holds
    // no bucket twice: its kept scores are appended as a list, not hashed.
    const bool direct = heads == 1;
    int TS = min(TSMAX, max(64, direct ? 2 * E : E + E / 2));
    for (;;) {  // block-uniform, at most two rounds
        if (!direct)
            for (int i = t; i < TS; i += HM_THREADS) {
                hkey[i] = -1;
                hval[i] = 0u;
            }
        if (t == 0) {
            s_full = 0;
            s_uniq = 0;
            s_vmin = ~0u;
            s_vmax = 0u;
        }
        __syncthreads();

        // 1. union of the scores at or above tau*, best score per bucket
        int fresh = 0, full = 0, qn = 0;
        uint32_t vmin = ~0u, vmax = 0u;
        if (!s_over) {
            for (int i0 = 0; i0 < E; i0 += HM_THREADS * HM_UNROLL) {
                float4 sv[HM_UNROLL];
                int32_t g[HM_UNROLL];
#pragma unroll
                for (int u = 0; u < HM_UNROLL; ++u) {
                    const int i = i0 + u * HM_THREADS + t;
                    sv[u] = make_float4(NEG, NEG, NEG, NEG);
                    g[u] = 0;
                    if (i < E) {
                        int h = 0;
                        while (i >= s_off[h + 1]) ++h;
                        const int64_t j = (r0 + h) * ws.cap + (i - s_off[h]);
                        sv[u] = reinterpret_cast<const float4 *>(ws.cand4)[j];
                        g[u] = ws.cand_g[j];
                    }
                }
                // kept scores are queued per warp and inserted 32 at a time, one
                // per lane (about one score in four is kept)
#pragma unroll
                for (int u = 0; u < HM_UNROLL; ++u) {
                    const float x[4] = {sv[u].x, sv[u].y, sv[u].z, sv[u].w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const bool k = x[e] >= tstar && x[e] > NEG;
                        const unsigned bal = __ballot_sync(LSA_FULL, k);
                        if (k) {
                            const uint32_t v = f2ord(x[e]);
                            wq[warp][qn + __popc(bal & ((1u << lane) - 1u))] = make_uint2((uint32_t)(g[u] + e), v);
                            vmin = min(vmin, v);
                            vmax = max(vmax, v);
                        }
                        qn += __popc(bal);
                        if (qn >= 32) {  // warp-uniform
                            __syncwarp();
                            const uint2 w = wq[warp][lane];
                            if (direct) {
                                int base = 0;
                                if (lane == 0) base = atomicAdd(&s_uniq, 32);
                                base = __shfl_sync(LSA_FULL, base, 0);
                                if (base + lane < TS) {
                                    hkey[base + lane] = (int32_t)w.x;
                                    hval[base + lane] = w.y;
                                } else {
                                    full = 1;
                                }
                            } else {
                                const int r = hash_insert(hkey, hval, TS, (int32_t)w.x, w.y);
                                fresh += r > 0;
                                full |= r < 0;
                            }
                            __syncwarp();
                            if (lane < qn - 32) wq[warp][lane] = wq[warp][32 + lane];
                            __syncwarp();
                            qn -= 32;
                        }
                    }
                }
            }
            __syncwarp();
            if (direct) {
                int base = 0;
                if (lane == 0 && qn) base = atomicAdd(&s_uniq, qn);
                base = __shfl_sync(LSA_FULL, base, 0);
                if (lane < qn) {
                    if (base + lane < TS) {
                        hkey[base + lane] = (int32_t)wq[warp][lane].x;
                        hval[base + lane] = wq[warp][lane].y;
                    } else {
                        full = 1;
                    }
                }
            } else if (lane < qn) {
                const uint2 w = wq[warp][lane];
                const int r = hash_insert(hkey, hval, TS, (int32_t)w.x, w.y);
                fresh += r > 0;
                full |= r < 0;
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            fresh += __shfl_xor_sync(LSA_FULL, fresh, o);
            full |= __shfl_xor_sync(LSA_FULL, full, o);
            vmin = min(vmin, __shfl_xor_sync(LSA_FULL, vmin, o));
            vmax = max(vmax, __shfl_xor_sync(LSA_FULL, vmax, o));
        }
        if (lane == 0) {
            if (fresh) atomicAdd(&s_uniq, fresh);
            if (full) s_full = 1;
            atomicMin(&s_vmin, vmin);
            atomicMax(&s_vmax, vmax);
        }
        __syncthreads();
        if (!s_full || TS == TSMAX) break;
        TS = TSMAX;
        __syncthreads();  // s_full read by every thread before the next round resets it
    }
    for (int i = t; i < 256; i += HM_THREADS) hist[i] = 0;
    __syncthreads();
    if (t == 0) s_exact = s_over | s_full;
    const int U = s_uniq;
    __syncthreads();

    // 2. the cut: all of a small union; else every bucket from the histogram
    //    bin holding the P-th best value up, which holds the top P; a radix
    //    select to the P-th value itself when that is more than the slots
    if (!s_exact) {
        const float lo = ord2f(s_vmin), hi = ord2f(s_vmax);
        const float scale = hi > lo ? 256.0f / (hi - lo) : 0.0f;
        const int scan = direct ? min(U, TS) : TS;  // slots that may hold a bucket
        int bstar = 0;
        uint32_t cut = 0u;
        if (U > KC) {
            const int n_round = (scan + HM_THREADS - 1) / HM_THREADS * HM_THREADS;
            for (int i = t; i < n_round; i += HM_THREADS) {
                const int bin = (i < scan && hkey[i] >= 0) ? merge_bin(ord2f(hval[i]), lo, scale) : -1;
                // lanes with the same bin add once (values cluster in few bins)
                const unsigned peers = __match_any_sync(LSA_FULL, bin);
                if (bin >= 0 && lane == __ffs(peers) - 1) atomicAdd(&hist[bin], __popc(peers));
            }
            __syncthreads();
            if (t < 32) {  // warp 0: lane l owns bins 255-8l .. 248-8l
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
                if (excl < P && P <= incl) {
                    int acc = excl;
                    for (int e = 0; e < 8; ++e) {
                        const int d = 255 - 8 * lane - e;
                        acc += hist[d];
                        if (acc >= P) {
                            s_bstar = d;
                            s_keep = acc;
                            break;
                        }
                    }
                }
            }
            __syncthreads();
            bstar = s_bstar;
            if (s_keep > KC) {  // block-uniform: too many at the boundary bin
                auto get = [&](int64_t i) { return hkey[i] >= 0 ? ord2f(hval[i]) : NEG; };
                cut = block_select_kth_largest(scan, P, get, hist, sh);
                bstar = -1;
            }
        }
        for (int i = t; i < scan; i += HM_THREADS) {
            const int32_t id = hkey[i];
            const uint32_t v = hval[i];
            const bool take = id >= 0 && (U <= KC || (bstar >= 0 ? merge_bin(ord2f(v), lo, scale) >= bstar : v >= cut));
            if (take) {
                const int j = atomicAdd(&s_out, 1);
                if (j < KC) {
                    o4[j] = make_float4(ord2f(v), NEG, NEG, NEG);
                    og[j] = id;
                }
            }
        }
        __syncthreads();
        if (t == 0 && s_out > KC) s_exact = 1;
    }
    __syncthreads();
    if (t == 0) {
        m.cnt[q] = s_exact ? -1 : s_out;  // -1: k_heads_exact redoes the query
        m.tau[q] = NEG;
        m.horizon[q] = ws.horizon[r0];
    }
}

// One marked query of k_heads_exact, all threads of the block.
__device__ void heads_exact_query(int64_t q, int heads, int P, const uint16_t *__restrict__ cbf, const IndexWs &ws,
                                  const IndexWs &m, float *qf, int *hist, int *sh, int *wsum, int &s_out)
{
    const int64_t r0 = q * heads;
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const float NEG = __int_as_float(0xff800000);

    const int64_t N = (int64_t)ws.horizon[r0] * LSA_NBKT;
    float4 *o4 = reinterpret_cast<float4 *>(m.cand4) + q * m.cap;
    int32_t *og = m.cand_g + q * m.cap;
    for (int i = t; i < heads * LSA_D; i += HM_THREADS) qf[i] = bf_bits2f(ws.qhat[r0 * LSA_D + i]);
    if (t == 0) s_out = 0;
    __syncthreads();
    auto best = [&](int64_t b) {
        const uint16_t *c = cbf + b * LSA_D;
        float s = dot_bf16_row(qf, c);
        for (int h = 1; h < heads; ++h) s = fmaxf(s, dot_bf16_row(qf + h * LSA_D, c));
        return s;
    };
    if (N <= P) {
        for (int64_t b = t; b < N; b += HM_THREADS) {
            o4[b] = make_float4(best(b), NEG, NEG, NEG);
            og[b] = (int32_t)b;
        }
        if (t == 0) s_out = (int)N;
    } else {
        const float ts = ord2f(block_select_kth_largest(N, P, best, hist, sh));
        for (int64_t b = t; b < N; b += HM_THREADS) {
            const float s = best(b);
            if (s > ts) {
                const int j = atomicAdd(&s_out, 1);  // fewer than P buckets score above ts
                o4[j] = make_float4(s, NEG, NEG, NEG);
                og[j] = (int32_t)b;
            }
        }
        __syncthreads();
        // ties at ts in ascending bucket order, up to P in all
        for (int64_t base = 0; base < N; base += HM_THREADS) {
            if (s_out >= P) break;  // block-uniform (read after a barrier)
            const int64_t b = base + t;
            const bool tie = (b < N) && (best(b) == ts);
            const unsigned bal = __ballot_sync(LSA_FULL, tie);
            if (lane == 0) wsum[warp] = __popc(bal);
            __syncthreads();
            int before = s_out;
            for (int w = 0; w < warp; ++w) before += wsum[w];
            before += __popc(bal & ((1u << lane) - 1u));
            if (tie && before < P) {
                o4[before] = make_float4(ts, NEG, NEG, NEG);
                og[before] = (int32_t)b;
            }
            __syncthreads();
            if (t == 0) {
                int tot = 0;
                for (int w = 0; w < HM_THREADS / 32; ++w) tot += wsum[w];
                s_out = min(P, s_out + tot);
            }
            __syncthreads();
        }
    }
    __syncthreads();
    if (t == 0) m.cnt[q] = s_out;
    __syncthreads();
}


// The exact path of the merge, for the queries k_heads_merge marked (cnt -1):
// the top P buckets by best head score, each score recomputed on the CUDA
// cores, ties at the P-th score in ascending bucket order.  Each CTA scans
// the flags of its share of the queries and redoes the marked ones.
__global__ void __launch_bounds__(HM_THREADS) k_heads_exact(int64_t nq, int heads, int P,
                                                           const uint16_t *__restrict__ cbf, IndexWs ws, IndexWs m)
{
    pdl_wait();
    pdl_release();
    __shared__ float qf[LSA_MAXHEADS * LSA_D];
    __shared__ int hist[256];
    __shared__ int sh[4];
    __shared__ int wsum[HM_THREADS / 32];
    __shared__ int s_out, s_n;
    __shared__ int ql[HM_THREADS];  // marked queries of the current range, base-relative
    const int t = threadIdx.x, lane = t & 31;
    const int64_t per = (nq + gridDim.x - 1) / gridDim.x;
    const int64_t qa = (int64_t)blockIdx.x * per, qb = min(nq, qa + per);
    for (int64_t base = qa; base < qb; base += HM_THREADS) {
        if (t == 0) s_n = 0;
        __syncthreads();
        const bool mark = base + t < qb && m.cnt[base + t] < 0;
        const unsigned bal = __ballot_sync(LSA_FULL, mark);
        int at = 0;
        if (lane == 0 && bal) at = atomicAdd(&s_n, __popc(bal));
        at = __shfl_sync(LSA_FULL, at, 0);
        if (mark) ql[at + __popc(bal & ((1u << lane) - 1u))] = t;
        __syncthreads();
        const int n = s_n;
        for (int k = 0; k < n; ++k)  // block-uniform
            heads_exact_query(base + ql[k], heads, P, cbf, ws, m, qf, hist, sh, wsum, s_out);
        __syncthreads();
    }
}
// Expansion of an already merged candidate set (one-bucket entries, at most
// m.cap per query, tau = -inf), e.g. the top P of a context-parallel merge.
static cudaError_t launch_rank_expand(const IndexArgs &a, const IndexWs &ex, int KC, int TW, bool small,
                                      cudaStream_t st);

cudaError_t launch_expand_merged(const IndexArgs &a, const IndexWs &m, cudaStream_t st)
{
    if (a.nq <= 0) return cudaSuccess;
    const int TW = (int)((a.n_blocks + 31) / 32) + 1;
    return launch_rank_expand(a, m, m.cap, TW, a.nq <= SMALL_NQ, st);
}

size_t rank_expand_smem_bytes(int cap, int64_t n_blocks)
{
    return rank_expand_smem(cap, (int)((n_blocks + 31) / 32) + 1);
}

// ---------------------------------------------------------------------------
// Expansion of every query's candidates into its list.  Many queries: one
// 256-thread CTA per query does everything.  Few: one 1024-thread CTA per
// query ranks and cuts, and k_rx_emit writes the far keys block by block.
static cudaError_t launch_rank_expand(const IndexArgs &a, const IndexWs &ex, int KC, int TW, bool small,
                                      cudaStream_t st)
{
    const size_t smr = rank_expand_smem(KC, TW);
    int kt = kt_begin("k_rank_expand", st);
    if (small) {
        cudaFuncSetAttribute(k_rank_expand<1024>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smr);
        cudaError_t e = launch_k(true, k_rank_expand<1024>, dim3((unsigned)a.nq), dim3(1024), smr, st, a.pos,
                                 a.members, a.count, a.centroid_bf16, a.lists, a.lens, a.Lmax, a.k, a.sink, a.window,
                                 a.P, KC, TW, ex);
        kt_end(kt, st);
        if (e != cudaSuccess) return e;
        count_launches(1);
        if (ex.cap >= 3) {
            kt = kt_begin("k_rx_emit", st);
            const unsigned gx = (unsigned)((min(KC, RX_SPLIT) + 7) / 8);
            e = launch_k(true, k_rx_emit, dim3(gx, (unsigned)a.nq), dim3(256), 0, st, a.pos, a.members, a.lists,
                         a.Lmax, a.sink, a.window, ex);
            kt_end(kt, st);
            if (e != cudaSuccess) return e;
            count_launches(1);
        }
    } else {
        cudaFuncSetAttribute(k_rank_expand<256>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smr);
        k_rank_expand<256><<<(unsigned)a.nq, 256, smr, st>>>(a.pos, a.members, a.count, a.centroid_bf16, a.lists,
                                                             a.lens, a.Lmax, a.k, a.sink, a.window, a.P, KC, TW, ex);
        kt_end(kt, st);
        count_launches(1);
    }
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
cudaError_t launch_index(const IndexArgs &a, const IndexWs &ws, const IndexWs *merged, const TreeView *tree,
                         cudaStream_t st, int n_sm)
{
    if (a.nq <= 0) return cudaSuccess;
    cudaError_t e;
    const int heads = a.heads > 1 ? a.heads : 1;
    const int64_t rows = a.nq * heads;  // one scoring row per (query, index head)
    {
        int64_t blocks = (rows + 7) / 8;
        if (blocks > (int64_t)n_sm * 32) blocks = (int64_t)n_sm * 32;
        const int kt = kt_begin("k_qnorm", st);
        e = launch_k(rows <= SMALL_NQ, k_qnorm, dim3((unsigned)blocks), dim3(256), 0, st, a.qidx, a.pos, rows, heads,
                     a.pos_shift, a.n_blocks, ws);
        kt_end(kt, st);
        if (e != cudaSuccess) return e;
        count_launches(1);
    }
    const int64_t nb_total = a.n_blocks * LSA_NBKT;
    const bool small = a.nq <= SMALL_NQ;
    if (a.mode == 0 && nb_total > 0) {
        if (rows <= SMALL_NQ) {  // stream every centroid once for the whole batch, keep the scores
            const int dsm = DS_WARPS * 2 * 32 * DS_ROW + (int)rows * (HIST_BINS + LSA_D) * 4;
            auto ds = rows <= 1 ? k_dscore<1> : rows <= 2 ? k_dscore<2> : rows <= 4 ? k_dscore<4>
                    : rows <= 8 ? k_dscore<8> : k_dscore<SMALL_NQ>;
            cudaFuncSetAttribute(ds, cudaFuncAttributeMaxDynamicSharedMemorySize, dsm);
            int kt = kt_begin("k_dscore", st);
            e = launch_k(true, ds, dim3((unsigned)((nb_total + DS_SPAN - 1) / DS_SPAN)), dim3(DS_WARPS * 32),
                         (size_t)dsm, st, rows, nb_total, a.centroid_bf16, a.P, ws);
            kt_end(kt, st);
            if (e != cudaSuccess) return e;
            count_launches(1);
            kt = kt_begin("k_dfilter", st);
            e = launch_k(true, k_dfilter, dim3((unsigned)((nb_total / 4 + 255) / 256)), dim3(256), 0, st, rows, a.P,
                         ws);
            kt_end(kt, st);
            if (e != cudaSuccess) return e;
            count_launches(1);
        } else {  // two passes on the tensor cores: threshold, then filter
            ScoreTcArgs sa;
            sa.nq = rows;
            sa.nb_total = nb_total;
            sa.P = a.P;
            sa.mode = 0;
            sa.chunk_tiles = 0;
            sa.wait_limit = a.wait_limit;
            sa.extra_tx = a.extra_tx;
            // sampled threshold: single-head Flat search that expands its own
            // candidates (the multi-head and shard merges rely on an exact tau)
            sa.sample = (heads == 1 && !a.no_expand) ? a.sample : 0;
            sa.sample_margin = a.sample_margin;
            sa.sample_min_n = a.sample_min_n;
            int whole = 0;
            if ((e = launch_score_tc(sa, ws, a.centroid_bf16, st, n_sm, &whole)) != cudaSuccess) return e;
            if (!whole) {  // thresholds from the merged histograms
                const int kt = kt_begin("k_tau", st);
                k_tau<<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(rows, a.P, ws);
                kt_end(kt, st);
                count_launches(1);
                if ((e = cudaGetLastError()) != cudaSuccess) return e;
            }
            sa.mode = 1;
            sa.extra_tx = 0;
            if ((e = launch_score_tc(sa, ws, a.centroid_bf16, st, n_sm, nullptr)) != cudaSuccess) return e;
        }
    } else if (tree && tree->n_levels > 0) {
        int64_t B1 = ((int64_t)a.P + 1) / 2;
        if (B1 < a.beam) B1 = a.beam;
        // candidates per level: the children of at most B1 kept nodes plus one run
        const int CM = (int)(2 * B1 + LSA_RUN + 2);
        const int KM = (int)B1;
        const int kt = kt_begin("k_tree_beam", st);
        if (small) {  // one query per CTA of 16 warps
            auto kern = k_tree_beam<16, 1>;
            const size_t tb = tree_beam_team_bytes(CM, KM, 16);
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tb);
            e = launch_k(true, kern, dim3((unsigned)a.nq), dim3(512), tb, st, a.nq, *tree, a.beam, a.P, CM, KM, ws);
        } else {  // BEAM_TEAM warps per query, teams of a CTA independent
            auto kern = k_tree_beam<BEAM_TEAM, BEAM_MINB>;
            const size_t tb = tree_beam_team_bytes(CM, KM, BEAM_TEAM);
            const int per_cta = 8 / BEAM_TEAM;
            const int qpb = (int)max((size_t)1, min((size_t)per_cta, (SM_SMEM / BEAM_MINB - 1024) / tb));
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)(qpb * tb));
            e = launch_k(false, kern, dim3((unsigned)((a.nq + qpb - 1) / qpb)), dim3(32 * BEAM_TEAM * qpb), qpb * tb,
                         st, a.nq, *tree, a.beam, a.P, CM, KM, ws);
        }
        kt_end(kt, st);
        if (e != cudaSuccess) return e;
        count_launches(1);
    }
    if (merged) {  // several index heads: one candidate set per query
        const int TS = heads_merge_slots(heads, a.P);
        const size_t smh = (size_t)TS * 8;
        cudaFuncSetAttribute(k_heads_merge, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smh);
        int kt = kt_begin("k_heads_merge", st);
        e = launch_k(small, k_heads_merge, dim3((unsigned)a.nq), dim3(HM_THREADS), smh, st, heads, a.P, TS,
                     a.centroid_bf16, ws, *merged);
        kt_end(kt, st);
        if (e != cudaSuccess) return e;
        const unsigned xg = (unsigned)min((int64_t)n_sm, a.nq);
        kt = kt_begin("k_heads_exact", st);
        e = launch_k(small, k_heads_exact, dim3(xg), dim3(HM_THREADS), 0, st, a.nq, heads, a.P, a.centroid_bf16, ws,
                     *merged);
        kt_end(kt, st);
        if (e != cudaSuccess) return e;
        count_launches(2);
        if (a.no_expand) return cudaGetLastError();  // a shard's local candidate set stops here
    }
    const IndexWs &ex = merged ? *merged : ws;
    const int TW = (int)((a.n_blocks + 31) / 32) + 1;
    // candidates held in shared memory: the filter keeps about 1.2-1.45 P per
    // query on the measured workloads; a query with more takes the exact path
    // (a merged set never has more than its slots)
    const int KC = merged ? merged->cap : (int)min((int64_t)ws.cap, pow2_ceil64(((int64_t)a.P * 3 + 1) / 2));
    return launch_rank_expand(a, ex, KC, TW, small, st);
}

// this file's bounds-check word (debug build; always 0 in the release build)
LSA_BOUNDS_READER(read_bounds_error_index)

}  // namespace lsa
