"""Pins for the CPU oracle: each test ties one oracle function to something
other than itself -- a closed form, a library routine, brute force on tiny
inputs, a special case whose answer the LSA pages fix, or a count the pages
print.  CPU only."""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle as O
from hierarchical_key_clustering_b200 import inputs as I

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- scalars

def test_bf16_round_matches_torch():
    """bf16 round-to-nearest-even against torch's conversion (library routine)."""
    rng = np.random.default_rng(1)
    x = np.concatenate([rng.standard_normal(4000).astype(np.float32),
                        np.array([0.0, -0.0, 1.0, -1.0, 1.00390625, 1.01171875, 3.0e-39, 65504.0,
                                  1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -9], np.float32)])
    ours = O.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_sumsq_order_close_to_fp64():
    rng = np.random.default_rng(2)
    for _ in range(200):
        x = rng.standard_normal(64).astype(np.float32)
        got = O.sumsq(x)
        ref = float(np.sum(x.astype(np.float64) ** 2))
        assert abs(got - ref) <= 1e-6 * ref


def test_normalize_unit_length_and_zero():
    rng = np.random.default_rng(3)
    for _ in range(100):
        x = (rng.standard_normal(64) * rng.uniform(0.01, 100)).astype(np.float32)
        n = O.normalize(x).astype(np.float64)
        assert abs(np.linalg.norm(n) - 1.0) < 1e-6
        assert np.allclose(n, x / np.linalg.norm(x.astype(np.float64)), atol=1e-7)
    assert np.all(O.normalize(np.zeros(64, np.float32)) == 0)


# ---------------------------------------------------------------- a1 pool

def test_pool_closed_form():
    """pooled key = sum of 4 length-normalised keys (fp64 closed form)."""
    keys = I.index_keys(0, 4096, 32)
    y = O.pool_norm(keys)
    k64 = keys.astype(np.float64)
    ref = (k64 / np.linalg.norm(k64, axis=1, keepdims=True)).reshape(-1, 4, 64).sum(axis=1)
    assert y.shape == (1024, 64)
    assert np.max(np.abs(y - ref)) < 2e-6
    assert np.all(np.linalg.norm(y.astype(np.float64), axis=1) <= 4.0 + 1e-5)


def test_pool_identical_keys_norm_four():
    rng = np.random.default_rng(4)
    v = rng.standard_normal(64).astype(np.float32)
    keys = np.tile(v, (8, 1))
    y = O.pool_norm(keys)
    assert np.allclose(np.linalg.norm(y.astype(np.float64), axis=1), 4.0, atol=1e-5)


# ---------------------------------------------------------------- a2 Ward

def _replay_sets(m, ti, tj):
    sets = {i: {i} for i in range(m)}
    history = [{k: set(v) for k, v in sets.items()}]
    for i, j in zip(ti, tj):
        sets[i] |= sets.pop(j)
        history.append({k: set(v) for k, v in sets.items()})
    return history


def _delta_sse(items64, A, B):
    a = items64[sorted(A)]
    b = items64[sorted(B)]
    ma, mb = a.mean(axis=0), b.mean(axis=0)
    return len(A) * len(B) / (len(A) + len(B)) * float(np.sum((ma - mb) ** 2))


@pytest.mark.parametrize("seed,m,cap,target", [(0, 16, 4, 8), (1, 24, 4, 12), (2, 20, 3, 9), (3, 32, 4, 16)])
def test_ward_brute_force_each_merge(seed, m, cap, target):
    """At every merge, the LW-tracked cost equals the fp64 increase of the sum
    of squared errors recomputed from the explicit member sets, and the pair
    chosen is the fp64 argmin over eligible pairs."""
    rng = np.random.default_rng(seed)
    items = rng.standard_normal((m, 64)).astype(np.float32)
    root, (ti, tj, td) = O.ward(items, cap=cap, n_target=target, trace=True)
    assert len(ti) == m - target
    hist = _replay_sets(m, ti, tj)
    it64 = items.astype(np.float64)
    for step, (i, j, d) in enumerate(zip(ti, tj, td)):
        sets = hist[step]
        ref = _delta_sse(it64, sets[i], sets[j])
        assert abs(d - ref) <= 1e-5 * max(ref, 1e-12)
        best = min(_delta_sse(it64, sets[a], sets[b])
                   for a in sets for b in sets if a < b and len(sets[a]) + len(sets[b]) <= cap)
        assert ref <= best * (1 + 1e-6) + 1e-12
    final = hist[-1]
    for c, members in final.items():
        for t in members:
            assert root[t] == c


def test_ward_textbook_agglomeration_matches_scipy():
    """With no size cap and one final cluster, Ward's method is the textbook
    agglomeration: same merge sets and heights as scipy's ward linkage
    (height = sqrt(2 * increase of SSE))."""
    from scipy.cluster.hierarchy import linkage
    rng = np.random.default_rng(7)
    m = 24
    items = rng.standard_normal((m, 64)).astype(np.float32)
    root, (ti, tj, td) = O.ward(items, cap=m, n_target=1, trace=True)
    Z = linkage(items.astype(np.float64), method="ward")
    # scipy cluster ids: < m are items, m + s is the cluster formed at step s
    sp_sets = {i: frozenset([i]) for i in range(m)}
    sp_merges = []
    for s, (a, b, h, _) in enumerate(Z):
        new = sp_sets[int(a)] | sp_sets[int(b)]
        sp_sets[m + s] = new
        sp_merges.append((new, h))
    hist = _replay_sets(m, ti, tj)
    ours = []
    for step, (i, j, d) in enumerate(zip(ti, tj, td)):
        ours.append((frozenset(hist[step][i] | hist[step][j]), math.sqrt(2.0 * d)))
    assert [s for s, _ in ours] == [s for s, _ in sp_merges]
    for (_, h1), (_, h2) in zip(ours, sp_merges):
        assert abs(h1 - h2) <= 1e-4 * h2


def _check_cache_invariants(cache):
    nblk = cache.nblk
    for b in range(nblk):
        ib = cache.item_bucket[b]
        assert ib.min() == 0 and ib.max() == 63
        sizes = np.bincount(ib, minlength=64)
        assert np.all((sizes >= 1) & (sizes <= 4))
        # buckets ordered by their lowest item
        firsts = [int(np.nonzero(ib == r)[0][0]) for r in range(64)]
        assert firsts == sorted(firsts)
        positions = []
        for r in range(64):
            g = b * 64 + r
            items = np.nonzero(ib == r)[0]
            want = (b * 512 + 4 * items[:, None] + np.arange(4)[None, :]).ravel()
            cnt = cache.count[g]
            assert cnt == 4 * len(items)
            assert np.array_equal(cache.members[g, :cnt], want)
            assert np.all(cache.members[g, cnt:] == -1)
            positions.extend(want.tolist())
        assert sorted(positions) == list(range(b * 512, (b + 1) * 512))


def test_cache_partition_and_sizes():
    """Buckets partition each block's 512 positions; 4..16 keys each; exactly 64."""
    keys = I.index_keys(0, 4096, 32)
    cache = O.build_cache(keys)
    _check_cache_invariants(cache)
    assert 4 <= cache.count.min() and cache.count.max() <= 16
    assert cache.count.mean() == 8.0


def test_cache_centroids_are_normalised_member_sums():
    keys = I.index_keys(5, 2048, 32)
    cache = O.build_cache(keys)
    y = cache.pooled.astype(np.float64)
    for g in range(cache.members.shape[0]):
        items = cache.members[g, :cache.count[g]:4] // 4
        s = y[items].sum(axis=0)
        ref = s / np.linalg.norm(s)
        assert np.max(np.abs(cache.centroid[g] - ref)) < 1e-6
    ref_bf = torch.from_numpy(cache.centroid).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(cache.centroid_bf16, ref_bf)


def test_ward_identical_items_tie_break():
    """128 identical items: every cost is 0, so the lowest-(i, j) rule alone
    decides: items 0-3, 4-7, ..., 80-83 form 21 four-item buckets, (84, 85) a
    two-item bucket, and items 86..127 stay single (64 buckets in all)."""
    items = np.tile(np.linspace(-1, 1, 64, dtype=np.float32), (128, 1))
    root = O.ward(items)
    groups = {}
    for t, r in enumerate(root):
        groups.setdefault(int(r), []).append(t)
    got = sorted(groups.values())
    want = [list(range(4 * g, 4 * g + 4)) for g in range(21)] + [[84, 85]] + [[t] for t in range(86, 128)]
    assert got == sorted(want)
    assert len(groups) == 64


def test_ward_identical_pairs_become_buckets():
    """64 distinct, well-separated values each held by two items: the 64
    zero-cost merges pair exactly the equal items."""
    rng = np.random.default_rng(11)
    vals = rng.standard_normal((64, 64)).astype(np.float32) * 10
    perm = rng.permutation(128)
    items = np.empty((128, 64), np.float32)
    items[perm] = np.repeat(vals, 2, axis=0)
    root = O.ward(items)
    pair_of = np.repeat(np.arange(64), 2)[np.argsort(perm)]
    for a in range(128):
        for b in range(a + 1, 128):
            assert (root[a] == root[b]) == (pair_of[a] == pair_of[b])


def test_ward_separated_groups_never_mix():
    rng = np.random.default_rng(12)
    e = np.zeros(64, np.float32)
    e[0] = 50.0
    side = rng.integers(0, 2, 128)
    items = (rng.standard_normal((128, 64)) * 0.3).astype(np.float32) + np.where(side[:, None] == 1, e, -e)
    root = O.ward(items)
    for t in range(128):
        assert side[t] == side[root[t]]


# ---------------------------------------------------------------- a3 tree

def test_tree_levels_and_weights():
    keys = I.index_keys(0, 4096, 32)
    cache = O.build_cache(keys)
    tree = O.build_tree(cache)
    nb = cache.nblk * 64
    assert tree.n_levels == math.ceil(math.log2(nb)) + 1
    assert tree.level_size[-1] == 1
    off = tree.level_offset
    root = off[-1] - 1
    assert tree.weight[root] == cache.nblk * 128
    for l in range(1, tree.n_levels):
        for u in range(tree.level_size[l]):
            v = off[l] + u
            kids = [c for c in tree.child[v] if c >= 0]
            assert len(kids) >= 1
            assert tree.weight[v] == sum(tree.weight[off[l - 1] + c] for c in kids)
            assert tree.max_block[v] == max(tree.max_block[off[l - 1] + c] for c in kids)
            assert tree.min_block[v] == min(tree.min_block[off[l - 1] + c] for c in kids)
            for c in kids:
                assert tree.parent[off[l - 1] + c] == u
        # every node below the top has exactly one parent that lists it
        if l < tree.n_levels:
            n_children = int((tree.child[off[l]:off[l] + tree.level_size[l]] >= 0).sum())
            assert n_children == tree.level_size[l - 1]


def test_tree_centroids_from_leaves():
    """A node's centroid is the normalised sum of its leaves' pooled keys."""
    keys = I.index_keys(1, 2048, 32)
    cache = O.build_cache(keys)
    tree = O.build_tree(cache)
    off = tree.level_offset
    y = cache.pooled.astype(np.float64)

    def leaves(l, u):
        if l == 0:
            return [u]
        out = []
        for c in tree.child[off[l] + u]:
            if c >= 0:
                out += leaves(l - 1, int(c))
        return out

    for l in range(tree.n_levels):
        for u in range(0, tree.level_size[l], max(1, tree.level_size[l] // 7)):
            s = np.zeros(64)
            for b in leaves(l, u):
                s += y[cache.members[b, :cache.count[b]:4] // 4].sum(axis=0)
            ref = s / np.linalg.norm(s)
            assert np.max(np.abs(tree.centroid[off[l] + u] - ref)) < 1e-6


def test_pairing_is_greedy_min_cost():
    """Tree pairing brute force: each pair taken is the least-cost pair among
    the nodes still unpaired (fp64), and at most one node stays alone."""
    rng = np.random.default_rng(21)
    for m in (2, 5, 9, 16):
        w = rng.integers(1, 20, m).astype(np.int32)
        mu = rng.standard_normal((m, 64)).astype(np.float32)
        partner = O.pair_run(mu, w)
        assert int((partner < 0).sum()) == m % 2
        mu64 = mu.astype(np.float64)

        def cost(a, b):
            return w[a] * w[b] / (w[a] + w[b]) * float(np.sum((mu64[a] - mu64[b]) ** 2))

        pairs = sorted({(min(i, int(p)), max(i, int(p))) for i, p in enumerate(partner) if p >= 0},
                       key=lambda ab: cost(*ab))
        free = set(range(m))
        for a, b in pairs:
            best = min(cost(x, y) for x in free for y in free if x < y)
            assert cost(a, b) <= best * (1 + 1e-5)
            free -= {a, b}


# ---------------------------------------------------------------- a4-a7

@pytest.fixture(scope="module")
def tiny():
    T = 4096
    keys = I.index_keys(0, T, 32)
    cache = O.build_cache(keys)
    pos = np.arange(T, dtype=np.int64)
    q = I.index_queries(0, keys, pos)
    return keys, cache, pos, q


def test_qnorm_is_bf16_of_unit_query(tiny):
    _, _, _, q = tiny
    qh = O.qnorm(q[:64])
    q64 = q[:64].astype(np.float64)
    unit = q64 / np.linalg.norm(q64, axis=1, keepdims=True)
    ref = torch.from_numpy(unit).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    diff = np.abs(O.bf16_bits_to_f32(qh) - O.bf16_bits_to_f32(ref))
    assert diff.max() <= 2.0 ** -8  # at most one bf16 ulp apart (fp32 vs fp64 normalisation)


def test_flat_rank_brute_force(tiny):
    """Flat ranking = every visible bucket, by fp64 score desc then id asc."""
    _, cache, pos, q = tiny
    cbf = O.bf16_bits_to_f32(cache.centroid_bf16).astype(np.float64)
    for p in (600, 1500, 2047, 3000, 4095):
        qh = O.qnorm(q[p])[0]
        H = p // 512
        ids, sc = O.flat_rank(qh, H, cache)
        assert len(ids) == 64 * H
        ref = (cbf[:64 * H] @ O.bf16_bits_to_f32(qh).astype(np.float64)).astype(np.float32)
        order = sorted(range(64 * H), key=lambda b: (-ref[b], b))
        assert list(ids) == order
        assert np.array_equal(sc, ref[order])


def test_dense_when_k_covers_everything(tiny):
    """Flat search with k >= p + 1 lists every causal key: dense attention."""
    _, cache, pos, q = tiny
    sel = np.array([0, 1, 3, 4, 511, 512, 513, 1023, 1024, 2500, 4095])
    lists, lens = O.index(q[sel], pos[sel], cache, k=4096)
    for i, p in enumerate(sel):
        assert lens[i] == p + 1
        assert np.array_equal(lists[i, :p + 1], np.arange(p + 1))
        assert np.all(lists[i, p + 1:] == -1)


def test_list_invariants(tiny):
    _, cache, pos, q = tiny
    k = 256
    lists, lens = O.index(q, pos, cache, k=k)
    for i in range(0, 4096, 37):
        p = int(pos[i])
        L = lists[i, :lens[i]]
        assert np.all(np.diff(L) > 0) and L[-1] == p and L[0] == 0
        near = set(range(min(4, p + 1))) | set(range(max(0, p - 512), p + 1))
        assert near <= set(L.tolist())
        H = p // 512
        clustered_near = len([t for t in near if t < 512 * H])
        avail = 512 * H - clustered_near
        assert lens[i] == len(near) + min(k, avail)
        assert np.all(lists[i, lens[i]:] == -1)


def test_worked_query_counts():
    """The blog's worked query (token 23,711): the first 4 and latest 512 keys
    are read unscored, leaving 23,195 far keys; Flat scores 2,944 buckets
    (46 complete blocks x 64)."""
    with open(os.path.join(GOLDEN, "worked_query.json")) as f:
        g = json.load(f)
    T = 24576
    keys = I.index_keys(3, T, 64)
    cache = O.build_cache(keys)
    p = g["query_position"]
    qh = O.qnorm(I.index_queries(3, keys, np.array([p]))[0])[0]
    ids, _ = O.flat_rank(qh, p // 512, cache)
    assert len(ids) == g["buckets_scored"]
    lists, lens = O.index(I.index_queries(3, keys, np.array([p])), np.array([p]), cache, k=10 ** 6)
    # every key up to p is listed (the unclustered ones all lie in the window),
    # so the far keys are the listed ones minus the 4 sink + 513 window keys
    assert lens[0] == p + 1
    assert lens[0] - (g["sink"] + g["window"] + 1) == g["far_keys"]


def test_expand_skips_near_and_refills():
    """The blog's rule: a key of an opened bucket that is already in the window
    or the first 4 is skipped and the next key takes its place; the list is
    sink + far + window, sorted."""
    cache = O.Cache(1536)
    cache.members[:] = -1
    cache.count[:] = 0
    # bucket 0: keys 600..603 (inside the window of p = 1030), bucket 1: 8..11,
    # bucket 2: 100..107, bucket 3: 2..3 and 40..41 (2, 3 are sink keys)
    spec = {0: [600, 601, 602, 603], 1: [8, 9, 10, 11], 2: list(range(100, 108)), 3: [2, 3, 40, 41]}
    for b, mem in spec.items():
        cache.members[b, :len(mem)] = mem
        cache.count[b] = len(mem)
    out, n = O.expand(np.array([0, 3, 1, 2]), cache, p=1030, k=7)
    want = [0, 1, 2, 3, 8, 9, 10, 11, 40, 41, 100] + list(range(518, 1031))
    assert n == len(want)
    assert list(out[:n]) == want
    assert np.all(out[n:] == -1)


# ---------------------------------------------------------------- multi-head Flat search

def test_heads_one_head_is_flat(tiny):
    _, cache, pos, q = tiny
    sel = np.arange(0, 4096, 53)
    lf, nf = O.index(q[sel], pos[sel], cache, k=256)
    lh, nh = O.index_heads(q[sel][:, None, :], pos[sel], cache, k=256)
    assert np.array_equal(nf, nh) and np.array_equal(lf, lh)


def test_heads_identical_and_rescaled_heads_are_flat(tiny):
    """Each head is normalised on its own, so copies of one query, each scaled
    by its own positive factor, select what the single query selects."""
    _, cache, pos, q = tiny
    sel = np.arange(7, 4096, 71)
    lf, nf = O.index(q[sel], pos[sel], cache, k=200)
    scale = np.array([1.0, 3.0, 0.25, 17.0], np.float32)
    qh = q[sel][:, None, :] * scale[None, :, None]
    lh, nh = O.index_heads(qh, pos[sel], cache, k=200)
    assert np.array_equal(nf, nh) and np.array_equal(lf, lh)


def test_heads_max_score_brute_force(tiny):
    """Buckets ranked by the best per-head score (fp64 products rounded to
    fp32, score desc then id asc), then the usual expansion."""
    keys, cache, pos, q = tiny
    cbf = O.bf16_bits_to_f32(cache.centroid_bf16).astype(np.float64)
    rng = np.random.default_rng(11)
    nh = 3
    for p in (700, 1800, 3333, 4095):
        qs = np.concatenate([q[p][None], rng.standard_normal((nh - 1, 64)).astype(np.float32)])
        H = p // 512
        best = np.full(64 * H, -np.inf, np.float32)
        for h in range(nh):
            qb = O.bf16_bits_to_f32(O.qnorm(qs[h])[0]).astype(np.float64)
            best = np.maximum(best, (cbf[:64 * H] @ qb).astype(np.float32))
        order = np.array(sorted(range(64 * H), key=lambda b: (-best[b], b)), np.int64)
        want, n = O.expand(order, cache, p=p, k=300)
        got, m = O.index_heads(qs[None], np.array([p]), cache, k=300)
        assert m[0] == n and np.array_equal(got[0, :m[0]], want[:n])


def test_heads_centroid_head_opens_its_bucket(tiny):
    """A head equal to a bucket's centroid scores that bucket near 1, above
    every other head's score for it, so its keys head the far part."""
    keys, cache, pos, q = tiny
    p = 4000
    b = 3 * 64 + 17
    c = O.bf16_bits_to_f32(cache.centroid_bf16[b])
    qs = np.stack([q[p], c, -q[p]])
    lists, lens = O.index_heads(qs[None], np.array([p]), cache, k=int(cache.count[b]))
    mem = cache.members[b, :cache.count[b]]
    far = [t for t in mem if 4 <= t < p - 512]
    assert set(far) <= set(lists[0, :lens[0]].tolist())


# ---------------------------------------------------------------- a6 tree search

def test_wide_beam_tree_equals_flat(tiny):
    """A beam at least as wide as every level keeps every visible node, so Tree
    search reduces to Flat search."""
    _, cache, pos, q = tiny
    tree = O.build_tree(cache)
    sel = np.arange(0, 4096, 61)
    lf, nf = O.index(q[sel], pos[sel], cache, k=256)
    lt, nt = O.index(q[sel], pos[sel], cache, k=256, mode="tree", tree=tree, beam=int(tree.level_size[0]))
    assert np.array_equal(nf, nt) and np.array_equal(lf, lt)


def test_tree_beam_keeps_visible_and_sizes(tiny):
    _, cache, pos, q = tiny
    tree = O.build_tree(cache)
    P = O.top_p(256)
    for p in (1024, 2600, 4095):
        qh = O.qnorm(q[p])[0]
        H = p // 512
        ids, sc = O.tree_rank(qh, H, tree, beam=32, P=P)
        assert len(ids) == min(P, 64 * H)  # P kept at level 0 whenever that many buckets are visible
        assert np.all(ids // 64 < H)  # only visible buckets
        assert len(set(ids.tolist())) == len(ids)
        assert np.all(np.diff(sc) <= 0)


# A hand-built tree of 16 leaves (levels of 16, 8, 4, 2, 1 nodes; node j of a
# level has children 2j, 2j + 1 below it).  The query is the unit vector e0
# and every node's bf16 centroid is (v / 64) e0, so a node scores exactly
# v / 64: the values below fix every beam decision, and the expected kept
# sets and per-level counts were worked out by hand from the beam rule
# (candidates = children of the nodes kept one level up, plus visible nodes
# whose parent is not visible; keep the best max(W, ceil(P / 2^l))).
# Leaves 0-7 score highest, so Flat search would take them first; the beam
# reaches them only through their ancestors.
_HB_VALUES = {
    0: [63, 62, 61, 60, 59, 58, 57, 56, 49, 48, 50, 55, 52, 53, 51, 54],
    1: [44, 39, 47, 46, 40, 43, 41, 42],
    2: [25, 5, 30, 31],
    3: [10, 20],
    4: [1],
}


def _hand_tree(block_of_leaf):
    t = O.Tree(16)
    assert t.level_size.tolist() == [16, 8, 4, 2, 1]
    off = t.level_offset
    e0 = np.zeros(64, np.float64)
    for lev, vals in _HB_VALUES.items():
        for j, v in enumerate(vals):
            g = off[lev] + j
            e0[0] = v / 64.0
            t.centroid_bf16[g] = O.f32_to_bf16_bits(e0.astype(np.float32))
            t.child[g] = [2 * j, 2 * j + 1] if lev > 0 else [-1, -1]
            t.parent[g] = j // 2 if lev < 4 else -1
            leaves = np.arange(j << lev, (j + 1) << lev)
            t.max_block[g] = max(block_of_leaf(int(x)) for x in leaves)
            t.min_block[g] = min(block_of_leaf(int(x)) for x in leaves)
    return t


def _e0_query():
    x = np.zeros(64, np.float32)
    x[0] = 1.0
    return O.f32_to_bf16_bits(x)


@pytest.mark.parametrize("case", [
    # (leaf -> block, H, W, P, expected level-0 ids in rank order, kept per level 0..4)
    ("all", 99, 1, 5, [11, 15, 13, 12, 14], [5, 3, 2, 1, 1]),
    ("all", 99, 1, 9, [0, 1, 11, 15, 13, 12, 14, 10, 8], [9, 5, 3, 2, 1]),
    ("all", 99, 3, 5, [0, 1, 11, 15, 14], [5, 3, 3, 2, 1]),
    ("quarter", 3, 1, 5, [0, 1, 11, 10, 8], [5, 3, 2, 1, 0]),
    ("half", 3, 1, 5, [0, 1, 2, 3, 4], [5, 3, 1, 0, 0]),
])
def test_tree_beam_width_per_level_hand_built(case):
    """The beam keeps max(W, ceil(P / 2^l)) nodes at level l (capped by the
    candidates): a floor in place of the ceiling, a min in place of the max,
    or W alone changes the counts or the kept leaves of at least one case.
    The 'quarter' and 'half' cases hide the right part of the tree (leaf i in
    block i // 4 or i // 2, horizon 3 blocks), so the search starts from
    visible nodes whose parent is not visible."""
    mapping, H, W, P, want_ids, want_kept = case
    blk = {"all": lambda i: 0, "quarter": lambda i: i // 4, "half": lambda i: i // 2}[mapping]
    tree = _hand_tree(blk)
    ids, sc, kept = O.tree_rank(_e0_query(), H, tree, beam=W, P=P, trace=True)
    assert kept.tolist() == want_kept
    assert ids.tolist() == want_ids
    assert np.array_equal(sc, np.array([_HB_VALUES[0][i] / 64.0 for i in want_ids], np.float32))


@pytest.mark.parametrize("k", [16, 64, 256, 1024])
def test_tree_narrowest_beam_still_fills_k(tiny, k):
    """With the narrowest beam (W = 1) the buckets kept at level 0 still hold
    k far keys whenever that many are visible: every list has
    min(p + 1, |near| + k) entries, as Flat search gives."""
    _, cache, pos, q = tiny
    tree = O.build_tree(cache)
    sel = np.arange(0, 4096, 37)
    lt, nt = O.index(q[sel], pos[sel], cache, k=k, mode="tree", tree=tree, beam=1)
    for i, p in enumerate(sel):
        w0 = max(0, p - 512)
        near = (p - w0 + 1) + min(4, w0)
        visible_far = 512 * min(p // 512, 8) - min(4, w0) - max(0, 512 * min(p // 512, 8) - w0)
        want = near + min(k, visible_far)
        assert nt[i] == want, (p, nt[i], want)


def test_tree_recall_of_flat_top_buckets_grows_with_beam(tiny):
    """Diagnostic of the beam's width: the share of Flat's top-P buckets that
    Tree search keeps rises with W, and is 1 once W covers every level."""
    _, cache, pos, q = tiny
    tree = O.build_tree(cache)
    P = O.top_p(64)
    sel = np.arange(1024, 4096, 29)
    recall = []
    for W in (1, 4, 8, 16, 32, 64, 512):
        r = []
        for p in sel:
            qh = O.qnorm(q[p])[0]
            H = p // 512
            fids, _ = O.flat_rank(qh, H, cache)
            tids, _ = O.tree_rank(qh, H, tree, beam=W, P=P)
            top = set(fids[:P].tolist())
            r.append(len(top & set(tids[:P].tolist())) / len(top))
        recall.append(float(np.mean(r)))
    assert all(b >= a - 1e-12 for a, b in zip(recall, recall[1:])), recall
    assert recall[-1] == 1.0 and recall[0] < 1.0, recall


# ---------------------------------------------------------------- a8 attention

def test_attention_single_key_is_value():
    rng = np.random.default_rng(5)
    Qb, Kb, Vb = I.qkv_bf16_bits(2, 4, 16, 8, 2)
    lists = np.array([[5, -1], [0, -1], [15, -1], [7, -1]], np.int32)
    lens = np.array([1, 1, 1, 1], np.int32)
    O_, lse = O.attention(Qb, Kb, Vb, lists, lens)
    V = O.bf16_bits_to_f32(Vb)
    for i in range(4):
        for h in range(8):
            assert np.array_equal(O_[i, h], V[lists[i, 0], h // 4])
    del rng


def test_attention_dense_causal_matches_torch_sdpa():
    """With every causal key listed, the oracle is causal softmax attention:
    compared with torch's scaled_dot_product_attention in fp64 (GQA by
    repeating KV heads)."""
    nq, hq, hkv = 40, 8, 2
    Qb, Kb, Vb = I.qkv_bf16_bits(3, nq, nq, hq, hkv)
    lists = np.full((nq, nq), -1, np.int32)
    for p in range(nq):
        lists[p, :p + 1] = np.arange(p + 1)
    lens = np.arange(1, nq + 1, dtype=np.int32)
    O_, lse = O.attention(Qb, Kb, Vb, lists, lens)
    f = lambda b: torch.from_numpy(O.bf16_bits_to_f32(b).astype(np.float64))
    q = f(Qb).permute(1, 0, 2)
    k = f(Kb).permute(1, 0, 2).repeat_interleave(hq // hkv, dim=0)
    v = f(Vb).permute(1, 0, 2).repeat_interleave(hq // hkv, dim=0)
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True).permute(1, 0, 2).numpy()
    assert np.max(np.abs(O_ - ref)) < 1e-6
    s = (q @ k.transpose(1, 2)) / math.sqrt(128)
    s = s.masked_fill(torch.triu(torch.ones(nq, nq, dtype=torch.bool), 1), float("-inf"))
    ref_lse = torch.logsumexp(s, dim=-1).permute(1, 0).numpy()
    assert np.max(np.abs(lse - ref_lse)) < 1e-5


def test_attention_identical_keys_average_values():
    nq, hq, hkv, n = 3, 4, 1, 50
    Qb, Kb, Vb = I.qkv_bf16_bits(4, nq, n, hq, hkv)
    Kb[:] = Kb[0]
    lists = np.tile(np.arange(n, dtype=np.int32), (nq, 1))
    lens = np.full(nq, n, np.int32)
    O_, _ = O.attention(Qb, Kb, Vb, lists, lens)
    V = O.bf16_bits_to_f32(Vb).astype(np.float64)
    assert np.max(np.abs(O_ - V[:, 0].mean(axis=0))) < 1e-6


def test_bucket_cache_bytes_per_token():
    """The pages' 24.5 B/token: per 512-key block, 64 buckets x (64 bf16
    centroid + 16 int32 member slots + 1 int32 count)."""
    per_block = 64 * (64 * 2 + 16 * 4 + 4)
    assert per_block / 512 == 24.5


# --- step 1, "Shrink": x_t = W v_t ------------------------------------------

BF16_ONE, BF16_MINUS_ONE = 0x3F80, 0xBF80


def test_shrink_one_hot_rows_select_dims():
    """W with one 1.0 per row picks input dims: a dropped term, a transposed
    operand or a wrong index breaks the equality."""
    rng = np.random.default_rng(5)
    D = 256
    V = I.normal_bf16_bits(5, 701, (37, D))
    idx = rng.choice(D, 64, replace=False)
    W = np.zeros((64, D), np.uint16)
    W[np.arange(64), idx] = BF16_ONE
    assert np.array_equal(O.shrink(V, W), O.bf16_bits_to_f32(V)[:, idx])


def test_shrink_signed_permutation_keeps_norms():
    """A signed permutation (orthogonal) of 64 dims: each output is plus or
    minus one input, so the norm of every row is unchanged."""
    rng = np.random.default_rng(6)
    V = I.normal_bf16_bits(6, 702, (50, 64))
    perm, sign = rng.permutation(64), rng.integers(0, 2, 64)
    W = np.zeros((64, 64), np.uint16)
    W[np.arange(64), perm] = np.where(sign == 1, BF16_MINUS_ONE, BF16_ONE)
    x, v = O.shrink(V, W), O.bf16_bits_to_f32(V)
    assert np.array_equal(x, np.where(sign == 1, -1.0, 1.0).astype(np.float32) * v[:, perm])
    assert np.allclose(np.linalg.norm(x.astype(np.float64), axis=1), np.linalg.norm(v.astype(np.float64), axis=1),
                       rtol=1e-12)


def test_shrink_small_integers_exact():
    """Small integers are exact in bf16, fp64 and fp32: the projection must
    equal the integer contraction sum_d v_td w_ed exactly (D = 1024)."""
    rng = np.random.default_rng(7)
    D = 1024
    vi = rng.integers(-4, 5, (19, D))
    wi = rng.integers(-3, 4, (64, D))
    to_bits = lambda a: (a.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)  # noqa: E731
    x = O.shrink(to_bits(vi), to_bits(wi))
    exact = np.einsum("td,ed->te", vi, wi)  # integer arithmetic
    assert np.array_equal(x, exact.astype(np.float32))


# ---------------------------------------------------------------- selection arguments the merges rely on

@pytest.mark.parametrize("seed", range(6))
def test_union_of_head_candidates_holds_top_p_by_best_score(seed):
    """Every head lists every bucket scoring >= tau_h, tau_h <= its P-th
    score.  Then the buckets listed at or above tau* = max_h tau_h, each with
    the best score any head listed for it, hold the top P by best score over
    all heads, with exact values (quantised scores make ties likely)."""
    rng = np.random.default_rng(seed)
    H, N, P = int(rng.integers(2, 9)), int(rng.integers(50, 400)), int(rng.integers(5, 40))
    S = np.round(rng.standard_normal((H, N)) * 8) / 8  # many ties
    taus = [np.sort(S[h])[::-1][P - 1] - rng.uniform(0, 0.5) for h in range(H)]
    tstar = max(taus)
    known = {}
    for h in range(H):
        for b in np.nonzero(S[h] >= taus[h])[0]:
            if S[h, b] >= tstar:
                known[b] = max(known.get(b, -np.inf), S[h, b])
    best = S.max(0)
    top = sorted(range(N), key=lambda b: (-best[b], b))[:P]
    got = sorted(known, key=lambda b: (-known[b], b))[:P]
    assert got == top
    assert all(known[b] == best[b] for b in top)


@pytest.mark.parametrize("seed", range(6))
def test_union_of_shard_top_p_holds_global_top_p(seed):
    """Each shard sends its own top P (by score desc, id asc); the top P of
    the union is the global top P."""
    rng = np.random.default_rng(100 + seed)
    N, P, R = int(rng.integers(80, 600)), int(rng.integers(5, 60)), int(rng.integers(2, 9))
    s = np.round(rng.standard_normal(N) * 6) / 6
    cuts = np.sort(rng.choice(np.arange(1, N), R - 1, replace=False))
    parts = np.split(np.arange(N), cuts)
    union = []
    for ids in parts:
        union += sorted(ids.tolist(), key=lambda b: (-s[b], b))[:P]
    key = lambda b: (-s[b], b)  # noqa: E731
    assert sorted(union, key=key)[:P] == sorted(range(N), key=key)[:P]
