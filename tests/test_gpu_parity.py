"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the
same seeded inputs.  Rules are in tests/parity.py."""
import numpy as np
import pytest
import torch

import oracle as O
from hierarchical_key_clustering_b200 import inputs as I
from hierarchical_key_clustering_b200 import lsa

from . import parity as PT

pytestmark = pytest.mark.gpu


def _need_gpu():
    if not torch.cuda.is_available():
        pytest.fail("a CUDA GPU is required for the -m gpu tests")


def _build_gpu(keys: np.ndarray, capacity=None, pieces=None, mode="flat", k=256, beam=32, cand_cap=0,
               index_heads=1):
    _need_gpu()
    T = keys.shape[0]
    cache = lsa.Cache(capacity or T)
    p = lsa.lsa_default_params(k=k, mode=mode, beam=beam, cand_cap=cand_cap, index_heads=index_heads)
    kd = PT.to_dev(keys)
    if pieces is None:
        pieces = [(0, T)]
    for a, b in pieces:
        lsa.lsa_build_cache(kd, a, b, cache, p)
    tree = None
    if mode == "tree":
        tree = lsa.Tree(max(T // 512, 1))
        lsa.lsa_build_tree(cache, tree, p)
    torch.cuda.synchronize()
    return cache, tree, p


def _index_gpu(cache, tree, p, qidx, pos, decode=False):
    nq = len(pos)
    Lmax = lsa.lsa_list_budget(p)
    lists = torch.empty((nq, Lmax), dtype=torch.int32, device="cuda")
    lens = torch.empty((nq,), dtype=torch.int32, device="cuda")
    ws = lsa.workspace(lsa.lsa_index_workspace_bytes(nq, cache.n_blocks, p))
    fn = lsa.lsa_index_decode if decode else lsa.lsa_index_prefill
    fn(PT.to_dev(qidx), PT.to_dev(np.asarray(pos, np.int64)), cache, tree, lists, lens, p, ws)
    torch.cuda.synchronize()
    return lists.cpu().numpy(), lens.cpu().numpy()


@pytest.fixture(scope="module")
def tiny():
    T = 4096
    keys = I.index_keys(0, T, 32)
    pos = np.arange(T, dtype=np.int64)
    q = I.index_queries(0, keys, pos)
    oc = O.build_cache(keys)
    return keys, q, pos, oc


def test_cache_bit_exact_tiny(tiny):
    keys, _, _, oc = tiny
    cache, _, _ = _build_gpu(keys)
    assert cache.n_blocks == 8
    PT.assert_cache_equal(PT.cache_to_numpy(cache, 4096), oc)


def test_cache_incremental_and_ragged_tail():
    """Building in uneven pieces gives the one-shot cache; a tail shorter than
    a block is pooled but not clustered."""
    T = 4096 + 300
    keys = I.index_keys(1, T, 32)
    oc = O.build_cache(keys)
    cache, _, _ = _build_gpu(keys, capacity=T + 212, pieces=[(0, 1001), (1001, 2600), (2600, 2601), (2601, T)])
    assert cache.n_blocks == 8
    g = PT.cache_to_numpy(cache, T)
    PT.assert_cache_equal(g, oc)


def test_flat_index_all_queries_tiny(tiny):
    keys, q, pos, oc = tiny
    cache, _, p = _build_gpu(keys, k=256)
    gl, gn = _index_gpu(cache, None, p, q, pos)
    ol, on = O.index(q, pos, oc, k=256)
    PT.assert_lists_match(gl, gn, ol, on, q, pos, oc, k=256)


@pytest.mark.parametrize("k", [1, 7, 256, 5000])
def test_flat_index_edge_positions(tiny, k):
    """Positions before the first block, inside the sink, at block edges, and k
    from 1 to more than every key (dense); ragged query count."""
    keys, q, _, oc = tiny
    pos = np.array([0, 1, 2, 3, 4, 5, 511, 512, 513, 515, 516, 1023, 1024, 1025, 1535, 2047, 2048, 3000, 4095,
                    4095, 2049] + list(range(600, 4096, 61)), np.int64)
    qq = q[pos]
    cache, _, p = _build_gpu(keys, k=k)
    gl, gn = _index_gpu(cache, None, p, qq, pos)
    ol, on = O.index(qq, pos, oc, k=k)
    PT.assert_lists_match(gl, gn, ol, on, qq, pos, oc, k=k)
    if k == 5000:
        for i, pp in enumerate(pos):
            assert gn[i] == pp + 1 and np.array_equal(gl[i, :pp + 1], np.arange(pp + 1))


def test_flat_exact_fallback_selection(tiny):
    """With only P candidate slots per query, most queries overflow and take the
    exact radix-select path; the lists must not change."""
    keys, q, pos, oc = tiny
    P = O.top_p(256)
    cache, _, p = _build_gpu(keys, k=256, cand_cap=P)
    sel = np.arange(0, 4096, 5)
    gl, gn = _index_gpu(cache, None, p, q[sel], pos[sel])
    ol, on = O.index(q[sel], pos[sel], oc, k=256)
    PT.assert_lists_match(gl, gn, ol, on, q[sel], pos[sel], oc, k=256)


@pytest.fixture(scope="module")
def ctx96k():
    """192 full blocks (12288 buckets) and a ragged tail of 300 keys."""
    T = 98304 + 300
    keys = I.index_keys(5, T, 32)
    pos = np.arange(T, dtype=np.int64)
    q = I.index_queries(5, keys, pos)
    return keys, q, O.build_cache(keys)


@pytest.mark.parametrize("stride,margin", [(2, 1.25), (4, 1.25), (4, 0.9), (2, 0.5), (2, 0.01)])
def test_flat_sampled_threshold(ctx96k, stride, margin):
    """Flat search's threshold taken from every stride-th centroid tile (a
    batch of > 28K queries, each seeing >= 128 blocks, so that one CTA scans a
    query tile's whole bucket range): the lists are the exact ones.  With
    margin 1.25 about 1.25 P buckets (~10 k far keys) lie above tau, so no
    query is redone and the lists equal the full histogram's bit for bit.
    Smaller margins (the default 0.9 among them) may put tau above the cut
    for some queries (0.5) or every one (0.01), which is then redone by the
    exact selection: its scores come from the CUDA cores instead of the
    tensor cores, so near-ties may order differently, and those lists are
    held to the oracle's near-tie rule on a denser sample."""
    keys, q, oc = ctx96k
    T = keys.shape[0]
    sel = np.arange(66000, T, dtype=np.int64)
    qq = q[sel]
    cache, _, p = _build_gpu(keys, k=256)
    try:
        lsa.lsa_debug_score_sample(1)
        el, en = _index_gpu(cache, None, p, qq, sel)
        lsa.lsa_debug_score_sample(stride, margin)
        lsa.lsa_kernel_timing(1)
        gl, gn = _index_gpu(cache, None, p, qq, sel)
        names = list(lsa.lsa_kernel_timing_read())
    finally:
        lsa.lsa_kernel_timing(0)
        lsa.lsa_debug_score_sample()
    assert "k_score_tc:sampled" in names
    assert np.array_equal(gn, en)
    if margin >= 1.0:
        L = int(en.max())
        mask = np.arange(L)[None, :] < en[:, None]
        assert np.array_equal(np.where(mask, gl[:, :L], -1), np.where(mask, el[:, :L], -1))
    sub = np.arange(0, len(sel), 41 if margin >= 1.0 else 7)
    ol, on = O.index(qq[sub], sel[sub], oc, k=256)
    PT.assert_lists_match(gl[sub], gn[sub], ol, on, qq[sub], sel[sub], oc, k=256)


@pytest.mark.parametrize("cand_cap", [0, 193])
def test_decode_positions_past_context(tiny, cand_cap):
    """Decode: new tokens at or past the clustered context see every block
    (small batches take the stored-score path; cand_cap = P forces its exact
    fallback selection)."""
    keys, _, _, oc = tiny
    T = 4096
    more = I.index_keys(0, T + 16, 32)
    pos = np.arange(T, T + 16, dtype=np.int64)
    qq = I.index_queries(9, more, pos)
    cache, _, p = _build_gpu(keys, k=256, cand_cap=cand_cap)
    for nq in (1, 3, 16):
        gl, gn = _index_gpu(cache, None, p, qq[:nq], pos[:nq], decode=True)
        ol, on = O.index(qq[:nq], pos[:nq], oc, k=256)
        PT.assert_lists_match(gl, gn, ol, on, qq[:nq], pos[:nq], oc, k=256)


@pytest.mark.parametrize("k", [1, 7, 256, 5000])
def test_small_batches_edge_positions(tiny, k):
    """Batches of <= 16 queries (one wide CTA per query ranks and cuts, the
    far keys are written block by block by a second kernel) at the edge
    positions: before the first block, in the sink, at block edges, with the
    window over clustered blocks, k from 1 to dense."""
    keys, q, _, oc = tiny
    pos = np.array([0, 1, 4, 5, 511, 512, 513, 515, 516, 1023, 1024, 1025, 1535, 2047, 2048, 2049, 3000, 4095,
                    4094, 600, 661, 3999, 1500, 2600], np.int64)
    cache, _, p = _build_gpu(keys, k=k)
    for a in range(0, len(pos), 16):
        pp = pos[a:a + 16]
        qq = q[pp]
        gl, gn = _index_gpu(cache, None, p, qq, pp)
        ol, on = O.index(qq, pp, oc, k=k)
        PT.assert_lists_match(gl, gn, ol, on, qq, pp, oc, k=k)


@pytest.mark.parametrize("heads,k,cand_cap", [(2, 256, 0), (4, 256, 0), (8, 5000, 0), (3, 7, 0), (4, 256, 193)])
def test_flat_index_heads_against_oracle(tiny, heads, k, cand_cap):
    """Multi-head Flat search (a bucket ranks by its best head score), every
    position class of the edge test, ragged count; cand_cap = P makes rows
    overflow, so queries take the merge's exact path."""
    keys, _, _, oc = tiny
    pos = np.array([0, 3, 4, 511, 512, 513, 1023, 1024, 2047, 2048, 3000, 4095] + list(range(600, 4096, 37)),
                   np.int64)
    qq = I.index_queries_heads(5, keys, pos, heads)
    cache, _, p = _build_gpu(keys, k=k, cand_cap=cand_cap, index_heads=heads)
    gl, gn = _index_gpu(cache, None, p, qq, pos)
    ol, on = O.index_heads(qq, pos, oc, k=k)
    PT.assert_lists_match(gl, gn, ol, on, qq, pos, oc, k=k)


def test_flat_index_heads_exact_path_many_queries(tiny):
    """With P entry slots per row most rows past the first blocks overflow, so
    their queries are redone by the exact kernel, which runs one CTA per SM:
    1600 queries give each CTA several marked queries to compact and work
    through."""
    keys, _, _, oc = tiny
    P = O.top_p(256)
    pos = np.concatenate([np.arange(512, 4096, 3), np.arange(2000, 2400)]).astype(np.int64)[:1600]
    qq = I.index_queries_heads(13, keys, pos, 3)
    cache, _, p = _build_gpu(keys, k=256, cand_cap=P, index_heads=3)
    gl, gn = _index_gpu(cache, None, p, qq, pos)
    sel = np.arange(0, len(pos), 7)
    ol, on = O.index_heads(qq[sel], pos[sel], oc, k=256)
    PT.assert_lists_match(gl[sel], gn[sel], ol, on, qq[sel], pos[sel], oc, k=256)


def test_flat_index_heads_decode_and_single_head(tiny):
    """Decode batches (stored-score path) with 4 heads, and identical heads,
    which must give the single-head lists exactly."""
    keys, _, _, oc = tiny
    T = 4096
    more = I.index_keys(0, T + 8, 32)
    pos = np.arange(T, T + 8, dtype=np.int64)
    qq = I.index_queries_heads(9, more, pos, 4)
    cache, _, p = _build_gpu(keys, k=256, index_heads=4)
    for nq in (1, 4):
        gl, gn = _index_gpu(cache, None, p, qq[:nq], pos[:nq], decode=True)
        ol, on = O.index_heads(qq[:nq], pos[:nq], oc, k=256)
        PT.assert_lists_match(gl, gn, ol, on, qq[:nq], pos[:nq], oc, k=256)
    same = np.ascontiguousarray(np.repeat(qq[:, :1], 4, axis=1))
    p1 = lsa.lsa_default_params(k=256)
    g4, n4 = _index_gpu(cache, None, p, same, pos)
    g1, n1 = _index_gpu(cache, None, p1, np.ascontiguousarray(same[:, 0]), pos)
    assert np.array_equal(n4, n1) and np.array_equal(g4, g1)


def test_tree_build_bit_exact(tiny):
    keys, _, _, oc = tiny
    ot = O.build_tree(oc)
    cache, tree, _ = _build_gpu(keys, mode="tree")
    assert tree.level_sizes() == ot.level_size.tolist()
    v = {k: t.cpu().numpy() for k, t in tree.views().items()}
    for name in ("child", "parent", "weight", "min_block", "max_block"):
        assert np.array_equal(v[name], getattr(ot, name)), f"tree {name} differs"
    assert np.array_equal(v["sum"].view(np.uint32), ot.sum.view(np.uint32))
    assert np.max(np.abs(v["centroid"] - ot.centroid)) <= 1e-6
    assert np.array_equal(v["centroid_bf16"].view(np.uint16), ot.centroid_bf16)


def _assert_tree_levels_equal(tree, ot):
    """Level by level (the GPU tree is laid out for its capacity, the
    oracle's compactly): every node array bit-exact, centroids within 1e-6."""
    assert tree.level_sizes() == ot.level_size.tolist()
    v = {k: t.cpu().numpy() for k, t in tree.views().items()}
    for l, n in enumerate(tree.level_sizes()):
        g0, o0 = tree.t.level_offset[l], int(ot.level_offset[l])
        for name in ("child", "parent", "weight", "min_block", "max_block"):
            assert np.array_equal(v[name][g0:g0 + n], getattr(ot, name)[o0:o0 + n]), f"level {l} {name} differs"
        assert np.array_equal(v["sum"][g0:g0 + n].view(np.uint32), ot.sum[o0:o0 + n].view(np.uint32))
        assert np.max(np.abs(v["centroid"][g0:g0 + n] - ot.centroid[o0:o0 + n])) <= 1e-6
        assert np.array_equal(v["centroid_bf16"][g0:g0 + n].view(np.uint16), ot.centroid_bf16[o0:o0 + n])


def test_tree_grows_in_place_as_blocks_complete(tiny):
    """Decode-time growth: the cache takes new keys (ragged steps included),
    and after each step the tree, extended by lsa_update_tree in a buffer laid
    out for 8 blocks, equals the oracle's tree over the same prefix and a full
    rebuild; the index over it matches the oracle's Tree lists."""
    _need_gpu()
    keys, q, pos, _ = tiny
    p = lsa.lsa_default_params(k=256, mode="tree", beam=32)
    cache, tree, full = lsa.Cache(4096), lsa.Tree(8), lsa.Tree(8)
    kd = PT.to_dev(keys)
    t = 0
    for t_end in (1536, 2048, 2748, 3072, 3584, 4096):
        lsa.lsa_build_cache(kd, t, t_end, cache, p)
        lsa.lsa_update_tree(cache, tree, p)
        t = t_end
        torch.cuda.synchronize()
        ot = O.build_tree(O.build_cache(keys[:t_end]))
        _assert_tree_levels_equal(tree, ot)
        lsa.lsa_build_tree(cache, full, p)
        torch.cuda.synchronize()
        va, vb = tree.views(), full.views()
        for l, n in enumerate(tree.level_sizes()):  # the nodes in use (the rest of the buffer is never written)
            g0 = tree.t.level_offset[l]
            assert all(torch.equal(va[k][g0:g0 + n], vb[k][g0:g0 + n]) for k in va), f"level {l} differs"
    oc = O.build_cache(keys)
    sel = np.arange(1000, 4096, 37)
    gl, gn = _index_gpu(cache, tree, p, q[sel], pos[sel])
    ol, on = O.index(q[sel], pos[sel], oc, k=256, mode="tree", tree=O.build_tree(oc), beam=32)
    PT.assert_lists_match(gl, gn, ol, on, q[sel], pos[sel], oc, k=256, tree=O.build_tree(oc), beam=32)


@pytest.mark.parametrize("beam", [32, 4, 512])
def test_tree_index_tiny(tiny, beam):
    keys, q, pos, oc = tiny
    ot = O.build_tree(oc)
    cache, tree, p = _build_gpu(keys, mode="tree", k=256, beam=beam)
    sel = np.arange(0, 4096, 3)
    gl, gn = _index_gpu(cache, tree, p, q[sel], pos[sel])
    ol, on = O.index(q[sel], pos[sel], oc, k=256, mode="tree", tree=ot, beam=beam)
    PT.assert_lists_match(gl, gn, ol, on, q[sel], pos[sel], oc, k=256, tree=ot, beam=beam)
    if beam == 512:  # wide beam: Tree search is Flat search
        fl, fn = O.index(q[sel], pos[sel], oc, k=256)
        PT.assert_lists_match(gl, gn, fl, fn, q[sel], pos[sel], oc, k=256)


@pytest.mark.parametrize("beam", [32, 4])
def test_tree_decode_small_batches(tiny, beam):
    """Tree search for decode batches of 1, 4 and 16 queries (the small-batch
    beam kernel: one query per 16-warp team) against the oracle, for tokens
    past the clustered context and for interior positions."""
    keys, q, pos, oc = tiny
    T = 4096
    ot = O.build_tree(oc)
    more = I.index_keys(0, T + 16, 32)
    dpos = np.concatenate([np.arange(T, T + 8, dtype=np.int64), np.array([513, 1024, 2047, 2600, 3000, 3583, 3584,
                                                                          4095], dtype=np.int64)])
    dq = I.index_queries(9, more, dpos)
    cache, tree, p = _build_gpu(keys, mode="tree", k=256, beam=beam)
    for nq in (1, 4, 16):
        for a in range(0, 16, nq):
            gl, gn = _index_gpu(cache, tree, p, dq[a:a + nq], dpos[a:a + nq], decode=True)
            ol, on = O.index(dq[a:a + nq], dpos[a:a + nq], oc, k=256, mode="tree", tree=ot, beam=beam)
            PT.assert_lists_match(gl, gn, ol, on, dq[a:a + nq], dpos[a:a + nq], oc, k=256, tree=ot, beam=beam)


@pytest.mark.parametrize("nq,consecutive", [(300, False), (1, False), (200, True)])
def test_attention_peaked_softmax(tiny, nq, consecutive):
    """Q scaled by 8 (exact in bf16): the softmax of each row is dominated by a
    few keys, so a dropped, duplicated or misplaced key moves the output by
    about the size of a value row and fails the tolerance.  The gather path,
    the split-list path (nq = 1) and the near-set tiles (consecutive
    queries).  Score rounding grows with the scores, so lse is held to 8x
    the usual bound."""
    _need_gpu()
    keys, q, pos, oc = tiny
    hq, hkv = 32, 8
    if consecutive:
        sel = np.arange(1500, 1500 + nq, dtype=np.int64)
    else:
        sel = np.sort(np.random.default_rng(nq).choice(4096, size=nq, replace=False)).astype(np.int64)
    ol, on = O.index(q[sel], pos[sel], oc, k=256)
    Qb, Kb, Vb = I.qkv_bf16_bits(21, nq, 4096, hq, hkv)
    Q8 = PT.bits_to_bf16(Qb) * 8
    Q8b = Q8.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    Oref, lse_ref = O.attention(Q8b, Kb, Vb, ol, on)
    Kd, Vd = PT.bits_to_bf16(Kb), PT.bits_to_bf16(Vb)
    Od = torch.empty_like(Q8)
    lse = torch.empty((nq, hq), dtype=torch.float32, device="cuda")
    ws = lsa.workspace(lsa.lsa_attention_workspace_bytes(nq, hq, 128, ol.shape[1]))
    lsa.lsa_sparse_attention(Q8, Kd, Vd, PT.to_dev(ol), PT.to_dev(on), Od, lse, ws=ws)
    torch.cuda.synchronize()
    PT.assert_attention_close(Od, Oref)
    assert np.abs(lse.cpu().numpy() - lse_ref).max() <= 8 * PT.LSE_TOL
    # the check has teeth: dropping each list's highest-scoring key for head 0
    # moves the oracle's output far past the tolerance
    Qf = O.bf16_bits_to_f32(Q8b).astype(np.float64)
    Kf = O.bf16_bits_to_f32(Kb).astype(np.float64)
    drop, dn = ol.copy(), on.copy()
    for i in range(nq):
        keys_i = ol[i, :on[i]]
        j = int(np.argmax(Kf[keys_i, 0] @ Qf[i, 0]))
        drop[i, j:dn[i] - 1] = drop[i, j + 1:dn[i]]
        drop[i, dn[i] - 1] = -1
        dn[i] -= 1
    Odrop, _ = O.attention(Q8b, Kb, Vb, drop, dn)
    assert np.abs(Odrop[:, 0] - Oref[:, 0]).max(axis=1).min() > PT.ATT_MAX


@pytest.mark.parametrize("rows,hq,hkv,consecutive", [(300, 32, 8, False), (1000, 8, 1, True), (4096, 32, 8, False),
                                                    (97, 16, 16, False), (513, 32, 8, True), (700, 16, 1, False)])
def test_attention_position_ranges_against_oracle(tiny, rows, hq, hkv, consecutive):
    """The gather taken in position ranges (one launch per KV head and range,
    a running result per (query, head) carried between launches), forced on
    the small workload with ranges of `rows` positions: ragged last ranges,
    queries with nothing in some ranges, an empty list and a one-key list,
    against the oracle (output and lse)."""
    _need_gpu()
    keys, q, pos, oc = tiny
    nq = max(300, -(-2048 // hkv))  # enough (query, KV head) units to keep whole lists (no key splits)
    if consecutive:
        sel = np.arange(4096 - nq, 4096, dtype=np.int64)
    else:
        sel = np.sort(np.random.default_rng(rows).choice(4096, size=nq, replace=False)).astype(np.int64)
    ol, on = O.index(q[sel], pos[sel], oc, k=256)
    ol[5] = -1
    on[5] = 0  # an empty list
    ol[6, 1:] = -1
    on[6] = 1  # one key
    Qb, Kb, Vb = I.qkv_bf16_bits(rows, nq, 4096, hq, hkv)
    Oref, lse_ref = O.attention(Qb, Kb, Vb, ol, on)
    Qd, Kd, Vd = PT.bits_to_bf16(Qb), PT.bits_to_bf16(Kb), PT.bits_to_bf16(Vb)
    Od = torch.empty_like(Qd)
    lse = torch.empty((nq, hq), dtype=torch.float32, device="cuda")
    lsa.lsa_debug_attention_ranges(rows)
    try:
        ws = lsa.workspace(lsa.lsa_attention_workspace_bytes(nq, hq, 128, ol.shape[1], 4096))
        lsa.lsa_kernel_timing(True)
        lsa.lsa_sparse_attention(Qd, Kd, Vd, PT.to_dev(ol), PT.to_dev(on), Od, lse, ws=ws)
        torch.cuda.synchronize()
        lsa.lsa_kernel_timing(False)
        kt = lsa.lsa_kernel_timing_read()
    finally:
        lsa.lsa_debug_attention_ranges(0)
    assert "k_range_plan" in kt and kt["k_attn"][1] == 1  # the phased path ran (one timed record)
    og = Od.float().cpu().numpy()
    assert np.all(og[5] == 0) and np.all(np.isneginf(lse.cpu().numpy()[5]))
    keep = np.ones(nq, bool)
    keep[5] = False
    PT.assert_attention_close(Od[torch.from_numpy(np.nonzero(keep)[0]).cuda()], Oref[keep],
                              lse[torch.from_numpy(np.nonzero(keep)[0]).cuda()], lse_ref[keep])


@pytest.mark.parametrize("hq,hkv,nq", [(8, 1, 300), (32, 8, 200), (32, 8, 1), (8, 1, 2), (16, 16, 50)])
def test_attention_against_oracle(tiny, hq, hkv, nq):
    """Attention over the oracle's own lists (isolates the kernel); nq = 1-2
    takes the split-list (decode) path."""
    _need_gpu()
    keys, q, pos, oc = tiny
    rng = np.random.default_rng(nq + hq)
    sel = np.sort(rng.choice(4096, size=nq, replace=False)).astype(np.int64)
    ol, on = O.index(q[sel], pos[sel], oc, k=256)
    Qb, Kb, Vb = I.qkv_bf16_bits(4, nq, 4096, hq, hkv)
    Oref, lse_ref = O.attention(Qb, Kb, Vb, ol, on)
    Qd, Kd, Vd = PT.bits_to_bf16(Qb), PT.bits_to_bf16(Kb), PT.bits_to_bf16(Vb)
    Od = torch.empty_like(Qd)
    lse = torch.empty((nq, hq), dtype=torch.float32, device="cuda")
    Lmax = ol.shape[1]
    ws = lsa.workspace(lsa.lsa_attention_workspace_bytes(nq, hq, 128, Lmax))
    lsa.lsa_sparse_attention(Qd, Kd, Vd, PT.to_dev(ol), PT.to_dev(on), Od, lse, ws=ws)
    torch.cuda.synchronize()
    PT.assert_attention_close(Od, Oref, lse, lse_ref)


@pytest.mark.parametrize("hq,hkv,p0,nq", [(32, 8, 1000, 300), (8, 1, 0, 200), (16, 1, 3000, 100), (16, 16, 2000, 130),
                                          (32, 8, 500, 64)])
def test_attention_near_tiles_against_oracle(tiny, hq, hkv, p0, nq):
    """Consecutive queries: their sink and window keys go through the
    near-set tiles (from position 0, where sink and window meet, up), the rest
    of each list through the gather; the merge must match the oracle."""
    _need_gpu()
    keys, q, pos, oc = tiny
    sel = np.arange(p0, p0 + nq, dtype=np.int64)
    ol, on = O.index(q[sel], pos[sel], oc, k=256)
    Qb, Kb, Vb = I.qkv_bf16_bits(7, nq, 4096, hq, hkv)
    Oref, lse_ref = O.attention(Qb, Kb, Vb, ol, on)
    Qd, Kd, Vd = PT.bits_to_bf16(Qb), PT.bits_to_bf16(Kb), PT.bits_to_bf16(Vb)
    Od = torch.empty_like(Qd)
    lse = torch.empty((nq, hq), dtype=torch.float32, device="cuda")
    ws = lsa.workspace(lsa.lsa_attention_workspace_bytes(nq, hq, 128, ol.shape[1]))
    lsa.lsa_sparse_attention(Qd, Kd, Vd, PT.to_dev(ol), PT.to_dev(on), Od, lse, ws=ws)
    torch.cuda.synchronize()
    PT.assert_attention_close(Od, Oref, lse, lse_ref)


@pytest.mark.parametrize("hq,hkv,p0,nq", [(32, 8, 1000, 300), (16, 16, 0, 130)])
def test_attention_near_tiles_ignore_rows_past_the_queries(tiny, hq, hkv, p0, nq):
    """K and V rows past the last query position (not in any list) hold NaN,
    as an unwritten cache tail may: the near-set tiles load whole 64-key
    boxes, so their partial last chunk must keep those rows out of O."""
    _need_gpu()
    keys, q, pos, oc = tiny
    sel = np.arange(p0, p0 + nq, dtype=np.int64)
    ol, on = O.index(q[sel], pos[sel], oc, k=256)
    Qb, Kb, Vb = I.qkv_bf16_bits(11, nq, 4096, hq, hkv)
    Oref, lse_ref = O.attention(Qb, Kb, Vb, ol, on)
    Kb, Vb = Kb.copy(), Vb.copy()
    Kb[p0 + nq:] = 0x7FC0  # bf16 NaN
    Vb[p0 + nq:] = 0x7FC0
    Qd, Kd, Vd = PT.bits_to_bf16(Qb), PT.bits_to_bf16(Kb), PT.bits_to_bf16(Vb)
    Od = torch.empty_like(Qd)
    lse = torch.empty((nq, hq), dtype=torch.float32, device="cuda")
    ws = lsa.workspace(lsa.lsa_attention_workspace_bytes(nq, hq, 128, ol.shape[1]))
    lsa.lsa_sparse_attention(Qd, Kd, Vd, PT.to_dev(ol), PT.to_dev(on), Od, lse, ws=ws)
    torch.cuda.synchronize()
    assert torch.isfinite(Od.float()).all()
    PT.assert_attention_close(Od, Oref, lse, lse_ref)


def test_attention_near_tiles_irregular_lists(tiny):
    """Lists without a window (random subsets ending at the query's position),
    and a batch whose positions jump inside a tile: the near-set plan must
    take only what each list holds and fall back to the gather otherwise."""
    _need_gpu()
    rng = np.random.default_rng(11)
    nq, hq, hkv, T = 257, 32, 8, 4096
    p = np.arange(1500, 1500 + nq, dtype=np.int64)
    p[100:] += 7  # tiles 3 (queries 96..127) and up: 3 is not consecutive
    Lmax = 600
    lists = np.full((nq, Lmax), -1, np.int32)
    lens = np.zeros(nq, np.int32)
    for i in range(nq):
        if i % 3 == 0:  # dense tail and head, random middle
            mid = np.sort(rng.choice(np.arange(6, p[i] - 300), size=100, replace=False))
            li = np.concatenate([np.arange(0, 6), mid, np.arange(p[i] - 299, p[i] + 1)])
        else:  # random subset that ends at p
            li = np.concatenate([np.sort(rng.choice(p[i], size=rng.integers(1, 500), replace=False)), [p[i]]])
        lists[i, :len(li)] = li
        lens[i] = len(li)
    Qb, Kb, Vb = I.qkv_bf16_bits(8, nq, T, hq, hkv)
    Oref, lse_ref = O.attention(Qb, Kb, Vb, lists, lens)
    Qd, Kd, Vd = PT.bits_to_bf16(Qb), PT.bits_to_bf16(Kb), PT.bits_to_bf16(Vb)
    Od = torch.empty_like(Qd)
    lse = torch.empty((nq, hq), dtype=torch.float32, device="cuda")
    ws = lsa.workspace(lsa.lsa_attention_workspace_bytes(nq, hq, 128, Lmax))
    lsa.lsa_sparse_attention(Qd, Kd, Vd, PT.to_dev(lists), PT.to_dev(lens), Od, lse, ws=ws)
    torch.cuda.synchronize()
    PT.assert_attention_close(Od, Oref, lse, lse_ref)


def test_attention_dense_causal_single_key(tiny):
    """A one-key list returns that key's value row exactly (up to bf16)."""
    _need_gpu()
    nq, hq, hkv = 5, 8, 2
    Qb, Kb, Vb = I.qkv_bf16_bits(5, nq, 64, hq, hkv)
    lists = np.full((nq, 4), -1, np.int32)
    lists[:, 0] = [3, 0, 63, 17, 17]
    lens = np.ones(nq, np.int32)
    Qd, Kd, Vd = PT.bits_to_bf16(Qb), PT.bits_to_bf16(Kb), PT.bits_to_bf16(Vb)
    Od = torch.empty_like(Qd)
    lsa.lsa_sparse_attention(Qd, Kd, Vd, PT.to_dev(lists), PT.to_dev(lens), Od)
    torch.cuda.synchronize()
    V = O.bf16_bits_to_f32(Vb)
    og = Od.float().cpu().numpy()
    for i in range(nq):
        for h in range(hq):
            assert np.array_equal(og[i, h], V[lists[i, 0], h // (hq // hkv)])


def test_end_to_end_tiny_layer(tiny):
    """Indexer + attention through the C ABI against oracle lists + oracle
    attention for the whole tiny workload (8 query heads, 1 KV head)."""
    keys, q, pos, oc = tiny
    cache, _, p = _build_gpu(keys, k=256)
    Lmax = lsa.lsa_list_budget(p)
    nq = 4096
    lists = torch.empty((nq, Lmax), dtype=torch.int32, device="cuda")
    lens = torch.empty((nq,), dtype=torch.int32, device="cuda")
    ws = lsa.workspace(lsa.lsa_index_workspace_bytes(nq, cache.n_blocks, p))
    lsa.lsa_index_prefill(PT.to_dev(q), PT.to_dev(pos), cache, None, lists, lens, p, ws)
    Qb, Kb, Vb = I.qkv_bf16_bits(0, nq, 4096, 8, 1)
    Qd, Kd, Vd = PT.bits_to_bf16(Qb), PT.bits_to_bf16(Kb), PT.bits_to_bf16(Vb)
    Od = torch.empty_like(Qd)
    lsa.lsa_sparse_attention(Qd, Kd, Vd, lists, lens, Od)
    torch.cuda.synchronize()
    gl, gn = lists.cpu().numpy(), lens.cpu().numpy()
    ol, on = O.index(q, pos, oc, k=256)
    PT.assert_lists_match(gl, gn, ol, on, q, pos, oc, k=256)
    sel = np.arange(0, nq, 4)
    Oref, _ = O.attention(Qb[sel], Kb, Vb, gl[sel], gn[sel])
    PT.assert_attention_close(Od[sel], Oref)


def test_small_and_large_batch_paths_agree(tiny):
    """Batches of up to 16 queries (decode path: CUDA-core scores) and larger
    batches (prefill path: tensor-core scores) give the oracle's lists for the
    same queries; the two score sums may differ in the last bit, so lists may
    differ only by near-ties at the k cut, and almost never do."""
    keys, q, pos, oc = tiny
    cache, _, p = _build_gpu(keys, k=256)
    sel = np.arange(100, 4096, 97)[:40].astype(np.int64)
    big_l, big_n = _index_gpu(cache, None, p, q[sel], pos[sel])
    ol, on = O.index(q[sel], pos[sel], oc, k=256)
    PT.assert_lists_match(big_l, big_n, ol, on, q[sel], pos[sel], oc, k=256)
    same = 0
    for a in range(0, len(sel), 8):
        sl, sn = _index_gpu(cache, None, p, q[sel[a:a + 8]], pos[sel[a:a + 8]], decode=True)
        PT.assert_lists_match(sl, sn, ol[a:a + 8], on[a:a + 8], q[sel[a:a + 8]], pos[sel[a:a + 8]], oc, k=256)
        same += sum(int(sn[i] == big_n[a + i] and np.array_equal(sl[i], big_l[a + i])) for i in range(len(sn)))
    assert same >= len(sel) - 2


def test_prefill_from_host_matches_device_path(tiny):
    """The pipelined host-memory step (copy streams, query chunks) gives the
    same O, bit for bit, as build + index + attend on device inputs (8 KV
    heads: every chunk has enough (query, head) units to keep whole lists)."""
    _need_gpu()
    from hierarchical_key_clustering_b200.layer import SparseLayer
    keys, q, pos, _ = tiny
    nq, hq, hkv = 4096, 32, 8
    Qb, Kb, Vb = I.qkv_bf16_bits(9, nq, 4096, hq, hkv)
    Qd, Kd, Vd = PT.bits_to_bf16(Qb), PT.bits_to_bf16(Kb), PT.bits_to_bf16(Vb)
    dev_layer = SparseLayer(4096, k=256, max_queries=nq, Hq=hq)
    dev_layer.build(PT.to_dev(keys))
    dev_layer.index(PT.to_dev(q), PT.to_dev(pos))
    Od = torch.empty_like(Qd)
    dev_layer.attend(Qd, Kd, Vd, Od)
    host_layer = SparseLayer(4096, k=256, max_queries=nq, Hq=hq)
    pin = lambda t: t.cpu().pin_memory()  # noqa: E731
    h_O = torch.empty(Qd.shape, dtype=Qd.dtype).pin_memory()
    for chunks in (5, 1):
        h_O.zero_()
        host_layer.prefill_from_host(pin(torch.from_numpy(keys)), pin(torch.from_numpy(q)),
                                     pin(torch.from_numpy(pos)), pin(Qd), pin(Kd), pin(Vd), h_O, chunks=chunks)
        torch.cuda.synchronize()
        assert torch.equal(h_O, Od.cpu())


@pytest.mark.parametrize("D,t_begin,t_end", [(1024, 0, 4096), (128, 512, 2100), (64, 4, 700)])
def test_shrink_against_oracle(D, t_begin, t_end):
    """Step 1 on the tensor cores: keys within the fp32 accumulation bound of
    the oracle's product, rows outside the range untouched; the fused pooled
    items match the oracle's pooling of its keys within the bound's effect,
    and are bit-identical to the cache build pooling the kernel's own keys."""
    _need_gpu()
    Vb = I.normal_bf16_bits(21, 901, (t_end, D))
    Wb = I.normal_bf16_bits(22, 902, (64, D))
    Vd, Wd = PT.bits_to_bf16(Vb), PT.bits_to_bf16(Wb)
    keys = torch.full((t_end, 64), float("nan"), dtype=torch.float32, device="cuda")
    pooled = torch.full((t_end // 4, 64), float("nan"), dtype=torch.float32, device="cuda")
    lsa.lsa_shrink(Vd, Wd, t_begin, t_end, keys=keys, pooled=pooled)
    torch.cuda.synchronize()
    ref = O.shrink(Vb, Wb)
    g = keys.cpu().numpy()
    assert np.isnan(g[:t_begin]).all()
    # fp32 accumulation of D exact products: |err| <= 2 D 2^-24 sum |v w| (+ output rounding)
    absdot = np.abs(O.bf16_bits_to_f32(Vb)).astype(np.float64) @ np.abs(O.bf16_bits_to_f32(Wb)).astype(np.float64).T
    bound = 2 * D * 2.0**-24 * absdot + np.abs(ref) * 2.0**-24
    err = np.abs(g[t_begin:] - ref[t_begin:])
    assert (err <= bound[t_begin:]).all(), f"max err/bound {np.max(err / bound[t_begin:]):.3g}"
    i0, i1 = t_begin // 4, t_end // 4
    gp = pooled.cpu().numpy()
    assert np.isnan(gp[:i0]).all()
    rp = O.pool_norm(ref[4 * i0:4 * i1])
    rel = np.max(bound[t_begin:] / np.maximum(np.linalg.norm(ref[t_begin:], axis=1, keepdims=True), 1e-30))
    assert np.max(np.abs(gp[i0:i1] - rp)) <= 8 * rel + 1e-6
    # the cache build's own pooling of the kernel's keys: bit-identical
    cache = lsa.Cache(-(-t_end // 512) * 512)
    lsa.lsa_build_cache(keys, t_begin, t_end, cache, lsa.lsa_default_params())
    torch.cuda.synchronize()
    cp = cache.views()["pooled"].cpu().numpy()
    assert np.array_equal(cp[i0:i1].view(np.uint32), gp[i0:i1].view(np.uint32))
