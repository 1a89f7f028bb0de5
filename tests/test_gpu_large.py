"""GPU parity at the measured workload sizes: T = 131072, 1,048,576 (Flat and
Tree) and 10,000,000 tokens.  The bucket cache and the tree are compared in
full; the index lists and the attention on sampled queries (the oracle
computes those one by one), including decode positions past the context.
Rules are in tests/parity.py."""
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


def _gpu_index(cache, tree, p, q, pos, decode=False):
    nq = len(pos)
    Lmax = lsa.lsa_list_budget(p)
    lists = torch.empty((nq, Lmax), dtype=torch.int32, device="cuda")
    lens = torch.empty((nq,), dtype=torch.int32, device="cuda")
    ws = lsa.workspace(lsa.lsa_index_workspace_bytes(nq, cache.n_blocks, p))
    fn = lsa.lsa_index_decode if decode else lsa.lsa_index_prefill
    fn(PT.to_dev(q), PT.to_dev(np.asarray(pos, np.int64)), cache, tree, lists, lens, p, ws)
    torch.cuda.synchronize()
    return lists, lens


def _attention_sampled(lists_d, lens_d, sel, T_kv, hq, hkv, seed):
    """GPU attention over all listed queries; oracle on the sampled rows, with
    K/V rows gathered for exactly the listed positions."""
    nq = lists_d.shape[0]
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    Q = torch.randn((nq, hq, 128), generator=g, device="cuda").to(torch.bfloat16)
    K = torch.randn((T_kv, hkv, 128), generator=g, device="cuda").to(torch.bfloat16)
    V = torch.randn((T_kv, hkv, 128), generator=g, device="cuda").to(torch.bfloat16)
    O_ = torch.empty_like(Q)
    lse = torch.empty((nq, hq), dtype=torch.float32, device="cuda")
    ws = lsa.workspace(lsa.lsa_attention_workspace_bytes(nq, hq, 128, lists_d.shape[1], T_kv))
    lsa.lsa_sparse_attention(Q, K, V, lists_d, lens_d, O_, lse, ws=ws)
    torch.cuda.synchronize()
    lists = lists_d[sel].cpu().numpy()
    lens = lens_d[sel].cpu().numpy()
    used = np.unique(lists[lists >= 0])
    remap = {int(v): i for i, v in enumerate(used)}
    ll = np.where(lists >= 0, np.vectorize(lambda v: remap.get(int(v), -1))(lists), -1).astype(np.int32)
    ui = torch.from_numpy(used.astype(np.int64)).cuda()
    bits = lambda t: t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)  # noqa: E731
    Oref, lse_ref = O.attention(bits(Q[torch.from_numpy(sel).cuda()]), bits(K.index_select(0, ui)),
                                bits(V.index_select(0, ui)), ll, lens)
    return PT.assert_attention_close(O_[torch.from_numpy(sel).cuda()], Oref, lse[torch.from_numpy(sel).cuda()],
                                     lse_ref)


def _check_tree(gtree, otree):
    assert gtree.level_sizes() == otree.level_size.tolist()
    v = {k: t.cpu().numpy() for k, t in gtree.views().items()}
    for name in ("child", "parent", "weight", "min_block", "max_block"):
        assert np.array_equal(v[name], getattr(otree, name)), f"tree {name} differs"
    assert np.array_equal(v["sum"].view(np.uint32), otree.sum.view(np.uint32))
    assert np.array_equal(v["centroid_bf16"].view(np.uint16), otree.centroid_bf16)


@pytest.fixture(scope="module")
def big128k():
    _need_gpu()
    wl = I.WORKLOADS["flat_128k"]
    T, k = wl["T"], wl["k"]
    keys = I.index_keys(0, T, wl["n_components"])
    oc = O.build_cache(keys)
    p = lsa.lsa_default_params(k=k)
    cache = lsa.Cache(T)
    lsa.lsa_build_cache(PT.to_dev(keys), 0, T, cache, p)
    torch.cuda.synchronize()
    return wl, keys, oc, cache


def test_flat_128k_cache_index_attention(big128k):
    wl, keys, oc, cache = big128k
    T, k = wl["T"], wl["k"]
    p = lsa.lsa_default_params(k=k)
    PT.assert_cache_equal(PT.cache_to_numpy(cache, T), oc)
    # all queries through the GPU (the benchmark's launch), 600 sampled for the oracle
    pos = np.arange(T, dtype=np.int64)
    q = I.index_queries(0, keys, pos)
    lists_d, lens_d = _gpu_index(cache, None, p, q, pos)
    sel = np.unique(np.concatenate([np.linspace(0, T - 1, 560).astype(np.int64),
                                    [0, 3, 511, 512, 1023, 1024, 65535, 65536, T - 2, T - 1]]))
    ol, on = O.index(q[sel], pos[sel], oc, k=k)
    PT.assert_lists_match(lists_d[torch.from_numpy(sel).cuda()].cpu().numpy(),
                          lens_d[torch.from_numpy(sel).cuda()].cpu().numpy(), ol, on, q[sel], pos[sel], oc, k=k)
    _attention_sampled(lists_d, lens_d, sel[::10], T, wl["hq"], wl["hkv"], seed=1)


def test_flat_128k_index_heads(big128k):
    """Multi-head Flat search with 8 index heads over every position, in the
    benchmark's launches (chunks of 16384 queries); sampled queries against
    the oracle."""
    wl, keys, oc, cache = big128k
    T, k, heads, chunk = wl["T"], wl["k"], 8, 16384
    p = lsa.lsa_default_params(k=k, index_heads=heads)
    pos = np.arange(T, dtype=np.int64)
    q = I.index_queries_heads(11, keys, pos, heads)
    Lmax = lsa.lsa_list_budget(p)
    lists = torch.empty((T, Lmax), dtype=torch.int32, device="cuda")
    lens = torch.empty((T,), dtype=torch.int32, device="cuda")
    ws = lsa.workspace(lsa.lsa_index_workspace_bytes(chunk, cache.n_blocks, p))
    qd, pd = PT.to_dev(q), PT.to_dev(pos)
    for a in range(0, T, chunk):
        lsa.lsa_index_prefill(qd[a:a + chunk], pd[a:a + chunk], cache, None, lists[a:a + chunk], lens[a:a + chunk],
                              p, ws)
    torch.cuda.synchronize()
    del ws
    sel = np.unique(np.concatenate([np.linspace(0, T - 1, 190).astype(np.int64),
                                    [0, 511, 512, 1024, 16383, 16384, 65536, T - 1]]))
    ol, on = O.index_heads(q[sel], pos[sel], oc, k=k)
    ix = torch.from_numpy(sel).cuda()
    PT.assert_lists_match(lists[ix].cpu().numpy(), lens[ix].cpu().numpy(), ol, on, q[sel], pos[sel], oc, k=k)


@pytest.fixture(scope="module")
def big1m():
    _need_gpu()
    wl = I.WORKLOADS["flat_1m"]
    T = wl["T"]
    keys_all = I.index_keys(0, T + wl["n_decode"], wl["n_components"])
    keys = keys_all[:T]
    oc = O.build_cache(keys)
    p = lsa.lsa_default_params(k=wl["k"], mode="tree", beam=32)
    cache = lsa.Cache(T)
    lsa.lsa_build_cache(PT.to_dev(keys), 0, T, cache, p)
    tree = lsa.Tree(T // 512)
    lsa.lsa_build_tree(cache, tree, p)
    torch.cuda.synchronize()
    return wl, keys_all, oc, cache, tree


def test_1m_cache_and_tree_bit_exact(big1m):
    wl, keys_all, oc, cache, tree = big1m
    PT.assert_cache_equal(PT.cache_to_numpy(cache, wl["T"]), oc)
    _check_tree(tree, O.build_tree(oc))


def _sample(n: int, count: int = 1024) -> np.ndarray:
    """Evenly spaced sample of `count` of n prefill queries (all of them when
    n <= count): the queries the oracle checks one by one."""
    return np.unique(np.linspace(0, n - 1, min(n, count)).astype(np.int64))


def _decode_one_by_one(cache, tree, p, dq, dpos):
    """lsa_index_decode at batch 1 for every decode token, in order."""
    gl, gn = [], []
    for i in range(len(dpos)):
        l1, n1 = _gpu_index(cache, tree, p, dq[i:i + 1], dpos[i:i + 1], decode=True)
        gl.append(l1.cpu().numpy()[0])
        gn.append(int(n1.cpu().numpy()[0]))
    return np.stack(gl), np.array(gn)


def _decode_attention(gl, gn, T_kv, hq, hkv, seed):
    """Batch-1 attention (the split-list path) for every decode token's list,
    against the oracle."""
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    nd = len(gn)
    Q = torch.randn((nd, hq, 128), generator=g, device="cuda").to(torch.bfloat16)
    K = torch.randn((T_kv, hkv, 128), generator=g, device="cuda").to(torch.bfloat16)
    V = torch.randn((T_kv, hkv, 128), generator=g, device="cuda").to(torch.bfloat16)
    Lmax = gl.shape[1]
    O_ = torch.empty_like(Q)
    lse = torch.empty((nd, hq), dtype=torch.float32, device="cuda")
    ws = lsa.workspace(lsa.lsa_attention_workspace_bytes(1, hq, 128, Lmax))
    ld, nd_ = PT.to_dev(gl), PT.to_dev(gn)
    for i in range(nd):
        lsa.lsa_sparse_attention(Q[i:i + 1], K, V, ld[i:i + 1], nd_[i:i + 1], O_[i:i + 1], lse[i:i + 1], ws=ws)
    torch.cuda.synchronize()
    used = np.unique(gl[gl >= 0])
    remap = np.full(T_kv, -1, np.int64)
    remap[used] = np.arange(len(used))
    ll = np.where(gl >= 0, remap[np.maximum(gl, 0)], -1).astype(np.int32)
    ui = torch.from_numpy(used.astype(np.int64)).cuda()
    bits = lambda t: t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)  # noqa: E731
    Oref, lse_ref = O.attention(bits(Q), bits(K.index_select(0, ui)), bits(V.index_select(0, ui)), ll, gn)
    return PT.assert_attention_close(O_, Oref, lse, lse_ref)


def test_1m_flat_prefill_and_decode(big1m):
    """1M Flat: every prefill query indexed in the benchmark's one launch,
    1024 evenly spaced of them against the oracle, attention of every query
    in one launch with 128 sampled; then each of the 64 decode tokens indexed
    and attended at batch 1, all against the oracle."""
    wl, keys_all, oc, cache, _ = big1m
    T, k, npre, ndec = wl["T"], wl["k"], wl["n_prefill"], wl["n_decode"]
    p = lsa.lsa_default_params(k=k)
    pos = np.arange(T - npre, T, dtype=np.int64)
    q = I.index_queries(0, keys_all, pos)
    lists_d, lens_d = _gpu_index(cache, None, p, q, pos)
    sel = _sample(npre)
    ol, on = O.index(q[sel], pos[sel], oc, k=k)
    ix = torch.from_numpy(sel).cuda()
    PT.assert_lists_match(lists_d[ix].cpu().numpy(), lens_d[ix].cpu().numpy(), ol, on, q[sel], pos[sel], oc, k=k)
    _attention_sampled(lists_d, lens_d, sel[::8], T + ndec, wl["hq"], wl["hkv"], seed=2)
    del lists_d, lens_d
    dpos = np.arange(T, T + ndec, dtype=np.int64)
    dq = I.index_queries(1, keys_all, dpos)
    gl, gn = _decode_one_by_one(cache, None, p, dq, dpos)
    ol, on = O.index(dq, dpos, oc, k=k)
    PT.assert_lists_match(gl, gn, ol, on, dq, dpos, oc, k=k)
    _decode_attention(gl, gn, T + ndec, wl["hq"], wl["hkv"], seed=12)


def test_1m_context_parallel_eight_ranks(big1m):
    """The 1M Flat prefill split over 8 ranks in the zig-zag layout (16 chunks
    of 128 blocks, rank r holding chunks r and 15 - r), the
    ranks run stage by stage in this process in the benchmark's chunks of
    16384 queries: lists equal the single-GPU lists of every query (the same
    tensor-core score for every (query, bucket), the same tie order), sampled
    lists equal the oracle's, sampled combined attention its attention."""
    from hierarchical_key_clustering_b200 import context_parallel as CP

    wl, keys_all, oc, cache, _ = big1m
    T, k, npre = wl["T"], wl["k"], wl["n_prefill"]
    hq, hkv, chunk, ranks = wl["hq"], wl["hkv"], 16384, 8
    pos = np.arange(T - npre, T, dtype=np.int64)
    q = I.index_queries(0, keys_all, pos)
    shards = [CP.Shard(r, ranks, T, k=k, max_queries=chunk, layout="zigzag") for r in range(ranks)]
    kd = PT.to_dev(keys_all[:T])
    built = [s.build(kd) for s in shards]
    M, C = torch.stack([b[0] for b in built]), torch.stack([b[1] for b in built])
    for s in shards:
        s.set_members(M, C)
    del kd
    g = torch.Generator(device="cuda")
    g.manual_seed(5)
    Q = torch.randn((npre, hq, 128), generator=g, device="cuda").to(torch.bfloat16)
    K = torch.randn((T, hkv, 128), generator=g, device="cuda").to(torch.bfloat16)
    V = torch.randn((T, hkv, 128), generator=g, device="cuda").to(torch.bfloat16)
    qd, pd = PT.to_dev(q), PT.to_dev(pos)
    lists = torch.empty((npre, shards[0].Lmax), dtype=torch.int32, device="cuda")
    lens = torch.empty((npre,), dtype=torch.int32, device="cuda")
    O_ = torch.empty_like(Q)
    lse = torch.empty((npre, hq), dtype=torch.float32, device="cuda")
    for c0 in range(0, npre, chunk):
        c1 = min(npre, c0 + chunk)
        X = torch.stack([s.index_local(qd[c0:c1], pd[c0:c1]) for s in shards]).reshape(-1)
        l_, n_ = shards[0].index_merge(X, pd[c0:c1])
        lists[c0:c1].copy_(l_)
        lens[c0:c1].copy_(n_)
        parts = [s.attend_local(Q[c0:c1], K, V, lists[c0:c1], lens[c0:c1]) for s in shards]
        o, l2 = CP.Shard.combine(torch.stack([x[0] for x in parts]), torch.stack([x[1] for x in parts]))
        O_[c0:c1].copy_(o)
        lse[c0:c1].copy_(l2)
    torch.cuda.synchronize()
    single_l, single_n = _gpu_index(cache, None, lsa.lsa_default_params(k=k), q, pos)
    same = (lens == single_n) & torch.all(lists == single_l, dim=1)
    assert same.float().mean().item() >= 0.999, f"only {same.float().mean().item():.4f} equal the single-GPU lists"
    sel = np.linspace(0, npre - 1, 96).astype(np.int64)
    ix = torch.from_numpy(sel).cuda()
    ol, on = O.index(q[sel], pos[sel], oc, k=k)
    PT.assert_lists_match(lists[ix].cpu().numpy(), lens[ix].cpu().numpy(), ol, on, q[sel], pos[sel], oc, k=k)
    sa = sel[::6]
    ia = torch.from_numpy(sa).cuda()
    la, na = lists[ia].cpu().numpy(), lens[ia].cpu().numpy()
    used = np.unique(la[la >= 0])
    remap = np.full(T, -1, np.int64)
    remap[used] = np.arange(len(used))
    ll = np.where(la >= 0, remap[np.maximum(la, 0)], -1).astype(np.int32)
    ui = torch.from_numpy(used.astype(np.int64)).cuda()
    bits = lambda t: t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)  # noqa: E731
    Oref, lse_ref = O.attention(bits(Q[ia]), bits(K.index_select(0, ui)), bits(V.index_select(0, ui)), ll, na)
    PT.assert_attention_close(O_[ia], Oref, lse[ia], lse_ref)


def test_1m_context_parallel_merge_past_shared_memory(big1m):
    """16 ranks in the zig-zag layout (32 chunks of 64 blocks) over the 1M
    workload: the union of the chunks' candidate sets (~32 x 1.1 P entries)
    no longer fits the merge kernel's shared memory, so the merge reads it
    from the exchange blocks; lists equal the single-GPU lists, sampled ones
    the oracle's."""
    from hierarchical_key_clustering_b200 import context_parallel as CP

    wl, keys_all, oc, cache, _ = big1m
    T, k, npre = wl["T"], wl["k"], wl["n_prefill"]
    ranks, nq = 16, 2048
    pos = np.arange(T - npre, T, dtype=np.int64)[np.linspace(0, npre - 1, nq).astype(np.int64)]
    q = I.index_queries(0, keys_all, pos)
    shards = [CP.Shard(r, ranks, T, k=k, max_queries=nq, layout="zigzag") for r in range(ranks)]
    kd = PT.to_dev(keys_all[:T])
    built = [s.build(kd) for s in shards]
    M, C = torch.stack([b[0] for b in built]), torch.stack([b[1] for b in built])
    for s in shards:
        s.set_members(M, C)
    del kd
    qd, pd = PT.to_dev(q), PT.to_dev(pos)
    X = torch.stack([s.index_local(qd, pd) for s in shards]).reshape(-1)
    cnt = lsa.lsa_shard_exchange_bytes(nq, shards[0].p)
    slots = lsa.lsa_shard_slots(shards[0].p)
    counts = torch.stack([X[i * cnt:i * cnt + nq * 4].view(torch.int32).clamp(max=slots)
                          for i in range(2 * ranks)]).sum(0)
    assert int(counts.min()) * 8 > 200 * 1024  # every query's union is read from global memory
    lists, lens = shards[0].index_merge(X, pd)
    single_l, single_n = _gpu_index(cache, None, lsa.lsa_default_params(k=k), q, pos)
    same = (lens == single_n) & torch.all(lists == single_l, dim=1)
    assert same.float().mean().item() >= 0.999, f"only {same.float().mean().item():.4f} equal the single-GPU lists"
    sel = np.linspace(0, nq - 1, 64).astype(np.int64)
    ix = torch.from_numpy(sel).cuda()
    ol, on = O.index(q[sel], pos[sel], oc, k=k)
    PT.assert_lists_match(lists[ix].cpu().numpy(), lens[ix].cpu().numpy(), ol, on, q[sel], pos[sel], oc, k=k)


def test_1m_tree_prefill_and_decode(big1m):
    """1M Tree (beam 32): every prefill query in one launch, 1024 evenly
    spaced against the oracle; each of the 64 decode tokens at batch 1 (the
    small-batch beam kernel) against the oracle."""
    wl, keys_all, oc, cache, tree = big1m
    T, k, npre, ndec = wl["T"], wl["k"], wl["n_prefill"], wl["n_decode"]
    ot = O.build_tree(oc)
    p = lsa.lsa_default_params(k=k, mode="tree", beam=32)
    pos = np.arange(T - npre, T, dtype=np.int64)
    q = I.index_queries(0, keys_all, pos)
    lists_d, lens_d = _gpu_index(cache, tree, p, q, pos)
    sel = _sample(npre)
    ix = torch.from_numpy(sel).cuda()
    ol, on = O.index(q[sel], pos[sel], oc, k=k, mode="tree", tree=ot, beam=32)
    PT.assert_lists_match(lists_d[ix].cpu().numpy(), lens_d[ix].cpu().numpy(), ol, on, q[sel], pos[sel], oc, k=k,
                          tree=ot, beam=32)
    del lists_d, lens_d
    dpos = np.arange(T, T + ndec, dtype=np.int64)
    dq = I.index_queries(1, keys_all, dpos)
    gl, gn = _decode_one_by_one(cache, tree, p, dq, dpos)
    ol, on = O.index(dq, dpos, oc, k=k, mode="tree", tree=ot, beam=32)
    PT.assert_lists_match(gl, gn, ol, on, dq, dpos, oc, k=k, tree=ot, beam=32)


def test_10m_flat_and_tree():
    """10,000,000 tokens: 19531 complete blocks and an unclustered tail of 128.
    The full cache and tree bit-exact; Flat and Tree prefill of the last 65536
    positions, each in one launch as the benchmark runs them, with 1024 evenly
    spaced queries of each against the oracle; all 128 decode tokens at batch
    1 in both modes against the oracle; attention over 41 GB of K/V for
    sampled prefill queries and for every Flat decode token."""
    _need_gpu()
    wl = I.WORKLOADS["flat_tree_10m"]
    T, k, npre, ndec = wl["T"], wl["k"], wl["n_prefill"], wl["n_decode"]
    hq, hkv = wl["hq"], wl["hkv"]
    keys_all = I.index_keys(0, T + ndec, wl["n_components"])
    keys = keys_all[:T]
    oc = O.build_cache(keys)
    p = lsa.lsa_default_params(k=k)
    cache = lsa.Cache(T)
    lsa.lsa_build_cache(PT.to_dev(keys), 0, T, cache, p)
    tree = lsa.Tree(T // 512)
    pt = lsa.lsa_default_params(k=k, mode="tree", beam=32)
    lsa.lsa_build_tree(cache, tree, pt)
    torch.cuda.synchronize()
    assert cache.n_blocks == 19531
    PT.assert_cache_equal(PT.cache_to_numpy(cache, T), oc)
    ot = O.build_tree(oc)
    _check_tree(tree, ot)
    del keys
    pos = np.arange(T - npre, T, dtype=np.int64)
    q = I.index_queries(0, keys_all, pos)
    sel = _sample(npre)
    ix = torch.from_numpy(sel).cuda()
    # Tree first (its lists are dropped before the Flat ones are made)
    tl, tn = _gpu_index(cache, tree, pt, q, pos)
    otl, otn = O.index(q[sel], pos[sel], oc, k=k, mode="tree", tree=ot, beam=32)
    PT.assert_lists_match(tl[ix].cpu().numpy(), tn[ix].cpu().numpy(), otl, otn, q[sel], pos[sel], oc, k=k,
                          tree=ot, beam=32)
    del tl, tn
    lists_d, lens_d = _gpu_index(cache, None, p, q, pos)
    ol, on = O.index(q[sel], pos[sel], oc, k=k)
    PT.assert_lists_match(lists_d[ix].cpu().numpy(), lens_d[ix].cpu().numpy(), ol, on, q[sel], pos[sel], oc, k=k)
    _attention_sampled(lists_d, lens_d, sel[::16], T + ndec, hq, hkv, seed=3)
    del lists_d, lens_d
    torch.cuda.empty_cache()
    dpos = np.arange(T, T + ndec, dtype=np.int64)
    dq = I.index_queries(1, keys_all, dpos)
    gl, gn = _decode_one_by_one(cache, None, p, dq, dpos)
    ol, on = O.index(dq, dpos, oc, k=k)
    PT.assert_lists_match(gl, gn, ol, on, dq, dpos, oc, k=k)
    _decode_attention(gl, gn, T + ndec, hq, hkv, seed=13)
    tgl, tgn = _decode_one_by_one(cache, tree, pt, dq, dpos)
    otl, otn = O.index(dq, dpos, oc, k=k, mode="tree", tree=ot, beam=32)
    PT.assert_lists_match(tgl, tgn, otl, otn, dq, dpos, oc, k=k, tree=ot, beam=32)
