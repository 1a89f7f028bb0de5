"""GPU parity of the context-parallel path: the ranks of a token-range split
run in one process, stage by stage (each stage's launches in sequence, no
kernel waiting on another), the all-gathers replaced by stacking the ranks'
tensors in rank order.  The lists must equal the oracle's unsharded Flat
search and the combined attention its unsharded attention.  Rules are in
tests/parity.py."""
import numpy as np
import pytest
import torch

import oracle as O
from hierarchical_key_clustering_b200 import context_parallel as CP
from hierarchical_key_clustering_b200 import inputs as I

from . import parity as PT

pytestmark = pytest.mark.gpu


def _run(keys, qidx, pos, world, k, heads=1, hq=8, hkv=2, seed=3, layout="contiguous"):
    if not torch.cuda.is_available():
        pytest.fail("a CUDA GPU is required for the -m gpu tests")
    T = keys.shape[0]
    nq = len(pos)
    shards = [CP.Shard(r, world, T, k=k, index_heads=heads, max_queries=nq, layout=layout) for r in range(world)]
    kd = PT.to_dev(keys)
    built = [s.build(kd) for s in shards]
    M = torch.stack([b[0] for b in built])
    C = torch.stack([b[1] for b in built])
    for s in shards:
        s.set_members(M, C)
    qd, pd = PT.to_dev(qidx), PT.to_dev(np.asarray(pos, np.int64))
    X = torch.stack([s.index_local(qd, pd) for s in shards]).reshape(-1)
    res = [s.index_merge(X, pd) for s in shards]
    torch.cuda.synchronize()
    lists = [r[0].cpu().numpy() for r in res]
    lens = [r[1].cpu().numpy() for r in res]
    Qb, Kb, Vb = I.qkv_bf16_bits(seed, nq, T, hq, hkv)
    f = lambda a: PT.bits_to_bf16(a)  # noqa: E731
    Qd, Kd, Vd = f(Qb), f(Kb), f(Vb)
    parts = [s.attend_local(Qd, Kd, Vd, res[0][0], res[0][1]) for s in shards]
    Oc, lse = CP.Shard.combine(torch.stack([p[0] for p in parts]), torch.stack([p[1] for p in parts]))
    torch.cuda.synchronize()
    return shards, shards[0].members, lists, lens, (Qb, Kb, Vb), Oc, lse


@pytest.fixture(scope="module")
def tiny():
    T = 4096
    keys = I.index_keys(0, T, 32)
    oc = O.build_cache(keys)
    return keys, oc


@pytest.mark.parametrize("world,layout", [(2, "contiguous"), (3, "contiguous"), (4, "contiguous"),
                                          (5, "contiguous"), (2, "zigzag"), (3, "zigzag"), (4, "zigzag")])
def test_shards_lists_and_attention_match_unsharded_oracle(tiny, world, layout):
    """2-5 ranks over 8 blocks (3 ranks: 3 + 3 + 2 blocks; 5 ranks: the last
    holds nothing), and the zig-zag layout (rank r holds chunks r and
    2 world - 1 - r; 4 ranks: 8 one-block chunks; 3 ranks: two chunks
    empty): member table bit-exact, every rank the same lists, lists as the
    oracle's unsharded Flat search, combined attention as its unsharded
    attention."""
    keys, oc = tiny
    pos = np.array([0, 3, 4, 511, 512, 1023, 1024, 1535, 2047, 2048, 3071, 3072, 4095] + list(range(700, 4096, 29)),
                   np.int64)
    q = I.index_queries(4, keys, pos)
    shards, M, lists, lens, (Qb, Kb, Vb), Oc, lse = _run(keys, q, pos, world, k=256, layout=layout)
    nb = 8 * 64
    assert np.array_equal(M[:nb].cpu().numpy(), oc.members)
    for r in range(1, world):
        assert np.array_equal(lists[r], lists[0]) and np.array_equal(lens[r], lens[0])
    ol, on = O.index(q, pos, oc, k=256)
    PT.assert_lists_match(lists[0], lens[0], ol, on, q, pos, oc, k=256)
    Oref, lse_ref = O.attention(Qb, Kb, Vb, lists[0], lens[0])
    PT.assert_attention_close(Oc, Oref, lse, lse_ref)


def test_shards_ragged_tail_heads_and_decode():
    """A tail past the last block on the last rank, 2 index heads, and
    decode-sized batches (the small-batch scoring path on every rank)."""
    T = 4096 + 300
    keys = I.index_keys(1, T, 32)
    oc = O.build_cache(keys)
    pos = np.array([600, 2000, 4095, 4096, 4200, T - 1] + list(range(900, T, 97)), np.int64)
    q = I.index_queries_heads(6, keys, pos, 2)
    _, _, lists, lens, (Qb, Kb, Vb), Oc, lse = _run(keys, q, pos, 3, k=200, heads=2, layout="zigzag")
    ol, on = O.index_heads(q, pos, oc, k=200)
    PT.assert_lists_match(lists[0], lens[0], ol, on, q, pos, oc, k=200)
    Oref, lse_ref = O.attention(Qb, Kb, Vb, lists[0], lens[0])
    PT.assert_attention_close(Oc, Oref, lse, lse_ref)
    for nq in (1, 4):
        dpos = pos[-nq:]
        dq = I.index_queries(7, keys, dpos)
        _, _, dl, dn, _, _, _ = _run(keys, dq, dpos, 2, k=200)
        ol, on = O.index(dq, dpos, oc, k=200)
        PT.assert_lists_match(dl[0], dn[0], ol, on, dq, dpos, oc, k=200)
