"""The C-ABI library builds, loads and exports every entry point that
include/lsa.h declares; host-only queries and argument checks behave as the
header says.  CPU only: no call here launches a kernel."""
import ctypes as C
import math
import os
import re

import pytest

from hierarchical_key_clustering_b200 import build, lsa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lsa.h")

FAKE = C.c_void_p(1 << 20)  # 256-aligned, never dereferenced by the calls below


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(lsa_\w+)\s*\(", text)))


def test_library_builds_and_exports_header_symbols():
    path = build.build()
    assert os.path.exists(path)
    raw = C.CDLL(path)
    names = header_functions()
    assert len(names) >= 15
    for n in names:
        assert hasattr(raw, n), f"{n} declared in lsa.h but not exported"
    assert set(names) == set(lsa.EXPORTS)


def test_default_params_and_budgets():
    p = lsa.lsa_default_params()
    assert (p.n_pool, p.block, p.n_buckets, p.cap_items, p.sink, p.window, p.k, p.beam, p.mode, p.index_heads) == \
        (4, 512, 64, 4, 4, 512, 4096, 32, 0, 1)
    assert lsa.lsa_list_budget(p) == 4096 + 4 + 512 + 1
    assert lsa.lsa_top_buckets(p) == 1153
    assert lsa.lsa_top_buckets(lsa.lsa_default_params(k=2048)) == 641
    assert lsa.lsa_top_buckets(lsa.lsa_default_params(k=256)) == 193


def test_cache_bytes_scoring_part_is_24_5_per_token():
    """Scoring-time cache (bf16 centroids, 16 member slots, count) = 24.5 B/token;
    the build-time arrays (pooled keys, fp32 centroids, item ids) come on top."""
    T = 1 << 20
    total = lsa.lib().lsa_cache_bytes(T)
    nb = T // 512 * 64
    scoring = nb * (64 * 2 + 16 * 4 + 4)
    build_only = T // 4 * 64 * 4 + nb * 64 * 4 + T // 512 * 128
    assert scoring / T == 24.5
    assert total >= scoring + build_only
    assert total - (scoring + build_only) < 6 * 256


def test_tree_layout_levels():
    for nblk in (1, 8, 256, 2048, 19531):
        t = lsa.lsa_tree()
        nbytes = lsa.lib().lsa_tree_bytes(nblk)
        assert lsa.lib().lsa_tree_bind(FAKE, nbytes, nblk, C.byref(t)) == 0
        nb = nblk * 64
        assert t.n_levels == math.ceil(math.log2(nb)) + 1
        sizes = [t.level_size[i] for i in range(t.n_levels)]
        assert sizes[0] == nb and sizes[-1] == 1
        assert all(sizes[i + 1] == (sizes[i] + 1) // 2 for i in range(len(sizes) - 1))
        assert t.level_offset[t.n_levels] == sum(sizes)
        assert t.cap_blocks == nblk and t.n_blocks == 0
    assert lsa.lib().lsa_tree_bytes(2048) > 0


def test_update_tree_argument_errors():
    """Host-side checks of lsa_update_tree (no GPU work is reached)."""
    L = lsa.lib()
    p = lsa.lsa_default_params(mode="tree")
    cache, tree = lsa.lsa_cache(), lsa.lsa_tree()
    _expect(L.lsa_cache_bind(FAKE, L.lsa_cache_bytes(8192), 8192, C.byref(cache)), 0)
    _expect(L.lsa_tree_bind(FAKE, L.lsa_tree_bytes(8), 8, C.byref(tree)), 0)
    _expect(L.lsa_update_tree(None, C.byref(tree), C.byref(p), None), -1)
    cache.n_blocks = 0
    _expect(L.lsa_update_tree(C.byref(cache), C.byref(tree), C.byref(p), None), -2)  # no complete block
    cache.n_blocks = 16
    _expect(L.lsa_update_tree(C.byref(cache), C.byref(tree), C.byref(p), None), -2)  # more than the tree holds
    cache.n_blocks, tree.n_blocks = 3, 5
    _expect(L.lsa_update_tree(C.byref(cache), C.byref(tree), C.byref(p), None), -2)  # cache behind the tree
    cache.n_blocks = 5
    _expect(L.lsa_update_tree(C.byref(cache), C.byref(tree), C.byref(p), None), 0)  # nothing new: no work
    unbound = lsa.lsa_tree()
    cache.n_blocks = 2
    _expect(L.lsa_update_tree(C.byref(cache), C.byref(unbound), C.byref(p), None), -1)


def _expect(code, want):
    assert code == want, lsa.lib().lsa_last_error_string().decode()


def test_argument_errors_return_codes():
    L = lsa.lib()
    p = lsa.lsa_default_params()
    cache = lsa.lsa_cache()
    nbytes = L.lsa_cache_bytes(4096)
    _expect(L.lsa_cache_bind(FAKE, nbytes, 4096, C.byref(cache)), 0)
    _expect(L.lsa_cache_bind(FAKE, nbytes - 1, 4096, C.byref(cache)), -2)
    _expect(L.lsa_cache_bind(C.c_void_p(1 << 20 | 16), nbytes, 4096, C.byref(cache)), -1)
    # params checks
    _expect(L.lsa_build_cache(FAKE, 0, 4096, C.byref(cache), None, None), -1)
    bad = lsa.lsa_default_params(n_pool=8)
    _expect(L.lsa_build_cache(FAKE, 0, 4096, C.byref(cache), C.byref(bad), None), -1)
    _expect(L.lsa_build_cache(FAKE, 0, 5000, C.byref(cache), C.byref(p), None), -2)
    _expect(L.lsa_build_cache(FAKE, 100, 50, C.byref(cache), C.byref(p), None), -2)
    _expect(L.lsa_build_cache(C.c_void_p(1 << 20 | 4), 0, 4096, C.byref(cache), C.byref(p), None), -1)
    # index: workspace and list budget checks
    cache.n_blocks = 8
    Lmax = L.lsa_list_budget(C.byref(p))
    _expect(L.lsa_index_prefill(FAKE, FAKE, 10, C.byref(cache), None, FAKE, FAKE, Lmax, C.byref(p), None, 0,
                                None), -5)
    _expect(L.lsa_index_prefill(FAKE, FAKE, 10, C.byref(cache), None, FAKE, FAKE, Lmax - 1, C.byref(p), FAKE,
                                1 << 40, None), -2)
    tp = lsa.lsa_default_params(mode="tree")
    _expect(L.lsa_index_prefill(FAKE, FAKE, 10, C.byref(cache), None, FAKE, FAKE, Lmax, C.byref(tp), FAKE,
                                1 << 40, None), -1)
    # index heads: 1..16, Flat only
    for bad_heads in (lsa.lsa_default_params(index_heads=0), lsa.lsa_default_params(index_heads=17),
                      lsa.lsa_default_params(index_heads=2, mode="tree")):
        _expect(L.lsa_index_prefill(FAKE, FAKE, 10, C.byref(cache), None, FAKE, FAKE, Lmax, C.byref(bad_heads),
                                    FAKE, 1 << 40, None), -1)
    # nq = 0 is a no-op
    _expect(L.lsa_index_prefill(None, None, 0, C.byref(cache), None, None, None, Lmax, C.byref(p), None, 0,
                                None), 0)
    # the static-scratch decode checks its parameters before sizing the request,
    # with the same code as lsa_index_decode (NULL pointers: nothing can launch)
    for bad_p in (lsa.lsa_default_params(index_heads=64), lsa.lsa_default_params(k=1 << 21),
                  lsa.lsa_default_params(n_pool=8), lsa.lsa_default_params(mode="tree", beam=0)):
        want = L.lsa_index_decode(None, None, 1, C.byref(cache), None, None, None, Lmax, C.byref(bad_p), None, 0,
                                  None)
        assert want == -1
        _expect(L.lsa_index_decode_static(None, None, 1, C.byref(cache), None, None, None, Lmax, C.byref(bad_p),
                                          None), -1)
    _expect(L.lsa_index_decode_static(None, None, 1, C.byref(cache), None, None, None, Lmax, None, None), -1)
    # attention shape checks
    _expect(L.lsa_sparse_attention(FAKE, FAKE, FAKE, 4, 32, 8, 64, 100, FAKE, FAKE, 10, 0.1, FAKE, None, None, 0,
                                   None), -1)
    _expect(L.lsa_sparse_attention(FAKE, FAKE, FAKE, 4, 30, 8, 128, 100, FAKE, FAKE, 10, 0.1, FAKE, None, None, 0,
                                   None), -1)
    _expect(L.lsa_sparse_attention(FAKE, FAKE, FAKE, 4, 64, 2, 128, 100, FAKE, FAKE, 10, 0.1, FAKE, None, None, 0,
                                   None), -1)
    _expect(L.lsa_sparse_attention(FAKE, FAKE, FAKE, 0, 32, 8, 128, 100, FAKE, FAKE, 10, 0.1, FAKE, None, None, 0,
                                   None), 0)
    assert "head_dim" in L.lsa_last_error_string().decode() or True


def test_workspace_queries():
    p = lsa.lsa_default_params(k=2048)
    a = lsa.lsa_index_workspace_bytes(1000, 256, p)
    b = lsa.lsa_index_workspace_bytes(2000, 256, p)
    assert 0 < a < b
    # many queries: no key split; one fp32 near-set partial per (query, head)
    # plus a (sink, window) plan per query and a record per tile, each array
    # 256-byte aligned
    near = lambda nq, hq: sum(-(-x // 256) * 256 for x in (nq * hq * 128 * 4, nq * hq * 2 * 4, nq * 8, nq * 16))
    assert lsa.lsa_attention_workspace_bytes(131072, 32, 128, 2565) == near(131072, 32)
    assert lsa.lsa_attention_workspace_bytes(1, 32, 128, 4613) > 0        # decode: split the list
    # position-range phases (no GPU here: L2 taken as 126 MiB, ranges of 129024 positions): at 1M keys, 9
    # ranges and 4613-entry lists (>= 256 per range) add the range bounds and one fp32 running result per
    # (query, head); at 10M keys (78 ranges) the lists are too short per range and nothing is added
    a256 = lambda x: -(-x // 256) * 256  # noqa: E731
    phase = a256(32768 * 10 * 4) + a256(32768 * 32 * 128 * 4) + a256(32768 * 32 * 2 * 4)
    assert lsa.lsa_attention_workspace_bytes(32768, 32, 128, 4613, 1 << 20) == max(phase, near(32768, 32))
    assert lsa.lsa_attention_workspace_bytes(65536, 32, 128, 4613, 10_000_000) == near(65536, 32)
    assert lsa.lsa_attention_workspace_bytes(32768, 32, 128, 4613, 0) == near(32768, 32)
    assert lsa.lsa_attention_workspace_bytes(32768, 32, 128, 4613, -1) == -1
    # index heads: the per-row arrays scale with heads, plus one merged set per query
    p4 = lsa.lsa_default_params(k=2048, index_heads=4)
    assert lsa.lsa_index_workspace_bytes(1000, 256, p4) > lsa.lsa_index_workspace_bytes(4000, 256, p)
    assert lsa.lsa_attention_workspace_bytes(1, 32, 64, 4613) == -1


@pytest.mark.parametrize("name", ["lsa_build_cache", "lsa_index_decode", "lsa_sparse_attention"])
def test_binding_raises_on_error(name):
    with pytest.raises(lsa.LsaError):
        if name == "lsa_build_cache":
            lsa._check(lsa.lib().lsa_build_cache(None, 0, 1, None, None, None))
        elif name == "lsa_index_decode":
            lsa._check(lsa.lib().lsa_index_decode(None, None, 1, None, None, None, None, 0, None, None, 0, None))
        else:
            lsa._check(lsa.lib().lsa_sparse_attention(None, None, None, 1, 0, 0, 128, 1, None, None, 1, 1.0, None,
                                                      None, None, 0, None))


def test_shard_sizes_and_argument_errors():
    """Context-parallel calls: slot count and exchange-block size as the
    header states them, and the argument checks (no kernel is launched)."""
    L = lsa.lib()
    p = lsa.lsa_default_params(k=2048)
    P = lsa.lsa_top_buckets(p)
    slots = lsa.lsa_shard_slots(p)
    assert slots == min(2 ** math.ceil(math.log2(2 * P)), 2 ** math.ceil(math.log2((3 * P + 1) // 2)))
    assert lsa.lsa_shard_exchange_bytes(1000, p) == 4096 + 1000 * slots * 8
    assert lsa.lsa_shard_exchange_bytes(1000, p) % 256 == 0
    assert lsa.lsa_shard_local_workspace_bytes(1000, 32, p) > lsa.lsa_index_workspace_bytes(1000, 32, p)
    assert lsa.lsa_shard_merge_workspace_bytes(1000, p) > 1000 * slots * 20
    cache = lsa.lsa_cache()
    _expect(L.lsa_cache_bind(FAKE, L.lsa_cache_bytes(4096), 4096, C.byref(cache)), 0)
    cache.n_blocks = 8
    big = 1 << 40
    Lmax = L.lsa_list_budget(C.byref(p))
    # local step: Tree mode, NULL exchange block, unaligned block, negative first block
    tp = lsa.lsa_default_params(k=2048, mode="tree")
    _expect(L.lsa_index_shard_local(FAKE, FAKE, 10, C.byref(cache), 0, FAKE, C.byref(tp), FAKE, big, None), -1)
    _expect(L.lsa_index_shard_local(FAKE, FAKE, 10, C.byref(cache), 0, None, C.byref(p), FAKE, big, None), -1)
    _expect(L.lsa_index_shard_local(FAKE, FAKE, 10, C.byref(cache), 0, C.c_void_p((1 << 20) + 16), C.byref(p),
                                    FAKE, big, None), -1)
    _expect(L.lsa_index_shard_local(FAKE, FAKE, 10, C.byref(cache), -1, FAKE, C.byref(p), FAKE, big, None), -2)
    _expect(L.lsa_index_shard_local(FAKE, FAKE, 10, C.byref(cache), 0, FAKE, C.byref(p), None, 0, None), -5)
    # merge: rank count, Tree mode, list budget, workspace
    for n_shards in (0, 33):
        _expect(L.lsa_index_shard_merge(FAKE, n_shards, FAKE, 10, FAKE, FAKE, 8, FAKE, FAKE, Lmax, C.byref(p), FAKE,
                                        big, None), -1)
    _expect(L.lsa_index_shard_merge(FAKE, 2, FAKE, 10, FAKE, FAKE, 8, FAKE, FAKE, Lmax, C.byref(tp), FAKE, big,
                                    None), -1)
    _expect(L.lsa_index_shard_merge(FAKE, 2, FAKE, 10, FAKE, FAKE, 8, FAKE, FAKE, Lmax - 1, C.byref(p), FAKE, big,
                                    None), -2)
    _expect(L.lsa_index_shard_merge(FAKE, 2, FAKE, 10, FAKE, FAKE, 8, FAKE, FAKE, Lmax, C.byref(p), FAKE, 16, None),
            -5)
    _expect(L.lsa_index_shard_merge(FAKE, 2, FAKE, 10, C.c_void_p((1 << 20) + 4), FAKE, 8, FAKE, FAKE, Lmax,
                                    C.byref(p), FAKE, big, None), -1)  # member rows are read 16 bytes at a time
    _expect(L.lsa_index_shard_merge(FAKE, 2, FAKE, 0, FAKE, FAKE, 8, FAKE, FAKE, Lmax, C.byref(p), None, 0, None), 0)
    # local lists, member slices, combine
    _expect(L.lsa_shard_local_lists(FAKE, FAKE, 10, Lmax, 100, 50, FAKE, FAKE, None), -2)
    _expect(L.lsa_shard_local_lists(FAKE, FAKE, 10, Lmax, 0, 50, FAKE, FAKE, None), -1)  # output aliases input
    _expect(L.lsa_shard_publish_members(C.byref(cache), -1, FAKE, FAKE, None), -2)
    _expect(L.lsa_attention_combine(FAKE, FAKE, 2, 10, 32, 64, FAKE, None, None), -1)
    _expect(L.lsa_attention_combine(FAKE, FAKE, 0, 10, 32, 128, FAKE, None, None), -2)
    _expect(L.lsa_attention_combine(FAKE, FAKE, 2, 0, 32, 128, FAKE, None, None), 0)


@pytest.mark.parametrize("nq,chunks,hkv,T", [(131072, 16, 8, 131072), (32768, 16, 8, 1048576), (1000, 16, 8, 4096),
                                             (300, 5, 1, 4096), (128, 1, 8, 4096), (5000, 3, 2, 10000)])
def test_prefill_chunk_plan(nq, chunks, hkv, T):
    """Host plan of prefill_from_host: contiguous chunks covering every query,
    starting on multiples of 128; the last chunk quartered only when each
    quarter keeps 2048 (query, KV head) units; each chunk's K/V rows reach
    its largest position (ascending positions: non-decreasing)."""
    import torch

    from hierarchical_key_clustering_b200.layer import chunk_plan

    pos = torch.arange(T - nq, T, dtype=torch.int64)
    bounds, need = chunk_plan(pos, chunks, hkv, T)
    assert bounds[0][0] == 0 and bounds[-1][1] == nq
    assert all(a[1] == b[0] for a, b in zip(bounds, bounds[1:]))
    assert all(c0 % 128 == 0 and c1 > c0 for c0, c1 in bounds)
    step = -(-(-(-nq // chunks)) // 128) * 128
    main = [b for b in bounds if b[1] - b[0] == step]
    assert len(main) >= len(bounds) - 4
    tail = bounds[len(main):]
    if len(tail) > 1:  # quartered: each piece a multiple of 128 (but the last) with >= 2048 units
        assert all((c1 - c0) * hkv >= 2048 for c0, c1 in tail[:-1])
    assert need == [min(T, int(pos[c1 - 1]) + 1) for c0, c1 in bounds]
    assert all(a <= b for a, b in zip(need, need[1:]))


@pytest.mark.parametrize("T", [100, 512, 4096, 4396, 131072, 1 << 20, 10_000_000])
def test_key_chunks_cover_the_keys_at_block_boundaries(T):
    """The pieces prefill_from_host copies and builds the cache from: they
    cover 0..T in order, every cut on a 512-key block boundary (so a block is
    always clustered from one piece), at most 8 of them."""
    from hierarchical_key_clustering_b200.layer import key_chunks

    k = key_chunks(T)
    assert k[0][0] == 0 and k[-1][1] == T and len(k) <= 8
    assert all(a[1] == b[0] for a, b in zip(k, k[1:]))
    assert all(a % 512 == 0 and b > a for a, b in k)
