"""Child process of tests/test_gpu_debug_bounds.py: the tiny workload through
the debug build of the library (liblsa_debug.so, every gather index and list
length checked on the device), against the oracle; then three inputs that
break an index on purpose, each of which the debug build's own checks catch
and skip.  Prints one JSON line of results.

Run as `LSA_BOUNDS_CHECKS=1 python -m tests.debug_bounds_run` from the
repository root."""
from __future__ import annotations

import json
import os

import numpy as np
import torch

import oracle as O
from hierarchical_key_clustering_b200 import inputs as I
from hierarchical_key_clustering_b200 import lsa

from . import parity as PT


def _index(cache, tree, p, q, pos, decode=False):
    nq = len(pos)
    lists = torch.full((nq, lsa.lsa_list_budget(p)), -7, dtype=torch.int32, device="cuda")
    lens = torch.zeros((nq,), dtype=torch.int32, device="cuda")
    ws = lsa.workspace(lsa.lsa_index_workspace_bytes(nq, cache.n_blocks, p))
    fn = lsa.lsa_index_decode if decode else lsa.lsa_index_prefill
    fn(PT.to_dev(q), PT.to_dev(pos), cache, tree, lists, lens, p, ws)
    torch.cuda.synchronize()
    return lists, lens


def main():
    assert lsa.debug_build() and lsa.library_path().endswith("liblsa_debug.so")
    out = {"library": os.path.basename(lsa.library_path())}
    T, k, hq, hkv, W = 4096, 256, 8, 1, 32
    keys_all = I.index_keys(0, T + 16, 32)
    keys = keys_all[:T]
    oc = O.build_cache(keys)
    ot = O.build_tree(oc)
    pf = lsa.lsa_default_params(k=k)
    pt = lsa.lsa_default_params(k=k, mode="tree", beam=W)
    cache = lsa.Cache(T)
    lsa.lsa_build_cache(PT.to_dev(keys), 0, T, cache, pf)
    tree = lsa.Tree(T // 512)
    lsa.lsa_build_tree(cache, tree, pt)
    torch.cuda.synchronize()
    PT.assert_cache_equal(PT.cache_to_numpy(cache, T), oc)

    # Flat prefill of every position, Tree prefill of a sample, decode batches
    pos = np.arange(T, dtype=np.int64)
    q = I.index_queries(0, keys, pos)
    fl, fn_ = _index(cache, None, pf, q, pos)
    ol, on = O.index(q, pos, oc, k=k)
    PT.assert_lists_match(fl.cpu().numpy(), fn_.cpu().numpy(), ol, on, q, pos, oc, k=k)
    sel = np.arange(0, T, 13)
    tl, tn = _index(cache, tree, pt, q[sel], pos[sel])
    otl, otn = O.index(q[sel], pos[sel], oc, k=k, mode="tree", tree=ot, beam=W)
    PT.assert_lists_match(tl.cpu().numpy(), tn.cpu().numpy(), otl, otn, q[sel], pos[sel], oc, k=k, tree=ot, beam=W)
    for nq in (1, 4):
        dpos = np.arange(T, T + nq, dtype=np.int64)
        dq = I.index_queries(1, keys_all, dpos)
        for prm, tr, mode in ((pf, None, "flat"), (pt, tree, "tree")):
            gl, gn = _index(cache, tr, prm, dq, dpos, decode=True)
            rl, rn = O.index(dq, dpos, oc, k=k, mode=mode, tree=ot if tr is not None else None, beam=W)
            PT.assert_lists_match(gl.cpu().numpy(), gn.cpu().numpy(), rl, rn, dq, dpos, oc, k=k,
                                  tree=ot if tr is not None else None, beam=W if tr is not None else None)

    # attention over the Flat lists (near-set tiles) and one split decode list
    Qb, Kb, Vb = I.qkv_bf16_bits(0, T, T, hq, hkv)
    f = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()  # noqa: E731
    Qd, Kd, Vd = f(Qb), f(Kb), f(Vb)
    Od = torch.empty_like(Qd)
    lse = torch.empty((T, hq), dtype=torch.float32, device="cuda")
    ws = lsa.workspace(lsa.lsa_attention_workspace_bytes(T, hq, 128, fl.shape[1]))
    lsa.lsa_sparse_attention(Qd, Kd, Vd, fl, fn_, Od, lse, ws=ws)
    torch.cuda.synchronize()
    a_sel = np.arange(0, T, 41)
    gl_np, gn_np = fl.cpu().numpy(), fn_.cpu().numpy()
    Oref, lref = O.attention(Qb[a_sel], Kb, Vb, gl_np[a_sel], gn_np[a_sel])
    out["attention_max_err"], out["attention_mean_err"] = PT.assert_attention_close(
        Od[torch.from_numpy(a_sel).cuda()], Oref, lse[torch.from_numpy(a_sel).cuda()], lref)
    one = torch.from_numpy(np.array([T - 1])).cuda()
    O1 = torch.empty((1, hq, 128), dtype=torch.bfloat16, device="cuda")
    ws1 = lsa.workspace(lsa.lsa_attention_workspace_bytes(1, hq, 128, fl.shape[1]))
    lsa.lsa_sparse_attention(Qd[one], Kd, Vd, fl[one], fn_[one], O1, ws=ws1)
    torch.cuda.synchronize()
    Oref1, _ = O.attention(Qb[T - 1:T], Kb, Vb, gl_np[T - 1:T], gn_np[T - 1:T])
    PT.assert_attention_close(O1, Oref1)
    out["clean_word"] = lsa.lsa_check_device_errors()

    # a list entry past the keys: caught by the attention's check (code 2)
    bad_l = torch.full((1, fl.shape[1]), -1, dtype=torch.int32, device="cuda")
    bad_l[0, :4] = torch.tensor([0, 1, 2, T + 5], dtype=torch.int32)
    bad_n = torch.tensor([4], dtype=torch.int32, device="cuda")
    lsa.lsa_sparse_attention(Qd[:1], Kd, Vd, bad_l, bad_n, O1, ws=ws1)
    torch.cuda.synchronize()
    out["list_word"] = lsa.lsa_check_device_errors()

    # member positions past the cache in block 3: caught by the expansion (code 4)
    mem = cache.views()["members"]
    saved = mem.clone()
    mem[3 * 64:4 * 64, 0] = 10 ** 8
    bpos = np.arange(T - 64, T, dtype=np.int64)
    _index(cache, None, pf, q[bpos], bpos)
    out["member_word"] = lsa.lsa_check_device_errors()
    mem.copy_(saved)

    # a child id past its level: caught by the tree search (code 8); a beam as
    # wide as every level keeps every visible node, so the search reaches it
    child = tree.views()["child"]
    saved_c = child.clone()
    lvl1 = int(tree.t.level_offset[1])
    child[lvl1 + 3, 1] = 10 ** 7
    pw = lsa.lsa_default_params(k=k, mode="tree", beam=int(T // 512 * 64))
    _index(cache, tree, pw, q[bpos], bpos)
    out["node_word"] = lsa.lsa_check_device_errors()
    child.copy_(saved_c)

    # the context is still usable and correct afterwards
    gl2, gn2 = _index(cache, None, pf, q[sel], pos[sel])
    PT.assert_lists_match(gl2.cpu().numpy(), gn2.cpu().numpy(), ol[sel], on[sel], q[sel], pos[sel], oc, k=k)
    out["after_word"] = lsa.lsa_check_device_errors()
    print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
