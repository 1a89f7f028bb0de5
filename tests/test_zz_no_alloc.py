"""lsa_index_decode_static: decode indexing with the library's own fixed
device scratch, for callers that cannot allocate device memory (an engine
that reserved all of it up front, a host that only holds pointers it was
given, a decode loop that must not stall on an allocation).

The call must give exactly what lsa_index_decode gives with a caller
workspace, on consecutive calls that share the one scratch array.  Kept in
the last-collected file so that a failure here leaves every other test run."""
import ctypes as C

import numpy as np
import pytest
import torch

from hierarchical_key_clustering_b200 import inputs as I
from hierarchical_key_clustering_b200 import lsa

pytestmark = pytest.mark.gpu


def _setup(k=256, mode="flat"):
    assert torch.cuda.is_available(), "needs a GPU"
    T = 4096
    keys_all = I.index_keys(2, T + 64, 32)
    p = lsa.lsa_default_params(k=k, mode=mode)
    cache = lsa.Cache(T)
    lsa.lsa_build_cache(torch.from_numpy(keys_all[:T]).cuda(), 0, T, cache, p)
    tree = None
    if mode == "tree":
        tree = lsa.Tree(T // 512)
        lsa.lsa_build_tree(cache, tree, p)
    return keys_all, cache, tree, p


def _both(keys_all, cache, tree, p, pos_np):
    q = torch.from_numpy(I.index_queries(3, keys_all, pos_np)).cuda()
    pos = torch.from_numpy(pos_np).cuda()
    nq = len(pos_np)
    Lmax = lsa.lsa_list_budget(p)
    la = torch.full((nq, Lmax), -7, dtype=torch.int32, device="cuda")
    na = torch.full((nq,), -7, dtype=torch.int32, device="cuda")
    lb, nb = la.clone(), na.clone()
    ws = lsa.workspace(lsa.lsa_index_workspace_bytes(nq, cache.n_blocks, p))
    lsa.lsa_index_decode(q, pos, cache, tree, la, na, p, ws)
    lsa.lsa_index_decode_static(q, pos, cache, tree, lb, nb, p)
    torch.cuda.synchronize()
    return la.cpu().numpy(), na.cpu().numpy(), lb.cpu().numpy(), nb.cpu().numpy()


@pytest.mark.parametrize("mode", ["flat", "tree"])
def test_static_scratch_matches_workspace_entry_point(mode):
    keys_all, cache, tree, p = _setup(mode=mode)
    # two calls in a row with different query sets: the second must not see
    # anything the first left in the shared scratch
    for pos_np in (np.arange(4096, 4100, dtype=np.int64),
                   np.array([4096, 4111, 4159, 700, 2047, 3333, 5], dtype=np.int64)):
        la, na, lb, nb = _both(keys_all, cache, tree, p, pos_np)
        assert np.array_equal(na, nb)
        assert np.array_equal(la, lb)
        assert np.all(na > 0)


def test_static_scratch_call_allocates_nothing_after_set_up():
    """Once a first call has set a device up (module loading under CUDA's lazy
    loading, the array's address), calls take no device memory: the driver's
    free-memory count is the same before and after two calls."""
    keys_all, cache, tree, p = _setup()
    pos_np = np.array([4096, 4100, 1500], dtype=np.int64)
    q = torch.from_numpy(I.index_queries(3, keys_all, pos_np)).cuda()
    pos = torch.from_numpy(pos_np).cuda()
    Lmax = lsa.lsa_list_budget(p)
    lists = torch.empty((3, Lmax), dtype=torch.int32, device="cuda")
    lens = torch.empty((3,), dtype=torch.int32, device="cuda")
    # a call with no queries sets up the array and launches nothing
    lsa.lsa_index_decode_static(q[:0], pos[:0], cache, tree, lists[:0], lens[:0], p)
    lsa.lsa_index_decode_static(q, pos, cache, tree, lists, lens, p)  # first call with work: loads the kernels
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(2):
        lsa.lsa_index_decode_static(q, pos, cache, tree, lists, lens, p)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0
    assert np.all(lens.cpu().numpy() > 0)


def test_static_scratch_rejects_requests_above_its_size():
    """A request above the array's size is refused before anything is enqueued.
    The pointers are NULL: whichever check runs first, no kernel can start."""
    keys_all, cache, tree, p = _setup()
    nq = 100000
    need = lsa.lsa_index_workspace_bytes(nq, cache.n_blocks, p)
    assert need > lsa.STATIC_SCRATCH_BYTES
    Lmax = lsa.lsa_list_budget(p)
    rc = lsa.lib().lsa_index_decode_static(None, None, nq, C.byref(cache.c), None, None, None, Lmax, C.byref(p),
                                           None)
    assert rc == -5
    msg = lsa.lib().lsa_last_error_string().decode()
    assert "static scratch" in msg and str(need) in msg
