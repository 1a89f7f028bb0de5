"""Failure detection on the GPU without a GPU fault: a bounded device-side
wait that runs out sets an error word the host reads, and the context stays
usable.  The library's test hook makes every tensor-core score CTA skip its
query-tile copy, so the barrier that waits for it never completes; waits are
cut to a short limit for that call.  Batches of more than 16 queries take the
tensor-core path (17: the bucket range split over many CTAs)."""
import numpy as np
import pytest
import torch

import oracle as O
from hierarchical_key_clustering_b200 import inputs as I
from hierarchical_key_clustering_b200 import lsa

from . import parity as PT

pytestmark = pytest.mark.gpu


def _index(cache, p, q, pos):
    nq = len(pos)
    lists = torch.full((nq, lsa.lsa_list_budget(p)), -7, dtype=torch.int32, device="cuda")
    lens = torch.zeros((nq,), dtype=torch.int32, device="cuda")
    ws = lsa.workspace(lsa.lsa_index_workspace_bytes(nq, cache.n_blocks, p))
    lsa.lsa_index_prefill(PT.to_dev(q), PT.to_dev(pos), cache, None, lists, lens, p, ws)
    torch.cuda.synchronize()
    return lists.cpu().numpy(), lens.cpu().numpy()


@pytest.mark.parametrize("nq", [17, 200])
def test_wait_that_runs_out_is_reported_and_context_survives(nq):
    assert torch.cuda.is_available()
    T = 4096
    keys = I.index_keys(0, T, 32)
    pos = np.linspace(600, T - 1, nq).astype(np.int64)
    q = I.index_queries(0, keys, pos)
    p = lsa.lsa_default_params(k=256)
    cache = lsa.Cache(T)
    lsa.lsa_build_cache(PT.to_dev(keys), 0, T, cache, p)
    assert lsa.lsa_check_device_errors() == 0
    lsa.lsa_debug_wait_test(True)
    try:
        _index(cache, p, q, pos)
        assert lsa.lsa_check_device_errors() == 1
        assert "wait ran out" in lsa.lib().lsa_last_error_string().decode()
    finally:
        lsa.lsa_debug_wait_test(False)
    # the word was cleared; the next call is normal and correct
    gl, gn = _index(cache, p, q, pos)
    assert lsa.lsa_check_device_errors() == 0
    oc = O.build_cache(keys)
    ol, on = O.index(q, pos, oc, k=256)
    PT.assert_lists_match(gl, gn, ol, on, q, pos, oc, k=256)
