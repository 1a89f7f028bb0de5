"""Host-side pieces of bench.py that feed its rooflines, checked on the CPU."""
import os
import sys

import numpy as np
import torch

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


def _near_far_brute(lst, n):
    """The run of consecutive positions ending the list (at most 1024) and the
    run 0, 1, .. starting it (at most 16, disjoint from the first)."""
    d = 0
    while d < min(n, 1024) and lst[n - 1 - d] == lst[n - 1] - d:
        d += 1
    s = 0
    while s < min(n - d, 16) and lst[s] == s:
        s += 1
    return s + d, n - s - d


def test_near_split_rows_matches_brute_force():
    rng = np.random.default_rng(3)
    lmax, nq = 2600, 300
    lists = np.full((nq, lmax), -1, np.int32)
    lens = np.zeros(nq, np.int32)
    for i in range(nq):
        p = int(rng.integers(0, 6000))
        window = list(range(max(0, p - rng.integers(0, 1200)), p + 1))
        sinks = list(range(min(int(rng.integers(0, 20)), max(0, window[0]))))
        lo = len(sinks)
        hi = window[0]
        far = sorted(set(rng.integers(lo, max(lo + 1, hi), size=int(rng.integers(0, 800))).tolist()) - set(sinks))
        far = [f for f in far if f < hi]
        row = sorted(set(sinks + far + window))[:lmax]
        lists[i, :len(row)] = row
        lens[i] = len(row)
    near, far = bench.near_split_rows(torch.from_numpy(lists), torch.from_numpy(lens), chunk=64)
    exp = [_near_far_brute(lists[i], int(lens[i])) for i in range(nq)]
    assert near == sum(e[0] for e in exp)
    assert far == sum(e[1] for e in exp)
    assert near + far == int(lens.sum())
