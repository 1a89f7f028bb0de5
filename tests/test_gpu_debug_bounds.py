"""The debug build of the library (liblsa_debug.so: every gather index the
kernels read from memory and every list length checked on the device, a
failed check reported through lsa_check_device_errors() and the access
skipped, never a trap).  It runs in a child process, since a process loads
one build of the library: the tiny workload (Flat and Tree prefill, decode
batches, attention with near-set tiles and with a split list) must match the
oracle with a clean error word, and three broken indices -- a list entry past
the keys, member positions past the cache, a tree child past its level --
must each be caught with its own code, the context staying usable."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_debug_build_tiny_workload_and_caught_indices():
    env = dict(os.environ, LSA_BOUNDS_CHECKS="1")
    r = subprocess.run([sys.executable, "-m", "tests.debug_bounds_run"], cwd=ROOT, env=env, capture_output=True,
                       text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    out = json.loads(r.stdout.strip().splitlines()[-1])
    assert out["library"] == "liblsa_debug.so"
    assert out["clean_word"] == 0
    assert out["list_word"] == 2
    assert out["member_word"] == 4
    assert out["node_word"] == 8
    assert out["after_word"] == 0
