"""numpy front end of the C oracle (lsa_oracle.c).

TEST INFRASTRUCTURE ONLY (tests, smoke check, benchmark CPU baseline).
Argument marshalling only: every step of the method runs in lsa_oracle.c,
which cites the LSA pages passage by passage.

Parity status per function:
  pool_norm, build_cache (Ward), build_tree, qnorm, flat ranking, expand,
  attention: pinned by the tests in tests/test_oracle_pins.py.
  tree_rank: pinned against beam decisions worked out by hand on a
  hand-built 16-leaf tree (kept set and node count at every level, hidden
  subtrees included), the narrowest beam still filling k, recall rising
  with the beam, and a wide beam equal to Flat search.  The beam-size rule
  itself is a reading (the pages give no rule that maps a beam of 32 to k
  keys); the pins fix that the oracle carries the reading out exactly.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "lsa_oracle.c")
LIB = os.path.join(HERE, "liblsa_oracle.so")

DIM = 64
BLOCK = 512
N_POOL = 4
ITEMS = 128
N_BUCKETS = 64
CAP_ITEMS = 4
MAX_LEVELS = 64

_lib = None


def build(force: bool = False) -> str:
    """Compile lsa_oracle.c into liblsa_oracle.so (gcc, OpenMP, no FP contraction)."""
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        cmd = ["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fPIC", "-shared", "-std=gnu11",
               "-o", LIB + ".tmp", SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(LIB + ".tmp", LIB)
    return LIB


def lib():
    global _lib
    if _lib is None:
        build()
        L = C.CDLL(LIB)
        P = C.c_void_p
        i64, i32, f32 = C.c_int64, C.c_int, C.c_float
        sigs = {
            "orc_f32_to_bf16": (C.c_uint16, [f32]),
            "orc_bf16_to_f32": (f32, [C.c_uint16]),
            "orc_sumsq": (f32, [P]),
            "orc_sqdist": (f32, [P, P]),
            "orc_normalize": (None, [P, P]),
            "orc_pool_norm": (None, [P, i64, P]),
            "orc_ward": (i32, [P, i32, i32, i32, P, P, P, P]),
            "orc_build_cache": (i64, [P, i64, i32, i32, P, P, P, P, P, P]),
            "orc_pair_run": (None, [P, P, i32, P]),
            "orc_tree_levels": (i32, [i64, P, i32]),
            "orc_build_tree": (i32, [P, P, P, i64, i32, P, P, P, P, P, P, P, P, P, i32]),
            "orc_qnorm": (None, [P, i64, P]),
            "orc_score": (f32, [P, P]),
            "orc_flat_rank": (i64, [P, i64, i32, P, P, P]),
            "orc_tree_rank": (i64, [P, i64, P, P, P, P, P, i32, i32, i64, P, P, P]),
            "orc_expand": (i32, [P, i64, P, P, i64, i32, i32, i32, P, i32]),
            "orc_index_heads": (i32, [P, P, i64, i32, i64, i32, P, P, P, i32, i32, i32, P, P, i32]),
            "orc_index": (i32, [P, P, i64, i64, i32, P, P, P, i32, P, P, P, P, P, i32,
                                i32, i32, i32, i32, P, P, i32]),
            "orc_attention": (None, [P, P, P, i64, i32, i32, i32, P, P, i32, f32, P, P]),
        }
        for name, (res, args) in sigs.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(C.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def list_budget(k: int, sink: int = 4, window: int = 512) -> int:
    """Longest possible list: sink + window (incl. the query) + k."""
    return k + sink + window + 1


def top_p(k: int, sink: int = 4, window: int = 512) -> int:
    """Buckets that always suffice for k far keys: every bucket holds >= 4 keys
    and at most sink + window clustered keys are skipped as near."""
    return (k + sink + window + N_POOL - 1) // N_POOL


# ---- scalar helpers -------------------------------------------------------

def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    x = _c(x, np.float32).ravel()
    f = lib().orc_f32_to_bf16
    return np.array([f(float(v)) for v in x], dtype=np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def sumsq(x: np.ndarray) -> float:
    return lib().orc_sumsq(_p(_c(x, np.float32)))


def normalize(x: np.ndarray) -> np.ndarray:
    x = _c(x, np.float32)
    out = np.empty(DIM, np.float32)
    lib().orc_normalize(_p(x), _p(out))
    return out


# ---- build path -----------------------------------------------------------

def shrink(Vb: np.ndarray, Wb: np.ndarray) -> np.ndarray:
    """Step 1, "Shrink" (sotaaz blog, "The same steps in general", step 1;
    zhichai forum post, "Key points"): x_t = W v_t, the product of the bf16
    inputs in fp64 (each bf16 product is exact there; the sum of D terms
    carries a relative error below D 2^-53), rounded once to fp32.
    Vb [T, D], Wb [64, D] bf16 bits."""
    V = bf16_bits_to_f32(np.asarray(Vb, np.uint16)).astype(np.float64)
    W = bf16_bits_to_f32(np.asarray(Wb, np.uint16)).astype(np.float64)
    return (V @ W.T).astype(np.float32)


def pool_norm(keys: np.ndarray) -> np.ndarray:
    keys = _c(keys, np.float32)
    n_items = keys.shape[0] // N_POOL
    out = np.empty((n_items, DIM), np.float32)
    lib().orc_pool_norm(_p(keys), n_items, _p(out))
    return out


def ward(items: np.ndarray, cap: int = CAP_ITEMS, n_target: int = N_BUCKETS, trace: bool = False):
    """Ward clustering of m unit-weight items. Returns root[m] (and the merge trace)."""
    items = _c(items, np.float32)
    m = items.shape[0]
    root = np.empty(m, np.int32)
    ti = np.empty(m, np.int32)
    tj = np.empty(m, np.int32)
    td = np.empty(m, np.float32)
    nm = lib().orc_ward(_p(items), m, cap, n_target, _p(root), _p(ti), _p(tj), _p(td))
    if trace:
        return root, (ti[:nm].copy(), tj[:nm].copy(), td[:nm].copy())
    return root


class Cache:
    """Host copy of a bucket cache (same layout as the CUDA cache)."""

    def __init__(self, T: int):
        self.T = T
        self.n_items = T // N_POOL
        self.nblk = T // BLOCK
        nb = self.nblk * N_BUCKETS
        self.pooled = np.zeros((self.n_items, DIM), np.float32)
        self.item_bucket = np.zeros((self.nblk, ITEMS), np.uint8)
        self.members = np.full((nb, 16), -1, np.int32)
        self.count = np.zeros(nb, np.int32)
        self.centroid = np.zeros((nb, DIM), np.float32)
        self.centroid_bf16 = np.zeros((nb, DIM), np.uint16)


def build_cache(keys: np.ndarray, cap_items: int = CAP_ITEMS, n_buckets: int = N_BUCKETS) -> Cache:
    keys = _c(keys, np.float32)
    c = Cache(keys.shape[0])
    r = lib().orc_build_cache(_p(keys), c.T, cap_items, n_buckets, _p(c.pooled), _p(c.item_bucket),
                              _p(c.members), _p(c.count), _p(c.centroid), _p(c.centroid_bf16))
    if r < 0:
        raise RuntimeError("oracle Ward did not reach the bucket count")
    return c


def pair_run(mu: np.ndarray, w: np.ndarray) -> np.ndarray:
    """Greedy Ward pairing of one run of nodes; partner[i] or -1."""
    mu = _c(mu, np.float32)
    w = _c(w, np.int32)
    partner = np.empty(len(w), np.int32)
    lib().orc_pair_run(_p(mu), _p(w), len(w), _p(partner))
    return partner


def tree_level_sizes(nb: int) -> np.ndarray:
    sizes = np.zeros(MAX_LEVELS, np.int64)
    L = lib().orc_tree_levels(nb, _p(sizes), MAX_LEVELS)
    return sizes[:L].copy()


class Tree:
    """Host copy of the bucket tree: all levels, global node ids."""

    def __init__(self, nb: int):
        self.level_size = tree_level_sizes(nb)
        self.n_levels = len(self.level_size)
        self.level_offset = np.concatenate([[0], np.cumsum(self.level_size)]).astype(np.int64)
        n = int(self.level_offset[-1])
        self.n_nodes = n
        self.child = np.full((n, 2), -1, np.int32)
        self.parent = np.full(n, -1, np.int32)
        self.weight = np.zeros(n, np.int32)
        self.min_block = np.zeros(n, np.int32)
        self.max_block = np.zeros(n, np.int32)
        self.sum = np.zeros((n, DIM), np.float32)
        self.centroid = np.zeros((n, DIM), np.float32)
        self.centroid_bf16 = np.zeros((n, DIM), np.uint16)


def build_tree(cache: Cache, n_buckets: int = N_BUCKETS) -> Tree:
    t = Tree(cache.nblk * n_buckets)
    sizes = np.zeros(MAX_LEVELS, np.int64)
    L = lib().orc_build_tree(_p(cache.pooled), _p(cache.members), _p(cache.count), cache.nblk, n_buckets,
                             _p(t.child), _p(t.parent), _p(t.weight), _p(t.min_block), _p(t.max_block),
                             _p(t.sum), _p(t.centroid), _p(t.centroid_bf16), _p(sizes), MAX_LEVELS)
    assert L == t.n_levels
    return t


# ---- query path -----------------------------------------------------------

def qnorm(q: np.ndarray) -> np.ndarray:
    q = _c(q, np.float32).reshape(-1, DIM)
    out = np.empty(q.shape, np.uint16)
    lib().orc_qnorm(_p(q), q.shape[0], _p(out))
    return out


def score(qhat_bits: np.ndarray, cbf_bits: np.ndarray) -> float:
    return lib().orc_score(_p(_c(qhat_bits, np.uint16)), _p(_c(cbf_bits, np.uint16)))


def flat_rank(qhat_bits: np.ndarray, H: int, cache: Cache, n_buckets: int = N_BUCKETS):
    n = H * n_buckets
    ids = np.empty(max(n, 1), np.int32)
    sc = np.empty(max(n, 1), np.float32)
    got = lib().orc_flat_rank(_p(_c(qhat_bits, np.uint16)), H, n_buckets, _p(cache.centroid_bf16),
                              _p(ids), _p(sc))
    return ids[:got], sc[:got]


def tree_rank(qhat_bits: np.ndarray, H: int, tree: Tree, beam: int, P: int, trace: bool = False):
    """Ranked level-0 ids and scores; with trace=True also the number of
    nodes the beam kept at each level (index = level)."""
    nb = int(tree.level_size[0])
    ids = np.empty(max(nb, 1), np.int32)
    sc = np.empty(max(nb, 1), np.float32)
    kept = np.zeros(max(tree.n_levels, 1), np.int64)
    got = lib().orc_tree_rank(_p(_c(qhat_bits, np.uint16)), H, _p(tree.child), _p(tree.parent),
                              _p(tree.max_block), _p(tree.centroid_bf16), _p(tree.level_size),
                              tree.n_levels, beam, P, _p(ids), _p(sc), _p(kept))
    if trace:
        return ids[:got], sc[:got], kept[:tree.n_levels]
    return ids[:got], sc[:got]


def expand(ranked: np.ndarray, cache: Cache, p: int, k: int, sink: int = 4, window: int = 512):
    ranked = _c(ranked, np.int32)
    Lmax = list_budget(k, sink, window)
    out = np.empty(Lmax, np.int32)
    n = lib().orc_expand(_p(ranked), len(ranked), _p(cache.members), _p(cache.count), p, k, sink,
                         window, _p(out), Lmax)
    return out, n


def index(qidx: np.ndarray, pos: np.ndarray, cache: Cache, k: int, mode: str = "flat",
          tree: Tree | None = None, beam: int = 32, sink: int = 4, window: int = 512):
    """Lists [nq, Lmax] (ascending, -1 padded) and lens [nq] for every query."""
    qidx = _c(qidx, np.float32).reshape(-1, DIM)
    pos = _c(pos, np.int64)
    nq = qidx.shape[0]
    Lmax = list_budget(k, sink, window)
    lists = np.empty((nq, Lmax), np.int32)
    lens = np.empty(nq, np.int32)
    if mode == "flat":
        m, tc, tp, tmb, tcb, tls, tl = 0, None, None, None, None, None, 0
    else:
        assert tree is not None
        m, tc, tp, tmb, tcb, tls, tl = (1, tree.child, tree.parent, tree.max_block, tree.centroid_bf16,
                                        tree.level_size, tree.n_levels)
    nul = C.c_void_p(0)
    r = lib().orc_index(_p(qidx), _p(pos), nq, cache.nblk, N_BUCKETS, _p(cache.members), _p(cache.count),
                        _p(cache.centroid_bf16), m, _p(tc) if tc is not None else nul,
                        _p(tp) if tp is not None else nul, _p(tmb) if tmb is not None else nul,
                        _p(tcb) if tcb is not None else nul, _p(tls) if tls is not None else nul, tl,
                        k, sink, window, beam, _p(lists), _p(lens), Lmax)
    if r < 0:
        raise RuntimeError("oracle index failed")
    return lists, lens


def index_heads(qidx: np.ndarray, pos: np.ndarray, cache: Cache, k: int, sink: int = 4, window: int = 512):
    """Multi-head Flat search (zhichai forum post, "Key points": N-LSA picks
    buckets by the best score across heads): qidx [nq, n_heads, 64]; a
    bucket scores the largest of its per-head scores.  Lists and lens as
    index()."""
    qidx = _c(qidx, np.float32)
    assert qidx.ndim == 3 and qidx.shape[2] == DIM
    pos = _c(pos, np.int64)
    nq, nh = qidx.shape[0], qidx.shape[1]
    Lmax = list_budget(k, sink, window)
    lists = np.empty((nq, Lmax), np.int32)
    lens = np.empty(nq, np.int32)
    r = lib().orc_index_heads(_p(qidx), _p(pos), nq, nh, cache.nblk, N_BUCKETS, _p(cache.members), _p(cache.count),
                              _p(cache.centroid_bf16), k, sink, window, _p(lists), _p(lens), Lmax)
    if r < 0:
        raise RuntimeError("oracle index failed")
    return lists, lens


def attention(Qb: np.ndarray, Kb: np.ndarray, Vb: np.ndarray, lists: np.ndarray, lens: np.ndarray,
              scale: float | None = None):
    """O [nq,Hq,dh] fp32 and lse [nq,Hq] from bf16-bit inputs."""
    Qb, Kb, Vb = _c(Qb, np.uint16), _c(Kb, np.uint16), _c(Vb, np.uint16)
    lists, lens = _c(lists, np.int32), _c(lens, np.int32)
    nq, Hq, dh = Qb.shape
    Hkv = Kb.shape[1]
    if scale is None:
        scale = 1.0 / np.sqrt(dh)
    O = np.empty((nq, Hq, dh), np.float32)
    lse = np.empty((nq, Hq), np.float32)
    lib().orc_attention(_p(Qb), _p(Kb), _p(Vb), nq, Hq, Hkv, dh, _p(lists), _p(lens), lists.shape[1],
                        float(scale), _p(O), _p(lse))
    return O, lse
