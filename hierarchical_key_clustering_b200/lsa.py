"""Python binding of liblsa.so (include/lsa.h): argument marshalling only.

Every step of the method runs in the CUDA kernels behind the C ABI; this
module only turns torch tensors into device pointers, carries the POD structs
and raises on a non-zero status.  There is no CPU fallback: if the library is
missing or a call fails, it raises.

The functions keep the C names (lsa_build_cache, lsa_build_tree,
lsa_index_prefill, lsa_index_decode, lsa_sparse_attention, ...).  Cache and
Tree own one torch byte buffer each, bound with lsa_cache_bind /
lsa_tree_bind, and expose torch views of the arrays for inspection.
"""
from __future__ import annotations

import ctypes as C
import os

import torch

from . import build as _build

MAX_LEVELS = 40
DIM = 64
HEAD_DIM = 128

LSA_OK = 0
LSA_MODE_FLAT = 0
LSA_MODE_TREE = 1
ERRORS = {-1: "LSA_ERR_ARG", -2: "LSA_ERR_SHAPE", -3: "LSA_ERR_CUDA", -4: "LSA_ERR_TIMEOUT",
          -5: "LSA_ERR_WORKSPACE"}


class LsaError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{ERRORS.get(code, code)}: {msg}")
        self.code = code


class lsa_params(C.Structure):
    _fields_ = [(n, C.c_int32) for n in
                ("n_pool", "block", "n_buckets", "cap_items", "sink", "window", "k", "beam", "mode", "cand_cap",
                 "index_heads")]


class lsa_cache(C.Structure):
    _fields_ = [("capacity", C.c_int64), ("n_blocks", C.c_int64), ("pooled", C.c_void_p),
                ("item_bucket", C.c_void_p), ("members", C.c_void_p), ("count", C.c_void_p),
                ("centroid", C.c_void_p), ("centroid_bf16", C.c_void_p)]


class lsa_tree(C.Structure):
    _fields_ = [("n_blocks", C.c_int64), ("n_levels", C.c_int32), ("cap_blocks", C.c_int32),
                ("level_size", C.c_int64 * MAX_LEVELS), ("level_offset", C.c_int64 * (MAX_LEVELS + 1)),
                ("child", C.c_void_p), ("parent", C.c_void_p), ("weight", C.c_void_p),
                ("min_block", C.c_void_p), ("max_block", C.c_void_p), ("sum", C.c_void_p),
                ("centroid", C.c_void_p), ("centroid_bf16", C.c_void_p)]


EXPORTS = ["lsa_default_params", "lsa_last_error_string", "lsa_launch_count", "lsa_check_device_errors",
           "lsa_debug_wait_test", "lsa_debug_attention_ranges", "lsa_debug_score_sample", "lsa_kernel_timing", "lsa_kernel_timing_read", "lsa_list_budget", "lsa_top_buckets",
           "lsa_cache_bytes", "lsa_cache_bind", "lsa_tree_bytes", "lsa_tree_bind",
           "lsa_index_workspace_bytes", "lsa_attention_workspace_bytes", "lsa_build_cache",
           "lsa_shrink", "lsa_build_tree", "lsa_update_tree", "lsa_index_prefill", "lsa_index_decode", "lsa_sparse_attention",
           "lsa_index_decode_static", "lsa_shard_slots", "lsa_shard_exchange_bytes",
           "lsa_shard_local_workspace_bytes", "lsa_shard_merge_workspace_bytes", "lsa_index_shard_local",
           "lsa_index_shard_merge", "lsa_shard_publish_members", "lsa_shard_local_lists", "lsa_attention_combine"]

_lib = None


def debug_build() -> bool:
    """LSA_BOUNDS_CHECKS=1 in the environment selects liblsa_debug.so, the
    build with the kernels' bounds checks compiled in."""
    return os.environ.get("LSA_BOUNDS_CHECKS", "0") not in ("", "0")


def library_path() -> str:
    return _build.LIB_DEBUG if debug_build() else _build.LIB


def lib():
    """Load liblsa.so, or liblsa_debug.so when debug_build() (building it if
    the sources are newer); raise if absent."""
    global _lib
    if _lib is None:
        path = library_path()
        if not os.path.exists(path) or _build._stale(path):
            try:
                _build.build(debug=debug_build())
            except Exception as e:  # no nvcc, no sources: there is no other path
                raise RuntimeError(f"{os.path.basename(path)} is missing and could not be built: {e}") from e
        L = C.CDLL(path)
        P, i64, i32, f32 = C.c_void_p, C.c_int64, C.c_int32, C.c_float
        pp, pc, pt = C.POINTER(lsa_params), C.POINTER(lsa_cache), C.POINTER(lsa_tree)
        sigs = {
            "lsa_default_params": (None, [pp]),
            "lsa_last_error_string": (C.c_char_p, []),
            "lsa_launch_count": (i64, []),
            "lsa_check_device_errors": (C.c_int, []),
            "lsa_debug_wait_test": (None, [i32]),
            "lsa_debug_attention_ranges": (None, [i64]),
            "lsa_debug_score_sample": (None, [i32, C.c_float]),
            "lsa_kernel_timing": (None, [i32]),
            "lsa_kernel_timing_read": (C.c_int, [C.c_char_p, i32, C.POINTER(C.c_double), C.POINTER(i64), i32]),
            "lsa_list_budget": (i32, [pp]),
            "lsa_top_buckets": (i32, [pp]),
            "lsa_cache_bytes": (i64, [i64]),
            "lsa_cache_bind": (C.c_int, [P, i64, i64, pc]),
            "lsa_tree_bytes": (i64, [i64]),
            "lsa_tree_bind": (C.c_int, [P, i64, i64, pt]),
            "lsa_index_workspace_bytes": (i64, [i64, i64, pp]),
            "lsa_attention_workspace_bytes": (i64, [i64, i32, i32, i32, i64]),
            "lsa_build_cache": (C.c_int, [P, i64, i64, pc, pp, P]),
            "lsa_shrink": (C.c_int, [P, i64, P, i64, i64, P, P, P]),
            "lsa_build_tree": (C.c_int, [pc, pt, pp, P]),
            "lsa_update_tree": (C.c_int, [pc, pt, pp, P]),
            "lsa_index_prefill": (C.c_int, [P, P, i64, pc, pt, P, P, i32, pp, P, i64, P]),
            "lsa_index_decode": (C.c_int, [P, P, i64, pc, pt, P, P, i32, pp, P, i64, P]),
            "lsa_index_decode_static": (C.c_int, [P, P, i64, pc, pt, P, P, i32, pp, P]),
            "lsa_sparse_attention": (C.c_int, [P, P, P, i64, i32, i32, i32, i64, P, P, i32, f32, P, P, P,
                                               i64, P]),
            "lsa_shard_slots": (i32, [pp]),
            "lsa_shard_exchange_bytes": (i64, [i64, pp]),
            "lsa_shard_local_workspace_bytes": (i64, [i64, i64, pp]),
            "lsa_shard_merge_workspace_bytes": (i64, [i64, pp]),
            "lsa_index_shard_local": (C.c_int, [P, P, i64, pc, i64, P, pp, P, i64, P]),
            "lsa_index_shard_merge": (C.c_int, [P, i32, P, i64, P, P, i64, P, P, i32, pp, P, i64, P]),
            "lsa_shard_publish_members": (C.c_int, [pc, i64, P, P, P]),
            "lsa_shard_local_lists": (C.c_int, [P, P, i64, i32, i64, i64, P, P, P]),
            "lsa_attention_combine": (C.c_int, [P, P, i32, i64, i32, i32, P, P, P]),
        }
        for name, (res, args) in sigs.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _check(code: int):
    if code != LSA_OK:
        raise LsaError(code, lib().lsa_last_error_string().decode())


def _ptr(t: torch.Tensor | None):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("device tensors only")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return C.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return C.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


# ---------------------------------------------------------------- params

def lsa_default_params(**overrides) -> lsa_params:
    p = lsa_params()
    lib().lsa_default_params(C.byref(p))
    for k, v in overrides.items():
        if v is not None:
            if isinstance(v, str) and k == "mode":
                v = {"flat": LSA_MODE_FLAT, "tree": LSA_MODE_TREE}[v]
            setattr(p, k, int(v))
    return p


def lsa_launch_count() -> int:
    return lib().lsa_launch_count()


def lsa_kernel_timing(enable: bool) -> None:
    """Bracket every kernel the library launches with CUDA events on its
    stream (profiling aid; not while a stream is being captured)."""
    lib().lsa_kernel_timing(1 if enable else 0)


def lsa_kernel_timing_read(max_kernels: int = 64) -> dict:
    """{kernel name: (milliseconds, launches)} summed since the last read, in
    first-launch order; waits for the recorded events."""
    name_len = 64
    names = C.create_string_buffer(name_len * max_kernels)
    ms = (C.c_double * max_kernels)()
    launches = (C.c_int64 * max_kernels)()
    n = lib().lsa_kernel_timing_read(names, name_len, ms, launches, max_kernels)
    _check(n if n < 0 else 0)
    out = {}
    for i in range(min(n, max_kernels)):
        nm = names.raw[i * name_len:(i + 1) * name_len].split(b"\0", 1)[0].decode()
        out[nm] = (ms[i], int(launches[i]))
    return out


def lsa_check_device_errors() -> int:
    """0 if no bounded device-side wait ran out since the last check (clears it)."""
    return lib().lsa_check_device_errors()


def lsa_debug_wait_test(enable: bool):
    lib().lsa_debug_wait_test(1 if enable else 0)


def lsa_debug_attention_ranges(range_rows: int):
    """Test hook: force the attention's position-range phases with ranges of
    range_rows positions (0: automatic)."""
    lib().lsa_debug_attention_ranges(int(range_rows))


def lsa_debug_score_sample(stride: int = 16, margin: float = 0.9):
    """Flat search's sampled threshold: every stride-th centroid tile, tau
    with about margin x P buckets above it (stride <= 1: exact histogram)."""
    lib().lsa_debug_score_sample(int(stride), float(margin))


def lsa_list_budget(p: lsa_params) -> int:
    return lib().lsa_list_budget(C.byref(p))


def lsa_top_buckets(p: lsa_params) -> int:
    return lib().lsa_top_buckets(C.byref(p))


def lsa_index_workspace_bytes(nq: int, n_blocks: int, p: lsa_params) -> int:
    return lib().lsa_index_workspace_bytes(nq, n_blocks, C.byref(p))


def lsa_attention_workspace_bytes(nq: int, Hq: int, head_dim: int, Lmax: int, Tk: int = 0) -> int:
    """Workspace of lsa_sparse_attention for nq queries over Tk keys (Tk = 0:
    without the position-range phases)."""
    return lib().lsa_attention_workspace_bytes(nq, Hq, head_dim, Lmax, Tk)


# ---------------------------------------------------------------- buffers

def _view(buf: torch.Tensor, base: int, ptr: int, dtype, shape):
    off = ptr - base
    n = 1
    for s in shape:
        n *= s
    nbytes = n * torch.empty((), dtype=dtype).element_size()
    return buf[off:off + nbytes].view(dtype).view(*shape)


class Cache:
    """Device bucket cache for `capacity` tokens in one torch buffer."""

    def __init__(self, capacity: int, device="cuda"):
        nbytes = lib().lsa_cache_bytes(capacity)
        self.buf = torch.empty(nbytes + 256, dtype=torch.uint8, device=device)
        base = self.buf.data_ptr()
        pad = (-base) % 256
        self._base = base + pad
        self.c = lsa_cache()
        _check(lib().lsa_cache_bind(C.c_void_p(self._base), nbytes, capacity, C.byref(self.c)))
        self.capacity = capacity

    @property
    def n_blocks(self) -> int:
        return self.c.n_blocks

    def views(self):
        nblk = self.capacity // 512
        nb = nblk * 64
        b, base = self.buf, self.buf.data_ptr()
        return dict(
            pooled=_view(b, base, self.c.pooled, torch.float32, (self.capacity // 4, DIM)),
            item_bucket=_view(b, base, self.c.item_bucket, torch.uint8, (nblk, 128)),
            members=_view(b, base, self.c.members, torch.int32, (nb, 16)),
            count=_view(b, base, self.c.count, torch.int32, (nb,)),
            centroid=_view(b, base, self.c.centroid, torch.float32, (nb, DIM)),
            centroid_bf16=_view(b, base, self.c.centroid_bf16, torch.int16, (nb, DIM)),
        )


class Tree:
    """Device tree of merged buckets over n_blocks blocks."""

    def __init__(self, n_blocks: int, device="cuda"):
        nbytes = lib().lsa_tree_bytes(n_blocks)
        self.buf = torch.empty(nbytes + 256, dtype=torch.uint8, device=device)
        base = self.buf.data_ptr()
        self._base = base + (-base) % 256
        self.t = lsa_tree()
        _check(lib().lsa_tree_bind(C.c_void_p(self._base), nbytes, n_blocks, C.byref(self.t)))

    @property
    def n_levels(self) -> int:
        return self.t.n_levels

    def level_sizes(self):
        return [self.t.level_size[i] for i in range(self.t.n_levels)]

    def views(self):
        n = self.t.level_offset[self.t.n_levels]
        b, base = self.buf, self.buf.data_ptr()
        return dict(
            child=_view(b, base, self.t.child, torch.int32, (n, 2)),
            parent=_view(b, base, self.t.parent, torch.int32, (n,)),
            weight=_view(b, base, self.t.weight, torch.int32, (n,)),
            min_block=_view(b, base, self.t.min_block, torch.int32, (n,)),
            max_block=_view(b, base, self.t.max_block, torch.int32, (n,)),
            sum=_view(b, base, self.t.sum, torch.float32, (n, DIM)),
            centroid=_view(b, base, self.t.centroid, torch.float32, (n, DIM)),
            centroid_bf16=_view(b, base, self.t.centroid_bf16, torch.int16, (n, DIM)),
        )


def workspace(nbytes: int, device="cuda") -> torch.Tensor:
    """A device byte buffer whose data pointer is 256-byte aligned."""
    return torch.empty(max(int(nbytes), 1), dtype=torch.uint8, device=device)


# ---------------------------------------------------------------- the five calls

def lsa_build_cache(keys: torch.Tensor, t_begin: int, t_end: int, cache: Cache, p: lsa_params, stream=None):
    _check(lib().lsa_build_cache(_ptr(keys), t_begin, t_end, C.byref(cache.c), C.byref(p), _stream(stream)))


def lsa_shrink(V: torch.Tensor, W: torch.Tensor, t_begin: int, t_end: int, keys=None, pooled=None, cache=None,
               stream=None):
    """x_t = W v_t for rows t_begin..t_end-1 of V (bf16 [T, D]) with W (bf16
    [64, D]); keys: fp32 [T, 64] output (optional); pooled: fp32 [T/4, 64]
    output, or the cache whose pooled items to write (optional)."""
    if V.dtype != torch.bfloat16 or W.dtype != torch.bfloat16:
        raise ValueError("V and W must be bfloat16")
    D = V.shape[1]
    if tuple(W.shape) != (64, D):
        raise ValueError(f"W must be [64, {D}]")
    pp_ = C.c_void_p(cache.c.pooled) if cache is not None else _ptr(pooled)
    _check(lib().lsa_shrink(_ptr(V), D, _ptr(W), t_begin, t_end, _ptr(keys), pp_, _stream(stream)))


def lsa_build_tree(cache: Cache, tree: Tree, p: lsa_params, stream=None):
    _check(lib().lsa_build_tree(C.byref(cache.c), C.byref(tree.t), C.byref(p), _stream(stream)))


def lsa_update_tree(cache: Cache, tree: Tree, p: lsa_params, stream=None):
    _check(lib().lsa_update_tree(C.byref(cache.c), C.byref(tree.t), C.byref(p), _stream(stream)))


def _index(fn, qidx, pos, cache, tree, lists, lens, p, ws, stream):
    nq = qidx.shape[0]
    assert qidx.numel() == nq * max(p.index_heads, 1) * 64, "qidx must be [nq, index_heads, 64]"
    Lmax = lists.shape[1] if lists.dim() == 2 else lsa_list_budget(p)
    _check(fn(_ptr(qidx), _ptr(pos), nq, C.byref(cache.c), C.byref(tree.t) if tree is not None else None,
              _ptr(lists), _ptr(lens), Lmax, C.byref(p), _ptr(ws), ws.numel() if ws is not None else 0,
              _stream(stream)))


def lsa_index_prefill(qidx, pos, cache: Cache, tree: Tree | None, lists, lens, p: lsa_params, ws, stream=None):
    _index(lib().lsa_index_prefill, qidx, pos, cache, tree, lists, lens, p, ws, stream)


def lsa_index_decode(qidx, pos, cache: Cache, tree: Tree | None, lists, lens, p: lsa_params, ws, stream=None):
    _index(lib().lsa_index_decode, qidx, pos, cache, tree, lists, lens, p, ws, stream)


def lsa_index_decode_static(qidx, pos, cache: Cache, tree: Tree | None, lists, lens, p: lsa_params, stream=None):
    """lsa_index_decode with the library's fixed device scratch (no workspace)."""
    _check(lib().lsa_index_decode_static(_ptr(qidx), _ptr(pos), qidx.shape[0], C.byref(cache.c),
                                         C.byref(tree.t) if tree is not None else None, _ptr(lists), _ptr(lens),
                                         lists.shape[1], C.byref(p), _stream(stream)))


def _static_scratch_bytes() -> int:
    """LSA_STATIC_SCRATCH_BYTES as include/lsa.h defines it (read from the
    header, so the binding keeps no second copy of the size)."""
    import re
    hdr = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "lsa.h")
    with open(hdr) as f:
        m = re.search(r"#define\s+LSA_STATIC_SCRATCH_BYTES\s+\((\d+)u\s*<<\s*(\d+)\)", f.read())
    if not m:
        raise RuntimeError("LSA_STATIC_SCRATCH_BYTES not found in include/lsa.h")
    return int(m.group(1)) << int(m.group(2))


STATIC_SCRATCH_BYTES = _static_scratch_bytes()


def lsa_sparse_attention(Q, K, V, lists, lens, O, lse=None, scale=None, ws=None, stream=None):
    nq, Hq, dh = Q.shape
    Tk, Hkv, _ = K.shape
    if scale is None:
        scale = dh ** -0.5
    _check(lib().lsa_sparse_attention(_ptr(Q), _ptr(K), _ptr(V), nq, Hq, Hkv, dh, Tk, _ptr(lists), _ptr(lens),
                                      lists.shape[1], float(scale), _ptr(O), _ptr(lse), _ptr(ws),
                                      ws.numel() if ws is not None else 0, _stream(stream)))


# ---------------------------------------------------------------- context parallelism

def lsa_shard_slots(p: lsa_params) -> int:
    return int(lib().lsa_shard_slots(C.byref(p)))


def lsa_shard_exchange_bytes(nq: int, p: lsa_params) -> int:
    return int(lib().lsa_shard_exchange_bytes(nq, C.byref(p)))


def lsa_shard_local_workspace_bytes(nq: int, n_blocks: int, p: lsa_params) -> int:
    return int(lib().lsa_shard_local_workspace_bytes(nq, n_blocks, C.byref(p)))


def lsa_shard_merge_workspace_bytes(nq: int, p: lsa_params) -> int:
    return int(lib().lsa_shard_merge_workspace_bytes(nq, C.byref(p)))


def lsa_index_shard_local(qidx, pos, cache: Cache, b_first: int, xchg, p: lsa_params, ws, stream=None):
    nq = qidx.shape[0]
    assert qidx.numel() == nq * max(p.index_heads, 1) * 64, "qidx must be [nq, index_heads, 64]"
    _check(lib().lsa_index_shard_local(_ptr(qidx), _ptr(pos), nq, C.byref(cache.c), b_first, _ptr(xchg), C.byref(p),
                                       _ptr(ws), ws.numel() if ws is not None else 0, _stream(stream)))


def lsa_index_shard_merge(xchg_all, n_shards: int, pos, members, count, n_blocks: int, lists, lens, p: lsa_params, ws,
                          stream=None):
    _check(lib().lsa_index_shard_merge(_ptr(xchg_all), n_shards, _ptr(pos), pos.shape[0], _ptr(members),
                                       _ptr(count), n_blocks, _ptr(lists), _ptr(lens), lists.shape[1], C.byref(p),
                                       _ptr(ws), ws.numel() if ws is not None else 0, _stream(stream)))


def lsa_shard_publish_members(cache: Cache, b_first: int, members_out, count_out, stream=None):
    _check(lib().lsa_shard_publish_members(C.byref(cache.c), b_first, _ptr(members_out), _ptr(count_out),
                                           _stream(stream)))


def lsa_shard_local_lists(lists, lens, t_begin: int, t_end: int, out_lists, out_lens, stream=None):
    _check(lib().lsa_shard_local_lists(_ptr(lists), _ptr(lens), lists.shape[0], lists.shape[1], t_begin, t_end,
                                       _ptr(out_lists), _ptr(out_lens), _stream(stream)))


def lsa_attention_combine(O_parts, lse_parts, O, lse=None, stream=None):
    n_parts, nq, Hq, D = O_parts.shape
    _check(lib().lsa_attention_combine(_ptr(O_parts), _ptr(lse_parts), n_parts, nq, Hq, D, _ptr(O), _ptr(lse),
                                       _stream(stream)))
