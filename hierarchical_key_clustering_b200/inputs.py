"""Seeded synthetic inputs for the LSA indexer and its sparse attention.

This module only draws random numbers; it holds none of the method's
arithmetic (no normalising, pooling, clustering, scoring or attention).
Both the CUDA path and the CPU oracle read the arrays it returns, so the
two sides always see the same bits.

Workload shape (Latent Sparse Attention pages: "Card catalog = semantic
clustering" key points; the five-step description "The same steps in
general"; and the configs this library is measured on):

* index keys: 64-dim fp32.  Positions are split in runs of 8; each run
  picks one component of an M-component mixture whose centres are
  Gaussian draws scaled to unit length and shared by the whole context.
  A key is its run's centre plus sigma * N(0, I) per coordinate
  (sigma = 0.3), left unnormalised (normalising is step a1 of the path).
* index queries: the query at position p is a noisy copy (sigma = 0.3 per
  coordinate) of the key at a source position drawn uniformly from
  [0, p-1] (source 0 when p = 0).
* Q/K/V for the attention: N(0, 1) rounded to bf16.

Every tensor has its own PCG64 stream derived from (seed, stream id), so
a change in one size never shifts another tensor's values.
"""
from __future__ import annotations

import numpy as np

STREAM_CENTRES = 0
STREAM_COMPONENTS = 1
STREAM_KEY_NOISE = 2
STREAM_QUERY_SOURCE = 3
STREAM_QUERY_NOISE = 4
STREAM_Q = 5
STREAM_K = 6
STREAM_V = 7

DIM = 64
RUN = 8
SIGMA = 0.3


def rng(seed: int, stream: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, stream])))


def mixture_centres(seed: int, n_components: int) -> np.ndarray:
    """[M, 64] fp32 unit-length centres (Gaussian draw divided by its length)."""
    c = rng(seed, STREAM_CENTRES).standard_normal((n_components, DIM))
    c /= np.linalg.norm(c, axis=1, keepdims=True)
    return c.astype(np.float32)


def index_keys(seed: int, n_tokens: int, n_components: int, sigma: float = SIGMA) -> np.ndarray:
    """[n_tokens, 64] fp32 index keys from the run-of-8 mixture generator."""
    centres = mixture_centres(seed, n_components)
    n_runs = (n_tokens + RUN - 1) // RUN
    comp = rng(seed, STREAM_COMPONENTS).integers(0, n_components, size=n_runs)
    noise = rng(seed, STREAM_KEY_NOISE).standard_normal((n_tokens, DIM), dtype=np.float32)
    keys = np.repeat(centres[comp], RUN, axis=0)[:n_tokens]
    keys += np.float32(sigma) * noise
    return np.ascontiguousarray(keys, dtype=np.float32)


def query_sources(seed: int, positions: np.ndarray) -> np.ndarray:
    """Source position of each query: uniform on [0, p-1], 0 when p = 0."""
    positions = np.asarray(positions, dtype=np.int64)
    u = rng(seed, STREAM_QUERY_SOURCE).random(positions.shape[0])
    src = np.floor(u * positions).astype(np.int64)
    return np.minimum(src, np.maximum(positions - 1, 0))


def index_queries(seed: int, keys: np.ndarray, positions: np.ndarray, sigma: float = SIGMA) -> np.ndarray:
    """[nq, 64] fp32 index queries: noisy copies of random earlier keys."""
    src = query_sources(seed, positions)
    noise = rng(seed, STREAM_QUERY_NOISE).standard_normal((len(src), DIM), dtype=np.float32)
    q = keys[src] + np.float32(sigma) * noise
    return np.ascontiguousarray(q, dtype=np.float32)


def index_queries_heads(seed: int, keys: np.ndarray, positions: np.ndarray, heads: int) -> np.ndarray:
    """[nq, heads, 64] fp32 index queries for multi-head search: head 0 is
    index_queries(seed, ...); head h > 0 is half of it plus the query of
    another seed for a position spread over the keys, so the heads agree in
    part and differ in part."""
    positions = np.asarray(positions, np.int64)
    q0 = index_queries(seed, keys, positions)
    out = [q0]
    for h in range(1, heads):
        other = (positions * (h + 3) + h) % keys.shape[0]
        out.append((np.float32(0.5) * q0 + index_queries(seed + 17 * h, keys, other)).astype(np.float32))
    return np.ascontiguousarray(np.stack(out, axis=1))


def normal_bf16_bits(seed: int, stream: int, shape) -> np.ndarray:
    """N(0,1) values rounded to bf16 (round to nearest even), as uint16 bits."""
    x = rng(seed, stream).standard_normal(shape, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def qkv_bf16_bits(seed: int, nq: int, n_kv: int, hq: int, hkv: int, head_dim: int = 128):
    """Q [nq,hq,d], K and V [n_kv,hkv,d] as bf16 bit patterns (uint16)."""
    q = normal_bf16_bits(seed, STREAM_Q, (nq, hq, head_dim))
    k = normal_bf16_bits(seed, STREAM_K, (n_kv, hkv, head_dim))
    v = normal_bf16_bits(seed, STREAM_V, (n_kv, hkv, head_dim))
    return q, k, v


# The workloads the library is measured on (sizes only).
WORKLOADS = {
    "tiny_flat_4k": dict(T=4096, n_components=32, k=256, hq=8, hkv=1, mode="flat",
                         n_prefill=4096, n_decode=0),
    "flat_128k": dict(T=131072, n_components=1024, k=2048, hq=32, hkv=8, mode="flat",
                      n_prefill=131072, n_decode=0),
    "flat_1m": dict(T=1048576, n_components=4096, k=4096, hq=32, hkv=8, mode="flat",
                    n_prefill=32768, n_decode=64),
    "tree_1m": dict(T=1048576, n_components=4096, k=4096, hq=32, hkv=8, mode="tree", beam=32,
                    n_prefill=32768, n_decode=64),
    "flat_tree_10m": dict(T=10_000_000, n_components=16384, k=4096, hq=32, hkv=8, mode="both",
                          beam=32, n_prefill=65536, n_decode=128),
}
