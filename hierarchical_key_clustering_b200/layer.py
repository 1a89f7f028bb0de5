"""One LSA attention layer on the GPU: bucket cache (+ tree), indexer and
sparse attention, with every buffer allocated once up front.

This is a convenience wrapper over the five C-ABI calls in lsa.py; it
computes nothing itself.
"""
from __future__ import annotations

import torch

from . import lsa


class SparseLayer:
    def __init__(self, capacity: int, k: int = 4096, mode: str = "flat", beam: int = 32, sink: int = 4,
                 window: int = 512, max_queries: int = 1, Hq: int = 32, head_dim: int = 128,
                 cand_cap: int = 0, device="cuda"):
        self.p = lsa.lsa_default_params(k=k, mode=mode, beam=beam, sink=sink, window=window, cand_cap=cand_cap)
        self.mode = mode
        self.cache = lsa.Cache(capacity, device)
        self.tree = lsa.Tree(max(capacity // 512, 1), device) if mode == "tree" else None
        self.Lmax = lsa.lsa_list_budget(self.p)
        self.max_queries = max_queries
        self.Hq = Hq
        nblk = capacity // 512
        self.ws_index = lsa.workspace(lsa.lsa_index_workspace_bytes(max_queries, nblk, self.p), device)
        self.ws_attn = lsa.workspace(lsa.lsa_attention_workspace_bytes(max_queries, Hq, head_dim, self.Lmax),
                                     device)
        self.lists = torch.empty((max_queries, self.Lmax), dtype=torch.int32, device=device)
        self.lens = torch.empty((max_queries,), dtype=torch.int32, device=device)

    def build(self, keys: torch.Tensor, t_begin: int = 0, t_end: int | None = None, stream=None):
        t_end = keys.shape[0] if t_end is None else t_end
        lsa.lsa_build_cache(keys, t_begin, t_end, self.cache, self.p, stream)
        if self.tree is not None:
            lsa.lsa_build_tree(self.cache, self.tree, self.p, stream)

    def index(self, qidx: torch.Tensor, pos: torch.Tensor, decode: bool = False, stream=None):
        nq = qidx.shape[0]
        assert nq <= self.max_queries
        fn = lsa.lsa_index_decode if decode else lsa.lsa_index_prefill
        fn(qidx, pos, self.cache, self.tree, self.lists[:nq], self.lens[:nq], self.p, self.ws_index, stream)
        return self.lists[:nq], self.lens[:nq]

    def attend(self, Q, K, V, O, lse=None, stream=None):
        nq = Q.shape[0]
        lsa.lsa_sparse_attention(Q, K, V, self.lists[:nq], self.lens[:nq], O, lse, ws=self.ws_attn,
                                 stream=stream)
        return O
