"""One LSA attention layer on the GPU: bucket cache (+ tree), indexer and
sparse attention, with every buffer allocated once up front.

This is a convenience wrapper over the five C-ABI calls in lsa.py; it
computes nothing itself.
"""
from __future__ import annotations

import torch

from . import lsa


def chunk_plan(pos, chunks: int, n_kv_heads: int, tk: int):
    """Query chunks of prefill_from_host and the K/V rows each one needs.

    The queries are cut into `chunks` pieces rounded up to multiples of 128
    (so the near-set tiles of the attention do not change).  The last
    chunk's copy back is the only one nothing overlaps, so it is split into
    quarters (multiples of 128 queries) when each quarter still has the
    2048 (query, KV head) units that keep its attention on whole lists.
    A chunk's lists hold positions up to its largest query position, so it
    needs K/V rows [0, min(tk, max pos + 1)).  Returns ([(c0, c1)], [rows])."""
    nq = len(pos)
    step = -(-nq // max(1, chunks))
    step = -(-step // 128) * 128
    bounds = [(c0, min(nq, c0 + step)) for c0 in range(0, nq, step)]
    c0, c1 = bounds[-1]
    q4 = -(-((c1 - c0) // 4) // 128) * 128
    if len(bounds) > 1 and q4 >= 128 and q4 * n_kv_heads >= 2048:
        bounds = bounds[:-1] + [(a, min(c1, a + q4)) for a in range(c0, c1, q4)]
    need = [min(tk, int(pos[c0:c1].max()) + 1) for c0, c1 in bounds]
    return bounds, need


def key_chunks(T: int, pieces: int = 8):
    """[(a, b)] cutting positions 0..T into about `pieces` ranges at block
    (512-key) boundaries, the last one ending at T: building the cache range
    by range gives the same cache as one build (items and blocks are pooled
    and clustered on their own), so each range can be built as soon as its
    keys are on the device."""
    nblk = T // 512
    cuts = sorted({min(nblk, (nblk * i) // pieces) * 512 for i in range(1, pieces)} - {0})
    edges = [0] + [c for c in cuts if 0 < c < T] + [T]
    return [(a, b) for a, b in zip(edges, edges[1:]) if b > a]


class SparseLayer:
    def __init__(self, capacity: int, k: int = 4096, mode: str = "flat", beam: int = 32, sink: int = 4,
                 window: int = 512, max_queries: int = 1, Hq: int = 32, head_dim: int = 128,
                 cand_cap: int = 0, index_heads: int = 1, device="cuda"):
        self.p = lsa.lsa_default_params(k=k, mode=mode, beam=beam, sink=sink, window=window, cand_cap=cand_cap,
                                        index_heads=index_heads)
        self.mode = mode
        self.cache = lsa.Cache(capacity, device)
        self.tree = lsa.Tree(max(capacity // 512, 1), device) if mode == "tree" else None
        self.Lmax = lsa.lsa_list_budget(self.p)
        self.max_queries = max_queries
        self.Hq = Hq
        nblk = capacity // 512
        self.ws_index = lsa.workspace(lsa.lsa_index_workspace_bytes(max_queries, nblk, self.p), device)
        self.ws_attn = lsa.workspace(lsa.lsa_attention_workspace_bytes(max_queries, Hq, head_dim, self.Lmax,
                                                                       capacity), device)
        self.lists = torch.empty((max_queries, self.Lmax), dtype=torch.int32, device=device)
        self.lens = torch.empty((max_queries,), dtype=torch.int32, device=device)
        self._h2d = self._d2h = None  # copy streams of prefill_from_host
        self._dbuf, self._dbuf_key = None, None

    def build(self, keys: torch.Tensor, t_begin: int = 0, t_end: int | None = None, stream=None):
        t_end = keys.shape[0] if t_end is None else t_end
        lsa.lsa_build_cache(keys, t_begin, t_end, self.cache, self.p, stream)
        if self.tree is not None:
            lsa.lsa_build_tree(self.cache, self.tree, self.p, stream)

    def build_from_rows(self, V: torch.Tensor, W: torch.Tensor, t_begin: int = 0, t_end: int | None = None,
                        stream=None):
        """Build (or grow) the cache from model rows instead of index keys:
        each row of V (bf16 [T, D], e.g. a position's key over all KV heads)
        is projected by W (bf16 [64, D]) and pooled straight into the cache
        (one fused tensor-core kernel), then the completed blocks are
        clustered and the tree, if any, grown.  t_begin must be a multiple
        of 4."""
        t_end = V.shape[0] if t_end is None else t_end
        lsa.lsa_shrink(V, W, t_begin, t_end, cache=self.cache, stream=stream)
        lsa.lsa_build_cache(None, t_begin, t_end, self.cache, self.p, stream)
        if self.tree is not None and self.cache.n_blocks > 0:
            lsa.lsa_update_tree(self.cache, self.tree, self.p, stream)

    def append(self, keys: torch.Tensor, t_begin: int, t_end: int, stream=None):
        """Grow the cache with the index keys of positions t_begin..t_end-1
        (keys holds positions 0..t_end-1): items and blocks that complete are
        pooled and clustered, and the tree, if any, is extended in place."""
        lsa.lsa_build_cache(keys, t_begin, t_end, self.cache, self.p, stream)
        if self.tree is not None and self.cache.n_blocks > 0:
            lsa.lsa_update_tree(self.cache, self.tree, self.p, stream)

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

    def prefill_from_host(self, h_keys, h_qidx, h_pos, h_Q, h_K, h_V, h_O, lse=None, chunks: int | None = None,
                          kv_cache=None, kv_first: int = 0):
        """One prefill step whose inputs and output live in pinned host memory.

        Three streams overlap the transfers with the kernels.  The index
        keys go first, in whole-block pieces, and each piece is pooled and
        clustered as soon as it lands, while the index queries follow for the
        index.  Q then arrives in query
        chunks (multiples of 128 queries, so the near-set tiles of the
        attention do not change), each preceded by
        the K and V rows its queries can list (positions up to the chunk's
        largest query position; the rest of K and V follows the last chunk),
        and each chunk's attention starts when its rows are on the device;
        each chunk's O is copied back while the next chunks compute.  Every
        copy and kernel of the call is ordered after the work already queued
        on the current stream, and the current stream waits for the last copy
        back, so the call behaves as one stream-ordered step.  The results are
        those of build + index + attend on device copies of the inputs, up to
        the attention's summation order when a chunk holds so few (query, KV
        head) units that the attention splits lists over warps.

        chunks (None: automatic) -- 16, or 2 when the attention takes its keys
        in position ranges (long contexts, see lsa_sparse_attention): every
        range's rows are then reused by all queries of a call, so fewer and
        larger calls pay more than finer copy overlap.

        kv_cache=(K, V): device tensors [Tk, Hkv, 128] that already hold the
        K/V rows of positions < kv_first (the KV cache of the earlier
        context); h_K/h_V then hold only rows kv_first..Tk-1, which are copied
        into them before the attention that can read them.
        """
        nq = h_Q.shape[0]
        assert nq <= self.max_queries
        dev = self.lists.device
        cs = torch.cuda.current_stream(dev)
        if self._h2d is None:
            self._h2d, self._d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        hs = (h_keys, h_qidx, h_pos, h_Q, h_O) + (() if kv_cache is not None else (h_K, h_V))
        key = tuple((tuple(t.shape), t.dtype) for t in hs)
        if self._dbuf_key != key:
            self._dbuf = [torch.empty(t.shape, dtype=t.dtype, device=dev) for t in hs]
            self._dbuf_key = key
        d_keys, d_q, d_pos, d_Q, d_O = self._dbuf[:5]
        if kv_cache is not None:
            d_K, d_V = kv_cache
            assert d_K.shape[0] == kv_first + h_K.shape[0] and d_V.shape == d_K.shape
        else:
            d_K, d_V = self._dbuf[5:]
            kv_first = 0
        tk = d_K.shape[0]
        if chunks is None:
            hq = h_Q.shape[1]
            ranged = (lsa.lsa_attention_workspace_bytes(nq, hq, 128, self.Lmax, tk) >
                      lsa.lsa_attention_workspace_bytes(nq, hq, 128, self.Lmax, 0))
            chunks = 2 if ranged else 16
        bounds, need = chunk_plan(h_pos, chunks, h_K.shape[1], tk)
        kb = key_chunks(h_keys.shape[0])
        self._h2d.wait_stream(cs)
        with torch.cuda.stream(self._h2d):
            e_keys = []  # the keys in whole-block pieces: each piece is pooled and clustered once it lands
            for a, b in kb:
                d_keys[a:b].copy_(h_keys[a:b], non_blocking=True)
                e_keys.append(torch.cuda.Event())
                e_keys[-1].record()
            d_q.copy_(h_qidx, non_blocking=True)
            d_pos.copy_(h_pos, non_blocking=True)
            e_idx = torch.cuda.Event()
            e_idx.record()
            e_in, have = [], kv_first
            for (c0, c1), n in zip(bounds, need):
                if n > have:
                    d_K[have:n].copy_(h_K[have - kv_first:n - kv_first], non_blocking=True)
                    d_V[have:n].copy_(h_V[have - kv_first:n - kv_first], non_blocking=True)
                    have = n
                d_Q[c0:c1].copy_(h_Q[c0:c1], non_blocking=True)
                e_in.append(torch.cuda.Event())
                e_in[-1].record()
            if have < tk:
                d_K[have:].copy_(h_K[have - kv_first:], non_blocking=True)
                d_V[have:].copy_(h_V[have - kv_first:], non_blocking=True)
            e_all = torch.cuda.Event()
            e_all.record()
        for (a, b), ek in zip(kb, e_keys):
            cs.wait_event(ek)
            lsa.lsa_build_cache(d_keys, a, b, self.cache, self.p, cs)
        if self.tree is not None:
            lsa.lsa_build_tree(self.cache, self.tree, self.p, cs)
        cs.wait_event(e_idx)
        self.index(d_q, d_pos, stream=cs)
        e_o = []
        for (c0, c1), ei in zip(bounds, e_in):
            cs.wait_event(ei)
            lsa.lsa_sparse_attention(d_Q[c0:c1], d_K, d_V, self.lists[c0:c1], self.lens[c0:c1], d_O[c0:c1],
                                     None if lse is None else lse[c0:c1], ws=self.ws_attn, stream=cs)
            e_o.append(torch.cuda.Event())
            e_o[-1].record(cs)
        with torch.cuda.stream(self._d2h):
            for (c0, c1), eo in zip(bounds, e_o):
                self._d2h.wait_event(eo)
                h_O[c0:c1].copy_(d_O[c0:c1], non_blocking=True)
        cs.wait_stream(self._d2h)
        cs.wait_event(e_all)
        return h_O
