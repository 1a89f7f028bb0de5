"""Context parallelism for one LSA layer: the token range split over ranks.

The pages' end-to-end runs split the KV cache by token range over 8 GPUs
(zhichai forum post, "Reported numbers"; sotaaz blog, "Why 72x in one layer
becomes 9x").  The complete 512-key blocks are cut into chunks of
consecutive blocks and every rank holds one or more chunks -- their bucket
cache and their K/V rows (the rank holding the last chunk also the
unclustered tail); queries are replicated.  One step:

  1. each rank clusters its chunks and publishes their slices of the member
     table; the slices are all-gathered into the replicated global table;
  2. each rank finds, per query and chunk, a candidate set holding that
     chunk's top P buckets; the sets are all-gathered and every rank computes
     the same global top P and the same list;
  3. each rank attends over the list entries its chunks own; the partial
     outputs and their log-sum-exps are all-gathered and combined.

Layouts:
  * "contiguous": `world` chunks, rank r holds chunk r.  A causal prefill
    over the last positions lists far more of the early context (every
    query sees it) than of the late one, so the early ranks do most of the
    attention.
  * "zigzag": 2 x world chunks, rank r holds chunks r and 2 world - 1 - r,
    so every rank holds an early and a late stretch of the context and the
    ranks' attention work evens out.

`Shard` is one rank's state and its stages (every computation is a call
into the C ABI); `prefill` runs the stages with the all-gathers of a
torch.distributed process group in between.  With a `gather` callable of
its own a caller can run the stages of all ranks in one process.
"""
from __future__ import annotations

import torch

from . import lsa

BLOCK = 512
LAYOUTS = ("contiguous", "zigzag")


def n_chunks(world: int, layout: str = "contiguous") -> int:
    assert layout in LAYOUTS
    return world if layout == "contiguous" else 2 * world


def chunk_range(T: int, chunk: int, chunks: int):
    """Blocks [b0, b1) and tokens [t0, t1) of chunk `chunk` of `chunks`:
    ceil(n_blocks / chunks) blocks per chunk in order (the last chunks may
    hold fewer or none), the last chunk also the tail past the last complete
    block.  Returns (b0, b1, t0, t1, blocks per chunk)."""
    nblk = T // BLOCK
    per = max(1, -(-nblk // chunks))
    b0 = min(chunk * per, nblk)
    b1 = min(b0 + per, nblk)
    t0, t1 = b0 * BLOCK, b1 * BLOCK
    if chunk == chunks - 1:
        t1 = T
    return b0, b1, t0, t1, per


def rank_chunks(rank: int, world: int, layout: str = "contiguous"):
    """The chunks `rank` holds, in the order its exchange blocks list them."""
    if layout == "contiguous":
        return [rank]
    return [rank, 2 * world - 1 - rank]


def chunk_order(world: int, layout: str = "contiguous"):
    """For the all-gathered per-rank slices stacked as [rank][part]: the
    (rank, part) that holds each chunk, in chunk order."""
    where = {}
    for r in range(world):
        for i, c in enumerate(rank_chunks(r, world, layout)):
            where[c] = (r, i)
    return [where[c] for c in range(n_chunks(world, layout))]


def shard_range(T: int, rank: int, world: int):
    """The contiguous layout's range of `rank` (chunk_range of chunk `rank`
    of `world`)."""
    return chunk_range(T, rank, world)


class _Part:
    """One chunk held by a rank: its cache and buffers."""

    def __init__(self, T, chunk, chunks, p, max_queries, Lmax, device):
        self.chunk = chunk
        self.b0, self.b1, self.t0, self.t1, self.per = chunk_range(T, chunk, chunks)
        self.cache = lsa.Cache(max(self.t1 - self.t0, 1), device)
        nb_slice = self.per * 64
        self.members_slice = torch.full((nb_slice, 16), -1, dtype=torch.int32, device=device)
        self.count_slice = torch.zeros((nb_slice,), dtype=torch.int32, device=device)
        self.xchg = lsa.workspace(lsa.lsa_shard_exchange_bytes(max_queries, p), device)
        self.ws_local = lsa.workspace(lsa.lsa_shard_local_workspace_bytes(max_queries, self.b1 - self.b0, p), device)
        self.local_lists = torch.empty((max_queries, Lmax), dtype=torch.int32, device=device)
        self.local_lens = torch.empty((max_queries,), dtype=torch.int32, device=device)


class Shard:
    """One rank's part of a context-parallel Flat LSA layer over T tokens."""

    def __init__(self, rank: int, world: int, T: int, k: int = 4096, sink: int = 4, window: int = 512,
                 index_heads: int = 1, max_queries: int = 1, layout: str = "contiguous", device="cuda"):
        self.rank, self.world, self.T, self.layout = rank, world, T, layout
        self.chunks = n_chunks(world, layout)
        self.p = lsa.lsa_default_params(k=k, sink=sink, window=window, index_heads=index_heads)
        self.device = device
        self.n_blocks = T // BLOCK
        self.Lmax = lsa.lsa_list_budget(self.p)
        self.max_queries = max_queries
        self.parts = [_Part(T, c, self.chunks, self.p, max_queries, self.Lmax, device)
                      for c in rank_chunks(rank, world, layout)]
        self.members = None  # the replicated global table, after set_members
        self.count = None
        self.ws_merge = lsa.workspace(lsa.lsa_shard_merge_workspace_bytes(max_queries, self.p), device)
        self.lists = torch.empty((max_queries, self.Lmax), dtype=torch.int32, device=device)
        self.lens = torch.empty((max_queries,), dtype=torch.int32, device=device)

    @property
    def spans(self):
        """The token ranges [(t0, t1)] this rank holds."""
        return [(pt.t0, pt.t1) for pt in self.parts]

    # 1. cache and member table
    def build(self, keys: torch.Tensor, stream=None):
        """Cluster this rank's chunks (keys: every position's index key, or at
        least those of this rank's chunks at their absolute positions) and
        write their slices of the member table.  Returns the slices stacked
        [parts, slice, 16] and [parts, slice]."""
        for pt in self.parts:
            n = pt.t1 - pt.t0
            if n:
                lsa.lsa_build_cache(keys[pt.t0:pt.t1], 0, n, pt.cache, self.p, stream)
            lsa.lsa_shard_publish_members(pt.cache, pt.b0, pt.members_slice, pt.count_slice, stream)
        return (torch.stack([pt.members_slice for pt in self.parts]),
                torch.stack([pt.count_slice for pt in self.parts]))

    def set_members(self, members_all: torch.Tensor, count_all: torch.Tensor):
        """The all-gathered slices [rank, part, ...]: the global table, in
        chunk (block) order."""
        order = chunk_order(self.world, self.layout)
        self.members = torch.cat([members_all[r, i] for r, i in order]).reshape(-1, 16)
        self.count = torch.cat([count_all[r, i] for r, i in order]).reshape(-1)

    # 2. index
    def index_local(self, qidx: torch.Tensor, pos: torch.Tensor, stream=None) -> torch.Tensor:
        """This rank's exchange blocks, one per chunk, concatenated."""
        nq = qidx.shape[0]
        assert nq <= self.max_queries
        nbytes = lsa.lsa_shard_exchange_bytes(nq, self.p)
        out = []
        for pt in self.parts:
            xchg = pt.xchg[:nbytes]
            lsa.lsa_index_shard_local(qidx, pos, pt.cache, pt.b0, xchg, self.p, pt.ws_local, stream)
            out.append(xchg)
        return torch.cat(out) if len(out) > 1 else out[0]

    def index_merge(self, xchg_all: torch.Tensor, pos: torch.Tensor, stream=None):
        """The global top P of every query from all chunks' exchange blocks
        (in any order), expanded into the same lists on every rank."""
        nq = pos.shape[0]
        lists, lens = self.lists[:nq], self.lens[:nq]
        lsa.lsa_index_shard_merge(xchg_all, self.chunks, pos, self.members, self.count, self.n_blocks, lists, lens,
                                  self.p, self.ws_merge, stream)
        return lists, lens

    # 3. attention
    def attend_local(self, Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, lists, lens, ws=None, stream=None):
        """Attention over the entries of every list that this rank's chunks
        own (K, V: every position's rows, or at least those of this rank's
        chunks at their absolute positions): per chunk, the output normalised
        over them and their log-sum-exp (-inf for none), stacked
        [parts, nq, Hq, 128] and [parts, nq, Hq]."""
        nq, Hq = Q.shape[0], Q.shape[1]
        Os, ls = [], []
        for pt in self.parts:
            if pt.t1 == pt.t0:  # a chunk past the last block holds no keys
                Os.append(torch.zeros_like(Q))
                ls.append(torch.full((nq, Hq), float("-inf"), dtype=torch.float32, device=Q.device))
                continue
            ll, ln = pt.local_lists[:nq], pt.local_lens[:nq]
            lsa.lsa_shard_local_lists(lists, lens, pt.t0, pt.t1, ll, ln, stream)
            O_part = torch.empty_like(Q)
            lse_part = torch.empty((nq, Hq), dtype=torch.float32, device=Q.device)
            w = ws
            if w is None:
                w = lsa.workspace(lsa.lsa_attention_workspace_bytes(nq, Hq, Q.shape[2], self.Lmax, pt.t1 - pt.t0),
                                  Q.device)
            lsa.lsa_sparse_attention(Q, K[pt.t0:pt.t1], V[pt.t0:pt.t1], ll, ln, O_part, lse_part, ws=w,
                                     stream=stream)
            Os.append(O_part)
            ls.append(lse_part)
        return torch.stack(Os), torch.stack(ls)

    @staticmethod
    def combine(O_parts: torch.Tensor, lse_parts: torch.Tensor, stream=None):
        """O_parts [parts, nq, Hq, 128], lse_parts [parts, nq, Hq] (any
        leading shape: the parts of every rank)."""
        O_parts = O_parts.reshape(-1, *O_parts.shape[-3:])
        lse_parts = lse_parts.reshape(-1, *lse_parts.shape[-2:])
        O = torch.empty(O_parts.shape[1:], dtype=O_parts.dtype, device=O_parts.device)
        lse = torch.empty(lse_parts.shape[1:], dtype=torch.float32, device=lse_parts.device)
        lsa.lsa_attention_combine(O_parts, lse_parts, O, lse, stream)
        return O, lse


def all_gather_cat(t: torch.Tensor, group=None) -> torch.Tensor:
    """The ranks' tensors of equal shape, stacked in rank order."""
    import torch.distributed as dist

    world = dist.get_world_size(group)
    out = [torch.empty_like(t) for _ in range(world)]
    dist.all_gather(out, t.contiguous(), group=group)
    return torch.stack(out)


def prefill(shard: Shard, keys, qidx, pos, Q, K, V, group=None, gather=all_gather_cat):
    """One context-parallel step on this rank (every rank calls it with the
    same queries): build, index, attend.  keys, K and V hold (at least) the
    rows of this rank's chunks at their absolute positions.  Returns the
    combined output and log-sum-exp (identical on every rank) and the list
    of every query."""
    m, c = shard.build(keys)
    shard.set_members(gather(m, group), gather(c, group))
    x = shard.index_local(qidx, pos)
    lists, lens = shard.index_merge(gather(x, group).reshape(-1), pos)
    O_s, lse_s = shard.attend_local(Q, K, V, lists, lens)
    O, lse = shard.combine(gather(O_s, group), gather(lse_s, group))
    return O, lse, lists, lens
