"""Context parallelism for one LSA layer: the token range split over ranks.

The pages' end-to-end runs split the KV cache by token range over 8 GPUs
(zhichai forum post, "Reported numbers"; sotaaz blog, "Why 72x in one layer
becomes 9x").  Rank s holds a contiguous run of complete 512-key blocks (the
last rank also the unclustered tail), their bucket cache and their K/V rows;
queries are replicated.  One step:

  1. each rank clusters its blocks and publishes its slice of the member
     table; the slices are all-gathered into the replicated global table;
  2. each rank finds, per query, a candidate set holding its own top P
     buckets; the sets are all-gathered and every rank computes the same
     global top P and the same list;
  3. each rank attends over the list entries it owns; the partial outputs
     and their log-sum-exps are all-gathered and combined.

`Shard` is one rank's state and its stages (every computation is a call
into the C ABI); `prefill` runs the stages with the all-gathers of a
torch.distributed process group in between.  With a `gather` callable of
its own a caller can run the stages of all ranks in one process.
"""
from __future__ import annotations

import torch

from . import lsa

BLOCK = 512


def shard_range(T: int, rank: int, world: int):
    """Blocks [b0, b1) and tokens [t0, t1) of `rank`: ceil(n_blocks / world)
    blocks per rank in rank order (the last ranks may hold fewer or none),
    the last rank also the tail past the last complete block."""
    nblk = T // BLOCK
    per = max(1, -(-nblk // world))
    b0 = min(rank * per, nblk)
    b1 = min(b0 + per, nblk)
    t0, t1 = b0 * BLOCK, b1 * BLOCK
    if rank == world - 1:
        t1 = T
    return b0, b1, t0, t1, per


class Shard:
    """One rank's part of a context-parallel Flat LSA layer over T tokens."""

    def __init__(self, rank: int, world: int, T: int, k: int = 4096, sink: int = 4, window: int = 512,
                 index_heads: int = 1, max_queries: int = 1, device="cuda"):
        self.rank, self.world, self.T = rank, world, T
        self.b0, self.b1, self.t0, self.t1, self.per = shard_range(T, rank, world)
        self.p = lsa.lsa_default_params(k=k, sink=sink, window=window, index_heads=index_heads)
        self.device = device
        self.cache = lsa.Cache(max(self.t1 - self.t0, 1), device)
        self.n_blocks = T // BLOCK
        self.Lmax = lsa.lsa_list_budget(self.p)
        self.max_queries = max_queries
        nb_slice = self.per * 64
        self.members_slice = torch.full((nb_slice, 16), -1, dtype=torch.int32, device=device)
        self.count_slice = torch.zeros((nb_slice,), dtype=torch.int32, device=device)
        self.members = None  # the replicated global table, after set_members
        self.count = None
        self.xchg = lsa.workspace(lsa.lsa_shard_exchange_bytes(max_queries, self.p), device)
        self.ws_local = lsa.workspace(lsa.lsa_shard_local_workspace_bytes(max_queries, self.b1 - self.b0, self.p),
                                      device)
        self.ws_merge = lsa.workspace(lsa.lsa_shard_merge_workspace_bytes(max_queries, self.p), device)
        self.lists = torch.empty((max_queries, self.Lmax), dtype=torch.int32, device=device)
        self.lens = torch.empty((max_queries,), dtype=torch.int32, device=device)
        self.local_lists = torch.empty_like(self.lists)
        self.local_lens = torch.empty_like(self.lens)

    # 1. cache and member table
    def build(self, keys_local: torch.Tensor, stream=None):
        """Cluster this rank's blocks (keys of positions t0 .. t1-1) and write
        its slice of the member table."""
        n = keys_local.shape[0]
        assert n == self.t1 - self.t0
        if n:
            lsa.lsa_build_cache(keys_local, 0, n, self.cache, self.p, stream)
        lsa.lsa_shard_publish_members(self.cache, self.b0, self.members_slice, self.count_slice, stream)
        return self.members_slice, self.count_slice

    def set_members(self, members_all: torch.Tensor, count_all: torch.Tensor):
        """The all-gathered slices, in rank order: the global table."""
        self.members = members_all.reshape(-1, 16)
        self.count = count_all.reshape(-1)

    # 2. index
    def index_local(self, qidx: torch.Tensor, pos: torch.Tensor, stream=None) -> torch.Tensor:
        nq = qidx.shape[0]
        assert nq <= self.max_queries
        nbytes = lsa.lsa_shard_exchange_bytes(nq, self.p)
        xchg = self.xchg[:nbytes]
        lsa.lsa_index_shard_local(qidx, pos, self.cache, self.b0, xchg, self.p, self.ws_local, stream)
        return xchg

    def index_merge(self, xchg_all: torch.Tensor, pos: torch.Tensor, stream=None):
        nq = pos.shape[0]
        lists, lens = self.lists[:nq], self.lens[:nq]
        lsa.lsa_index_shard_merge(xchg_all, self.world, pos, self.members, self.count, self.n_blocks, lists, lens,
                                  self.p, self.ws_merge, stream)
        return lists, lens

    # 3. attention
    def attend_local(self, Q: torch.Tensor, K_local: torch.Tensor, V_local: torch.Tensor, lists, lens,
                     ws=None, stream=None):
        """Attention over this rank's entries of every list: output
        normalised over them and their log-sum-exp (-inf for none)."""
        nq, Hq = Q.shape[0], Q.shape[1]
        if self.t1 == self.t0:  # a rank past the last block holds no keys
            return torch.zeros_like(Q), torch.full((nq, Hq), float("-inf"), dtype=torch.float32, device=Q.device)
        ll, ln = self.local_lists[:nq], self.local_lens[:nq]
        lsa.lsa_shard_local_lists(lists, lens, self.t0, self.t1, ll, ln, stream)
        O_part = torch.empty_like(Q)
        lse_part = torch.empty((nq, Hq), dtype=torch.float32, device=Q.device)
        if ws is None:
            ws = lsa.workspace(lsa.lsa_attention_workspace_bytes(nq, Hq, Q.shape[2], self.Lmax), Q.device)
        lsa.lsa_sparse_attention(Q, K_local, V_local, ll, ln, O_part, lse_part, ws=ws, stream=stream)
        return O_part, lse_part

    @staticmethod
    def combine(O_parts: torch.Tensor, lse_parts: torch.Tensor, stream=None):
        """O_parts [ranks, nq, Hq, 128], lse_parts [ranks, nq, Hq]."""
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


def prefill(shard: Shard, keys_local, qidx, pos, Q, K_local, V_local, group=None, gather=all_gather_cat):
    """One context-parallel step on this rank (every rank calls it with the
    same queries): build, index, attend.  Returns the combined output and
    log-sum-exp (identical on every rank) and the list of every query."""
    m, c = shard.build(keys_local)
    shard.set_members(gather(m, group), gather(c, group))
    x = shard.index_local(qidx, pos)
    lists, lens = shard.index_merge(gather(x, group).reshape(-1), pos)
    O_s, lse_s = shard.attend_local(Q, K_local, V_local, lists, lens)
    O, lse = shard.combine(gather(O_s, group), gather(lse_s, group))
    return O, lse, lists, lens
