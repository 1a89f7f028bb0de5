"""Multi-process plumbing on CPU (gloo, world size 2, 127.0.0.1): the bench's
max-over-ranks timing and barriers, a torchrun launch of the reference arm
(rank 0 alone works and prints one JSON line), and the context-parallel
step's exchanges (which rank's tensor lands where; the GPU stages are stood
in for by CPU ones that record what they receive)."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench

    w, r, _ = bench.init_dist()
    assert (w, r) == (world, rank)
    bench.barrier(w)
    out[rank] = bench.max_over_ranks(10.0 + rank, w)  # each rank's "time"; the slowest decides
    bench.barrier(w)
    torch.distributed.destroy_process_group()


def test_max_over_ranks_and_barrier_gloo():
    world, port = 2, _free_port()
    out = mp.get_context("spawn").Manager().dict()  # no fork of a threaded process
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    assert dict(out) == {0: 11.0, 1: 11.0}


@pytest.mark.timeout(600)
def test_reference_arm_under_torchrun_two_ranks():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2", "--master-addr",
           "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"), "--impl", "reference",
           "--workload", "tiny_flat_4k", "--queries", "256", "--steps", "1", "--warmup", "0", "--gpus", "2"]
    env = dict(os.environ, OMP_NUM_THREADS="2", CUDA_VISIBLE_DEVICES="")
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=540, env=env, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout[-2000:]  # rank 0 only
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0


# ---------------------------------------------------------------- context parallelism

def test_shard_ranges_cover_every_block_once():
    from hierarchical_key_clustering_b200.context_parallel import shard_range

    for T, world in [(4096, 2), (4096, 3), (4096, 5), (4396, 3), (10_000_000, 8), (512, 4), (100, 2)]:
        nblk = T // 512
        rs = [shard_range(T, r, world) for r in range(world)]
        blocks = [b for b0, b1, _, _, _ in rs for b in range(b0, b1)]
        assert blocks == list(range(nblk))
        toks = [(t0, t1) for _, _, t0, t1, _ in rs]
        assert toks[0][0] == 0 and toks[-1][1] == T
        assert all(toks[i][1] == toks[i + 1][0] for i in range(world - 1))
        per = rs[0][4]
        for r, (b0, b1, t0, t1, _) in enumerate(rs):
            assert b1 == b0 or b0 == r * per  # a rank's table slice sits at rank x slice size
            assert t0 == 512 * b0


@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_zigzag_chunks_cover_every_block_once_and_balance(world):
    """Zig-zag: 2 x world chunks, rank r holds chunks r and 2 world - 1 - r;
    together they cover every block once, the tail goes with the last chunk,
    chunk_order lists each chunk's (rank, part), and for a causal prefill of
    the last positions every rank's share of the listed positions (each
    query reads all blocks before it: an early block is read by more
    queries) is close to the mean."""
    from hierarchical_key_clustering_b200 import context_parallel as CP

    for T in (4096, 4396, 1 << 20, 10_000_000):
        nblk = T // 512
        C = CP.n_chunks(world, "zigzag")
        blocks, toks = [], []
        for r in range(world):
            for c in CP.rank_chunks(r, world, "zigzag"):
                b0, b1, t0, t1, _ = CP.chunk_range(T, c, C)
                blocks += list(range(b0, b1))
                toks.append((c, t0, t1))
        assert sorted(blocks) == list(range(nblk))
        toks.sort()
        assert toks[0][1] == 0 and toks[-1][2] == T
        assert all(toks[i][2] == toks[i + 1][1] for i in range(len(toks) - 1))
        order = CP.chunk_order(world, "zigzag")
        assert [CP.rank_chunks(r, world, "zigzag")[i] for r, i in order] == list(range(C))
    # attention work per rank of a causal prefill of every position of a 1M context: keys before each query
    T = 1 << 20
    for layout, bound in (("zigzag", 1.3), ("contiguous", None)):
        C = CP.n_chunks(world, layout)
        work = []
        for r in range(world):
            w = 0
            for c in CP.rank_chunks(r, world, layout):
                _, _, t0, t1, _ = CP.chunk_range(T, c, C)
                # sum over queries p of |[t0, t1) n [0, p]| = sum_{t in [t0, t1)} (T - t)
                w += (t1 - t0) * T - (t1 * (t1 - 1) - t0 * (t0 - 1)) // 2
            work.append(w)
        mean = sum(work) / world
        if bound is not None:
            assert max(work) <= bound * mean, (layout, world, max(work) / mean)


class _FakeShard:
    """A rank's stages with CPU stand-ins that record their inputs."""

    def __init__(self, rank, world):
        self.rank, self.world, self.seen = rank, world, {}

    def build(self, keys_local):
        return (torch.full((2, 16), self.rank, dtype=torch.int32), torch.full((2,), 10 + self.rank, dtype=torch.int32))

    def set_members(self, M, C):
        self.seen["members"], self.seen["count"] = M.clone(), C.clone()

    def index_local(self, qidx, pos):
        return torch.tensor([self.rank, 100 + self.rank, 200 + self.rank], dtype=torch.uint8)

    def index_merge(self, X, pos):
        self.seen["xchg"] = X.clone()
        return X.to(torch.int32).reshape(1, -1), torch.tensor([X.numel()], dtype=torch.int32)

    def attend_local(self, Q, K, V, lists, lens):
        return torch.full((1, 2, 4), float(self.rank)), torch.full((1, 2), -float(self.rank))

    def combine(self, O_parts, lse_parts):
        self.seen["O_parts"], self.seen["lse_parts"] = O_parts.clone(), lse_parts.clone()
        return O_parts.sum(0), lse_parts.max(0).values


def _cp_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    from hierarchical_key_clustering_b200 import context_parallel as CP

    dist.init_process_group("gloo", rank=rank, world_size=world)
    sh = _FakeShard(rank, world)
    O, lse, lists, lens = CP.prefill(sh, None, None, None, None, None, None)
    out[rank] = dict(members=sh.seen["members"][:, 0, 0].tolist(), count=sh.seen["count"][:, 0].tolist(),
                     xchg=sh.seen["xchg"].tolist(), O=O[0, 0, 0].item(), lse=lse[0, 0].item(),
                     lists=lists.tolist(), parts=sh.seen["O_parts"][:, 0, 0, 0].tolist())
    dist.destroy_process_group()


def test_context_parallel_exchanges_gloo():
    """Every rank receives every rank's member slice, exchange block and
    attention part, in rank order, and computes the same list."""
    world, port = 2, _free_port()
    out = mp.get_context("spawn").Manager().dict()  # no fork of a threaded process
    mp.spawn(_cp_worker, args=(world, port, out), nprocs=world, join=True)
    for r in range(world):
        d = out[r]
        assert d["members"] == [0, 1] and d["count"] == [10, 11]
        assert d["xchg"] == [0, 100, 200, 1, 101, 201]
        assert d["parts"] == [0.0, 1.0] and d["O"] == 1.0 and d["lse"] == 0.0
        assert d["lists"] == out[0]["lists"]
