"""Benchmark of one LSA layer (indexer + sparse attention) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Workload (default): Flat LSA prefill at T = 131072 -- 64-dim index keys and
queries from the run-of-8 mixture generator (1024 components), k = 2048,
sink 4, window 512, attention with 32 query heads over 8 KV heads,
head_dim 128, bf16.  One step is the whole hot path over that batch:
bucket-cache build (normalise + pool + Ward for all 256 blocks), Flat index
of all 131072 queries, and sparse attention for all of them.
value = prefill tokens (queries) per second, whole job.

Also reported: decode us/token at T = 1,048,576 (index_decode + attention
for 64 new tokens, batch 1; for the 1M and 10M workloads, at their own T),
the roofline of the dominant kernel, the
oracle's CPU time on a bounded sample, and an end-to-end number through the
same C-ABI calls with inputs copied from pinned host memory every step and
the output copied back.

Multi-GPU: the layer does not shard here (each rank runs its own replica,
"replicas only"); value = all ranks' tokens / max-over-ranks time.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from hierarchical_key_clustering_b200 import inputs as I  # noqa: E402
from hierarchical_key_clustering_b200 import lsa  # noqa: E402
from hierarchical_key_clustering_b200.layer import SparseLayer  # noqa: E402

METRIC = "indexer+sparse-attn prefill tokens/s & decode us/token per layer; % roofline"
UNIT = "tokens/s"
L2_FLUSH_BYTES = 256 << 20
# DRAM bytes per far (query, KV head, key) row -- a list entry the gather
# kernel k_attn reads -- that ncu measured for the k_attn launch of each Flat
# workload (dram__bytes_read.sum + dram__bytes_write.sum of the full launch
# divided by the launch's far rows x Hkv):
#   flat_128k      20.21 GB + 1.08 GB over 131072 x 2048 x 8 far rows (the
#                  near-set tiles take sink and window; k_attn's reads include
#                  the tiles' partial results);
#   flat_1m        437.8 GB + 0.28 GB over 32768 x 4613 x 8 rows;
#   flat_tree_10m  1.09 TB + 0.55 GB over 65536 x 4613 x 8 rows (at 1M and
#                  10M a KV head does not fit in L2, the library keeps the
#                  near set in the gather, and every listed row is a far row).
# Re-measure when k_attn changes.
ATTN_DRAM_BYTES_PER_FAR_ROW = {"flat_128k": 9.92, "flat_1m": 362.3, "flat_tree_10m": 450.8}


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return dict(hbm=d["hbm_gbs"], bf16=d["bf16_tflops"], bf16_sust=d["bf16_tflops_sustained"], src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sust=1400.0, src="fallback")


class Clocks:
    """nvidia-smi sampling during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = f"/tmp/lsa_clocks_{os.getpid()}.csv"

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"], stdout=self.f,
                                         stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        med = float(np.median(sm)) if sm else None
        return {"sm_mhz": med, "sm_max_mhz": smax, "samples": len(sm), "reasons": sorted(reasons)}


def init_dist():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl" if torch.cuda.is_available() else "gloo",
                                             timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    dev = "cpu" if torch.distributed.get_backend() == "gloo" else "cuda"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


# --------------------------------------------------------------------------- workload

def make_prefill_inputs(wl: dict, seed: int = 0):
    T = wl["T"]
    keys = I.index_keys(seed, T, wl["n_components"])
    nq = wl["n_prefill"]
    pos = np.arange(T - nq, T, dtype=np.int64)
    q = I.index_queries(seed, keys, pos)
    return keys, q, pos


def device_qkv(nq, n_kv, hq, hkv, seed=0, dev="cuda"):
    g = torch.Generator(device=dev)
    g.manual_seed(seed * 1000 + 5)
    Q = torch.randn((nq, hq, 128), generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)
    K = torch.randn((n_kv, hkv, 128), generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)
    V = torch.randn((n_kv, hkv, 128), generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)
    return Q, K, V


def near_split_rows(lists: torch.Tensor, lens: torch.Tensor, chunk: int = 4096):
    """Per list, the rows the near-set tiles take -- the run of consecutive
    positions that ends the list (at most 1024) and the run 0, 1, .. that
    starts it (at most 16, disjoint from the first) -- as the attention's plan
    finds them for a tile of consecutive queries (the bench's queries are
    consecutive).  Returns (near rows, far rows) summed over the lists."""
    nq, lmax = lists.shape
    dev = lists.device
    ar_d = torch.arange(1024, device=dev)
    ar_s = torch.arange(min(16, lmax), device=dev)
    near = far = 0
    for c0 in range(0, nq, chunk):
        lst = lists[c0:c0 + chunk].long()
        n = lens[c0:c0 + chunk].long().clamp(max=lmax)
        tail = torch.gather(lst, 1, (n[:, None] - 1 - ar_d[None, :]).clamp(min=0))
        d = ((tail == tail[:, :1] - ar_d[None, :]) & (ar_d[None, :] < n[:, None])).int().cumprod(1).sum(1)
        head = lst[:, :len(ar_s)]
        s = ((head == ar_s[None, :]) & (ar_s[None, :] < (n - d)[:, None])).int().cumprod(1).sum(1)
        near += int((s + d).sum())
        far += int((n - s - d).sum())
    return near, far


def attn_algorithmic_bytes(far_rows: int, nq: int, hq: int, hkv: int) -> int:
    """Gather kernel k_attn: K and V rows of every far (query, KV head, key)
    + their list entries + Q read + O write + the near-set partial results
    (fp32 O and max/sum per (query, head)) it merges."""
    return far_rows * hkv * 2 * 256 + far_rows * 4 + nq * hq * 128 * 2 * 2 + nq * hq * 130 * 4


def measure_shrink(K: torch.Tensor, dev, hbm_peak: float):
    """Step 1 ("Shrink") on its own, outside the timed step: every position's
    key over all KV heads (D = Hkv x 128, the workload's K as [T, D]) projected
    by a synthetic bf16 W [64, D] and pooled straight into cache items (the
    fused tensor-core kernel); HBM-bound on reading K."""
    T = K.shape[0]
    V = K.reshape(T, -1)
    D = V.shape[1]
    g = torch.Generator(device=dev)
    g.manual_seed(64)
    W = (torch.randn((64, D), generator=g, device=dev) / D ** 0.5).to(torch.bfloat16)
    pooled = torch.empty((T // 4, 64), dtype=torch.float32, device=dev)
    ts = []
    for r in range(6):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        lsa.lsa_shrink(V, W, 0, T, pooled=pooled)
        e1.record()
        torch.cuda.synchronize()
        if r >= 2:
            ts.append(e0.elapsed_time(e1))
    ms = float(np.median(ts))
    nbytes = T * D * 2 + (T // 4) * 64 * 4 + 64 * D * 2
    gbs = nbytes / (ms / 1e3) / 1e9
    return {"kernel": "k_shrink", "T": T, "D": D, "ms": round(ms, 3), "bytes": nbytes,
            "achieved_gbs": round(gbs, 1), "frac": round(gbs / hbm_peak, 4), "bound": "hbm",
            "flop": 2 * T * D * 64}


def measure_index_heads(layer, keys_np, pos_np, wl: dict, dev, heads: int = 8, chunk: int = 16384):
    """Multi-head Flat search (a bucket ranks by its best score over `heads`
    index heads) for every prefill query of the workload, on the cache the
    timed step built, outside the timed step: queries [nq, heads, 64] from
    the seeded generator, indexed in chunks of `chunk` queries (the per-row
    candidate slots of chunk x heads rows), one event pair around all
    chunks."""
    nq = len(pos_np)
    chunk = min(chunk, nq)
    qh = torch.from_numpy(I.index_queries_heads(11, keys_np, pos_np, heads)).to(dev)
    pos = torch.from_numpy(pos_np).to(dev)
    p = lsa.lsa_default_params(k=wl["k"], index_heads=heads)
    ws = lsa.workspace(lsa.lsa_index_workspace_bytes(chunk, layer.cache.n_blocks, p), dev)
    lists, lens = layer.lists, layer.lens

    def run():
        for a in range(0, nq, chunk):
            b = min(nq, a + chunk)
            lsa.lsa_index_prefill(qh[a:b], pos[a:b], layer.cache, None, lists[:b - a], lens[:b - a], p, ws)

    ts = []
    for r in range(4):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        run()
        e1.record()
        torch.cuda.synchronize()
        if r >= 1:
            ts.append(e0.elapsed_time(e1))
    ms = float(np.median(ts))
    del ws, qh
    torch.cuda.empty_cache()
    return {"heads": heads, "queries": nq, "chunk": chunk, "ms": round(ms, 3),
            "tokens_per_s": round(nq / (ms / 1e3), 1)}


def measure_context_parallel(wl: dict, keys_np, pos_np, q_np, Q, K, V, dev, ranks: int, chunk: int = 16384):
    """The context-parallel step of the workload split over `ranks` token
    ranges, every rank's stages run one after another on this one GPU (the
    all-gathers become stacking): per stage, the slowest rank's kernel time
    over all queries (chunks of `chunk`), and the bytes each rank would
    send and receive.  Communication time is not included."""
    from hierarchical_key_clustering_b200 import context_parallel as CP

    T, nq, hq, hkv = wl["T"], len(pos_np), wl["hq"], wl["hkv"]
    chunk = min(chunk, nq)
    shards = [CP.Shard(r, ranks, T, k=wl["k"], max_queries=chunk, device=dev) for r in range(ranks)]
    keys = torch.from_numpy(keys_np).to(dev)
    qidx = torch.from_numpy(q_np).to(dev)
    pos = torch.from_numpy(pos_np).to(dev)
    Lmax = shards[0].Lmax
    ws_attn = lsa.workspace(lsa.lsa_attention_workspace_bytes(chunk, hq, 128, Lmax), dev)
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    t_build = []
    for s in shards:
        a, b = ev(), ev()
        a.record()
        s.build(keys[s.t0:s.t1])
        b.record()
        t_build.append((a, b))
    M = torch.stack([s.members_slice for s in shards])
    C = torch.stack([s.count_slice for s in shards])
    for s in shards:
        s.set_members(M, C)

    def one_pass(record):
        t_loc = [[] for _ in shards]
        t_att = [[] for _ in shards]
        t_mrg, t_cmb = [], []
        for c0 in range(0, nq, chunk):
            c1 = min(nq, c0 + chunk)
            xs = []
            for r, s in enumerate(shards):
                a, b = ev(), ev()
                a.record()
                xs.append(s.index_local(qidx[c0:c1], pos[c0:c1]))
                b.record()
                t_loc[r].append((a, b))
            X = torch.stack(xs).reshape(-1)
            a, b = ev(), ev()
            a.record()
            lists, lens = shards[0].index_merge(X, pos[c0:c1])  # every rank does the same
            b.record()
            t_mrg.append((a, b))
            parts = []
            for r, s in enumerate(shards):
                a, b = ev(), ev()
                a.record()
                parts.append(s.attend_local(Q[c0:c1], K[s.t0:s.t1], V[s.t0:s.t1], lists, lens, ws=ws_attn))
                b.record()
                t_att[r].append((a, b))
            Op, Lp = torch.stack([p_[0] for p_ in parts]), torch.stack([p_[1] for p_ in parts])
            a, b = ev(), ev()
            a.record()
            CP.Shard.combine(Op, Lp)
            b.record()
            t_cmb.append((a, b))
        torch.cuda.synchronize()
        if not record:
            return None
        ms = lambda L: sum(a.elapsed_time(b) for a, b in L)  # noqa: E731
        return ([ms(L) for L in t_loc], ms(t_mrg), [ms(L) for L in t_att], ms(t_cmb))

    one_pass(False)
    loc, mrg, att, cmb = one_pass(True)
    per_rank = [loc[r] + mrg + att[r] + cmb for r in range(ranks)]
    step = max(per_rank)
    xbytes = lsa.lsa_shard_exchange_bytes(nq, shards[0].p)
    part_bytes = nq * hq * (128 * 2 + 4)
    return {"ranks": ranks, "emulated_on_one_gpu": True, "queries": nq, "chunk": chunk,
            "build_ms_max_rank": round(max(a.elapsed_time(b) for a, b in t_build), 3),
            "index_local_ms": {"max_rank": round(max(loc), 3), "min_rank": round(min(loc), 3)},
            "merge_and_expand_ms": round(mrg, 3),
            "attention_local_ms": {"max_rank": round(max(att), 3), "min_rank": round(min(att), 3)},
            "combine_ms": round(cmb, 3), "step_ms_slowest_rank": round(step, 3),
            "tokens_per_s_without_communication": round(nq / (step / 1e3), 1),
            "allgather_bytes_sent_per_rank": xbytes + part_bytes,
            "allgather_bytes_received_per_rank": (ranks - 1) * (xbytes + part_bytes),
            "note": "kernel time per rank only; the all-gathers of exchange blocks and attention parts are not timed"}


def run_ours(args, world, rank, local):
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    wl = dict(I.WORKLOADS[args.workload])
    if args.queries:
        wl["n_prefill"] = min(args.queries, wl["n_prefill"])
    if args.mode:
        wl["mode"] = args.mode
    if wl["mode"] == "both":
        wl["mode"] = "flat"
    T, nq, hq, hkv = wl["T"], wl["n_prefill"], wl["hq"], wl["hkv"]
    keys_np, q_np, pos_np = make_prefill_inputs(wl)
    layer = SparseLayer(T, k=wl["k"], mode=wl["mode"], beam=wl.get("beam", 32), max_queries=nq, Hq=hq)
    keys = torch.from_numpy(keys_np).to(dev)
    qidx = torch.from_numpy(q_np).to(dev)
    pos = torch.from_numpy(pos_np).to(dev)
    Q, K, V = device_qkv(nq, T, hq, hkv)
    O = torch.empty_like(Q)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    st = torch.cuda.current_stream()

    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731

    def step(times=None):
        e0, e1, e2, e3 = ev(), ev(), ev(), ev()
        e0.record(st)
        layer.build(keys)
        e1.record(st)
        layer.index(qidx, pos)
        e2.record(st)
        layer.attend(Q, K, V, O)
        e3.record(st)
        if times is not None:
            times.append((e0, e1, e2, e3))

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    lens_np = layer.lens[:nq].cpu().numpy()

    launches0 = lsa.lsa_launch_count()
    lsa.lsa_attention_timing_read()  # drop the warm-up calls' events
    lsa.lsa_attention_timing(True)
    clk = Clocks(local)
    barrier(world)
    torch.cuda.synchronize()
    clk.start()
    times = []
    for _ in range(args.steps):
        flush.zero_()
        step(times)
    torch.cuda.synchronize()
    clocks = clk.stop()
    barrier(world)
    launches = lsa.lsa_launch_count() - launches0
    lsa.lsa_attention_timing(False)
    near_ms, gather_ms, n_calls = lsa.lsa_attention_timing_read()
    per = np.array([[a.elapsed_time(b), b.elapsed_time(c), c.elapsed_time(d), a.elapsed_time(d)]
                    for a, b, c, d in times])
    total_ms = float(per[:, 3].sum())
    total_ms = max_over_ranks(total_ms, world)
    ms_step = total_ms / args.steps
    value = world * nq * args.steps / (total_ms / 1e3)

    # roofline of the dominant kernel: k_attn, the far-key gather (one launch
    # per step), timed by the library's events around it on the step's stream
    pk = peaks()
    if near_ms > 0.0:  # the near-set tiles ran
        near_rows, far_rows = near_split_rows(layer.lists[:nq], layer.lens[:nq])
    else:
        near_rows, far_rows = 0, int(lens_np.astype(np.int64).sum())
    attn_ms = gather_ms / max(1, n_calls)
    abytes = attn_algorithmic_bytes(far_rows, nq, hq, hkv)
    achieved = abytes / (attn_ms / 1e3) / 1e9
    traffic = None
    per_row = ATTN_DRAM_BYTES_PER_FAR_ROW.get(args.workload) if wl["mode"] == "flat" else None
    if per_row is not None:
        traffic = int(per_row * far_rows * hkv)
    roofline = {"kernel": "k_attn", "bound": "hbm", "achieved": round(achieved, 1), "peak": pk["hbm"],
                "unit": "GB/s", "frac": round(achieved / pk["hbm"], 4), "traffic": traffic,
                "peak_source": pk["src"], "algorithmic_bytes": abytes, "launch_ms": round(attn_ms, 3),
                "traffic_note": "ncu DRAM bytes per far row of this workload's launch, times its far rows",
                "near": {"kernels": "k_near_plan + k_attn_near", "ms": round(near_ms / max(1, n_calls), 3),
                         "rows_per_query": round(near_rows / nq, 1),
                         "far_rows_per_query": round(far_rows / nq, 1)}}
    if traffic is not None:  # the same launch measured on the DRAM side: bytes that really crossed HBM
        roofline["dram_achieved"] = round(traffic / (attn_ms / 1e3) / 1e9, 1)
        roofline["dram_frac"] = round(traffic / (attn_ms / 1e3) / 1e9 / pk["hbm"], 4)

    roofline["shrink"] = measure_shrink(K, dev, pk["hbm"])
    index_heads = None
    if wl["mode"] == "flat" and not args.no_heads:
        index_heads = measure_index_heads(layer, keys_np, pos_np, wl, dev)
    context_parallel = None
    if args.cp > 1 and wl["mode"] == "flat":
        context_parallel = measure_context_parallel(wl, keys_np, pos_np, q_np, Q, K, V, dev, args.cp)

    # end to end: same calls, inputs from pinned host memory, output back to host
    e2e = None if args.no_e2e else run_e2e(args, layer, keys_np, q_np, pos_np, Q, K, V, dev, world)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl, keys_np, q_np, pos_np, K, V, hq, budget_s=args.cpu_budget)

    decode = None
    if not args.no_decode:
        del Q, K, V, O, flush, layer
        torch.cuda.empty_cache()
        dwl = "flat_1m" if args.workload == "flat_128k" else args.workload
        decode = run_decode(args, dev, dwl, wl["mode"])

    line = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": args.workload if not args.queries else f"{args.workload}[last {nq} queries]",
                   "T": T, "queries": nq, "k": wl["k"], "sink": 4, "window": 512,
                   "mode": wl["mode"], "Hq": hq, "Hkv": hkv, "head_dim": 128, "index_dim": 64,
                   "mixture_components": wl["n_components"], "parallelism": "replicas",
                   "l2": "256 MiB buffer written between timed steps; K/V exceed L2"},
        "breakdown_ms": {"build": round(float(per[:, 0].mean()), 3), "index": round(float(per[:, 1].mean()), 3),
                         "attention": round(float(per[:, 2].mean()), 3)},
        "roofline": roofline,
        "e2e": e2e,
        "gpu_launches": int(launches),
        "clocks": clocks,
        "decode": decode,
        "index_heads": index_heads,
    }
    if context_parallel is not None:
        line["context_parallel"] = context_parallel
    if cpu is not None:
        line["cpu_baseline"] = cpu
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_e2e(args, layer, keys_np, q_np, pos_np, Qd, Kd, Vd, dev, world):
    """The step through SparseLayer.prefill_from_host: inputs from pinned host
    memory, O back to pinned host memory, every step (transfers overlapped
    with the kernels on copy streams, the step still ends after its last
    copy back)."""
    st = torch.cuda.current_stream()
    pin = lambda a: torch.from_numpy(a).pin_memory()  # noqa: E731
    h_keys, h_q, h_pos = pin(keys_np), pin(q_np), pin(pos_np)
    h_Q, h_K, h_V = Qd.cpu().pin_memory(), Kd.cpu().pin_memory(), Vd.cpu().pin_memory()
    h_O = torch.empty(Qd.shape, dtype=Qd.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in (h_keys, h_q, h_pos, h_Q, h_K, h_V))
    d2h = h_O.numel() * h_O.element_size()

    def step():
        layer.prefill_from_host(h_keys, h_q, h_pos, h_Q, h_K, h_V, h_O)

    for _ in range(max(1, args.warmup)):
        step()
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for _ in range(args.steps):
        step()
    e1.record(st)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), world)
    nq = q_np.shape[0]
    return {"value": round(world * nq * args.steps / (ms / 1e3), 1), "unit": UNIT,
            "ms_per_step": round(ms / args.steps, 3), "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h)}


def run_decode(args, dev, workload="flat_1m", mode="flat"):
    """Decode at T = 1M (Flat, k = 4096): per new token, batch 1, the index of
    that token (lsa_index_decode) and its sparse attention.  The two calls are
    captured once in a CUDA graph; each token copies its query into the
    graph's input buffers and replays it (both inside the timed region).
    Mean us/token over 64 tokens; the eager (uncaptured) figure is kept too."""
    wl = I.WORKLOADS[workload]
    T, nd, hq, hkv = wl["T"], wl["n_decode"], wl["hq"], wl["hkv"]
    keys_all = I.index_keys(0, T + nd, wl["n_components"])
    pos_np = np.arange(T, T + nd, dtype=np.int64)
    q_np = I.index_queries(0, keys_all, pos_np)
    layer = SparseLayer(T, k=wl["k"], mode=mode, beam=wl.get("beam", 32), max_queries=1, Hq=hq)
    layer.build(torch.from_numpy(keys_all[:T]).to(dev))
    g = torch.Generator(device=dev)
    g.manual_seed(77)
    K = torch.randn((T + nd, hkv, 128), generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)
    V = torch.randn((T + nd, hkv, 128), generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)
    Qd = torch.randn((nd, 1, hq, 128), generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)
    qd = torch.from_numpy(q_np).to(dev)
    pd = torch.from_numpy(pos_np).to(dev)
    q_in, p_in, Q_in = qd[:1].clone(), pd[:1].clone(), Qd[0].clone()
    O = torch.empty((1, hq, 128), dtype=torch.bfloat16, device=dev)

    def token():
        layer.index(q_in, p_in, decode=True)
        layer.attend(Q_in, K, V, O)

    def feed(i):
        q_in.copy_(qd[i:i + 1])
        p_in.copy_(pd[i:i + 1])
        Q_in.copy_(Qd[i])

    for i in range(4):
        feed(i)
        token()
    torch.cuda.synchronize()
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    e0, e1 = ev(), ev()
    e0.record()
    for i in range(nd):
        feed(i)
        token()
    e1.record()
    torch.cuda.synchronize()
    eager_us = e0.elapsed_time(e1) * 1e3 / nd
    lens = int(layer.lens[:1].item())
    graph_us, note = None, None
    try:
        graph = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            token()
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        with torch.cuda.graph(graph):
            token()
        for i in range(4):
            feed(i)
            graph.replay()
        torch.cuda.synchronize()
        e0, e1 = ev(), ev()
        e0.record()
        for i in range(nd):
            feed(i)
            graph.replay()
        e1.record()
        torch.cuda.synchronize()
        graph_us = e0.elapsed_time(e1) * 1e3 / nd
    except Exception as ex:  # report, keep the eager number
        note = f"graph capture failed: {type(ex).__name__}: {ex}"[:200]
    # a block completes every 512 decode tokens: pool and cluster it and grow
    # the tree in place (the cache and tree are rewound to T - 512 each time,
    # re-running a range rewrites identical values); a full tree rebuild for
    # comparison
    keys_d = torch.from_numpy(keys_all[:T]).to(dev)
    nb = T // 512
    app = []
    for r in range(6):
        layer.cache.c.n_blocks = nb - 1
        if layer.tree is not None:
            layer.tree.t.n_blocks = nb - 1
        e0, e1 = ev(), ev()
        e0.record()
        layer.append(keys_d, T - 512, T)
        e1.record()
        torch.cuda.synchronize()
        if r >= 2:
            app.append(e0.elapsed_time(e1) * 1e3)
    rebuild_us = None
    if layer.tree is not None:
        reb = []
        for r in range(4):
            e0, e1 = ev(), ev()
            e0.record()
            lsa.lsa_build_tree(layer.cache, layer.tree, layer.p)
            e1.record()
            torch.cuda.synchronize()
            if r >= 1:
                reb.append(e0.elapsed_time(e1) * 1e3)
        rebuild_us = round(float(np.median(reb)), 1)
    out = {"workload": workload, "mode": mode, "T": T, "tokens": nd, "k": wl["k"], "list_len": lens,
           "us_per_token": round(graph_us if graph_us is not None else eager_us, 2),
           "us_per_token_eager": round(eager_us, 2),
           "block_append_us": round(float(np.median(app)), 1), "tree_rebuild_us": rebuild_us,
           "note": "batch 1; lsa_index_decode + lsa_sparse_attention per token, replayed from one CUDA graph; "
                   "block_append_us: pool + cluster one completed block and grow the tree in place (every 512 "
                   "tokens)"}
    if note:
        out["note"] = note
    return out


# --------------------------------------------------------------------------- CPU oracle

def cpu_baseline(wl, keys_np, q_np, pos_np, K, V, hq, budget_s=20.0, sample=None):
    """The oracle as it stands on this host's cores: full cache build + index and
    attention of evenly spaced sample queries, extrapolated to all queries."""
    import oracle as O
    cores = len(os.sched_getaffinity(0))
    os.environ.setdefault("OMP_NUM_THREADS", str(cores))
    O.build()
    nq = len(pos_np)
    t0 = time.perf_counter()
    oc = O.build_cache(keys_np)
    ot = O.build_tree(oc) if wl["mode"] == "tree" else None
    t_build = time.perf_counter() - t0
    Kb = K.view(torch.int16).cpu().numpy().view(np.uint16)
    Vb = V.view(torch.int16).cpu().numpy().view(np.uint16)
    hkv = Kb.shape[1]
    S = sample or 64
    done, t_q = 0, 0.0
    rng_idx = np.linspace(0, nq - 1, 4096).astype(np.int64)
    while True:
        sel = rng_idx[(np.arange(S) * 4096 // S)]
        Qb = I.normal_bf16_bits(1, I.STREAM_Q, (S, hq, 128))
        t0 = time.perf_counter()
        lists, lens = O.index(q_np[sel], pos_np[sel], oc, k=wl["k"], mode=wl["mode"], tree=ot,
                              beam=wl.get("beam", 32))
        O.attention(Qb, Kb, Vb, lists, lens)
        t_q = time.perf_counter() - t0
        done = S
        if t_q * 2 > budget_s or S >= 1024:
            break
        S *= 2
    per_q = t_q / done
    total = t_build + per_q * nq
    return {"value": round(nq / total, 2), "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"full cache build ({t_build:.2f} s) + index and attention of {done} evenly spaced of "
                      f"{nq} queries ({t_q:.2f} s), extrapolated to all queries",
            "hkv": hkv}


def run_reference(args, world, rank):
    """The reference arm: the CPU oracle on this host, same metric and workload."""
    if rank != 0:
        return
    wl = dict(I.WORKLOADS[args.workload])
    wl["mode"] = args.mode or ("flat" if wl["mode"] == "both" else wl["mode"])
    keys_np, q_np, pos_np = make_prefill_inputs(wl)
    T, nq, hq, hkv = wl["T"], wl["n_prefill"], wl["hq"], wl["hkv"]
    Kb = torch.from_numpy(I.normal_bf16_bits(0, I.STREAM_K, (T, hkv, 128)).view(np.int16)).view(torch.bfloat16)
    Vb = torch.from_numpy(I.normal_bf16_bits(0, I.STREAM_V, (T, hkv, 128)).view(np.int16)).view(torch.bfloat16)
    vals = []
    for _ in range(args.warmup + args.steps):
        vals.append(cpu_baseline(wl, keys_np, q_np, pos_np, Kb, Vb, hq, budget_s=args.cpu_budget, sample=32))
    vals = vals[args.warmup:]
    v = float(np.mean([x["value"] for x in vals]))
    line = {"metric": METRIC, "value": round(v, 2), "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(nq / v * 1e3, 1), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64/f32 (CPU oracle)", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": args.workload if not args.queries else f"{args.workload}[last {nq} queries]",
                   "T": T, "queries": nq, "k": wl["k"], "mode": wl["mode"],
                       "Hq": hq, "Hkv": hkv, "head_dim": 128, "parallelism": "host cores"},
            "cpu_baseline": {"value": round(v, 2), "unit": UNIT, "cores": vals[-1]["cores"], "kind": "oracle",
                             "sample": vals[-1]["sample"]},
            "e2e": {"value": round(v, 2), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "gpu_launches": 0}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="flat_128k", choices=sorted(I.WORKLOADS))
    ap.add_argument("--queries", type=int, default=0,
                    help="time only the last N prefill queries of the workload (profiling slices)")
    ap.add_argument("--mode", default=None, choices=["flat", "tree"], help="override the workload's search mode")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-heads", action="store_true", help="skip the multi-head Flat index measurement")
    ap.add_argument("--cp", type=int, default=0,
                    help="also run an N-way context-parallel split, its ranks one after another on this GPU")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=20.0)
    args = ap.parse_args()
    world, rank, local = init_dist()
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            run_ours(args, world, rank, local)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
