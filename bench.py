#!/usr/bin/env python
"""Benchmark of the balancer's per-layer, per-microbatch hot path on B200.

One step = one pass of the whole path over one microbatch: load -> plan ->
reroute (the "rebalance") -> replica weight sync -> replica gradient
reduction, all through the C ABI of libue.so, with every input resident in
HBM.  The headline value is the rebalance latency in microseconds per
layer-microbatch; weight-sync and grad-reduce bandwidths are reported beside
it against the measured HBM copy peak.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...   # the CPU oracle on the host cores

Under torchrun (N > 1) every rank runs an independent replica of the
workload on its own GPU (the path does not shard: no data-path collective);
timings are the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from moe_expert_load_ue_b200 import inputs  # noqa: E402

METRIC = "rebalance µs/layer-microbatch (load+plan+reroute); sync & grad-reduce HBM GB/s"
UNIT = "µs"
FALLBACK_HBM_GBS = 6650.0
VARIANTS = {"requeue": 1, "spread": 2, "requeue+spread": 3}     # plan variant bits (UE_PLAN_*)
# DRAM bytes of one launch from an ncu capture (dram__bytes_read.sum +
# dram__bytes_write.sum) next to that launch's algorithmic bytes, per kernel
# and full-size workload; summarised in profiles/.  The JSON's roofline.traffic
# scales the measured ratio to the mean launch of the run, and is null when the
# kernel's sources (its file and header, hashed together) no longer match the
# ones that were captured.
TRAFFIC = {
    ("grad_reduce", "671B-class"): {
        "sources": ["moe_expert_load_ue_b200/csrc/ue_grad_reduce.cu", "moe_expert_load_ue_b200/csrc/ue_grad.cuh"],
        "sha256": "84d2f94dab75115c86e4fb4eaed56f4b7ab6abc45c4dc9ee2dc5fe468a45f3f0",
        "dram_bytes": 7903370496, "algorithmic_bytes": 7927234560,
        "profile": "profiles/grad_reduce_and_sync_dram_671B-class.md"},
    ("sync", "671B-class"): {
        "sources": ["moe_expert_load_ue_b200/csrc/ue_sync.cu", "moe_expert_load_ue_b200/csrc/ue_bulk.cuh"],
        "sha256": "30d277eb08f295b207de478b8bbae039ddf6a66e4e350f56fe563415d7bd29e1",
        "dram_bytes": 4962409728, "algorithmic_bytes": 5020581888,
        "profile": "profiles/grad_reduce_and_sync_dram_671B-class.md"},
}


# Each ncu summary under profiles/ with the kernel sources it was captured on
# (the files hashed together, in this order); the JSON line's "profiles" object
# reports each as "current" or "stale" (the code changed since the capture).
PROFILES = {
    "profiles/launch_list_671B-class.md": {
        "sources": ["moe_expert_load_ue_b200/csrc/ue_load.cu", "moe_expert_load_ue_b200/csrc/ue_plan.cu", "moe_expert_load_ue_b200/csrc/ue_reroute.cu", "moe_expert_load_ue_b200/csrc/ue_sync.cu", "moe_expert_load_ue_b200/csrc/ue_bulk.cuh", "moe_expert_load_ue_b200/csrc/ue_grad_reduce.cu", "moe_expert_load_ue_b200/csrc/ue_grad.cuh"],
        "sha256": "e57c3082f70b10a83401255ec6446612178b7df6601eab8bc36b02c21d589931"},
    "profiles/hot_path_kernels_full_set_671B-class_small_experts.md": {
        "sources": ["moe_expert_load_ue_b200/csrc/ue_load.cu", "moe_expert_load_ue_b200/csrc/ue_plan.cu", "moe_expert_load_ue_b200/csrc/ue_reroute.cu"],
        "sha256": "03db1fa3cdc407f27b2380446dc7ffad9df87b426c73b4fe5146d8092f7f3170"},
    "profiles/grad_reduce_and_sync_dram_671B-class.md": {
        "sources": ["moe_expert_load_ue_b200/csrc/ue_grad_reduce.cu", "moe_expert_load_ue_b200/csrc/ue_grad.cuh", "moe_expert_load_ue_b200/csrc/ue_sync.cu", "moe_expert_load_ue_b200/csrc/ue_bulk.cuh"],
        "sha256": "b9abe4d9121c77eacef6677e75661787b8ba03244a94c6be4cc03dd3806bd751"},
    "profiles/grad_reduce_bulk_full_set_671B-class_small_experts.md": {
        "sources": ["moe_expert_load_ue_b200/csrc/ue_grad_reduce.cu", "moe_expert_load_ue_b200/csrc/ue_grad.cuh"],
        "sha256": "84d2f94dab75115c86e4fb4eaed56f4b7ab6abc45c4dc9ee2dc5fe468a45f3f0"},
    "profiles/reroute_pieces_full_set_sweep_256x32768.md": {
        "sources": ["moe_expert_load_ue_b200/csrc/ue_reroute_pieces.cu"],
        "sha256": "b7a569b8c061375205de5e91ce6748c7d57b75a3bdcb83db7cd7753fbcc90e82"},
    "profiles/dispatch_layout_671B-class_small_experts.md": {
        "sources": ["moe_expert_load_ue_b200/csrc/ue_reroute.cu"],
        "sha256": "6f1fe8f23d9a123d558ba2f6db0ed74b3e6aca91013f82ffdb93c6b289aa27e5"},
    "profiles/sync_and_grad_across_gpus_dram_671B-class_emulated.md": {
        "sources": ["moe_expert_load_ue_b200/csrc/ue_shard.cu", "moe_expert_load_ue_b200/csrc/ue_bulk.cuh", "moe_expert_load_ue_b200/csrc/ue_grad_reduce.cu", "moe_expert_load_ue_b200/csrc/ue_grad.cuh"],
        "sha256": "9c1747afaab1a7b76e1cb389c15d37ca9033c2971500ae78c90356b73e392cd6"},
}


def _sources_hash(sources) -> str | None:
    import hashlib
    m = hashlib.sha256()
    try:
        for src in sources:
            with open(os.path.join(ROOT, src), "rb") as f:
                m.update(f.read())
    except OSError:
        return None
    return m.hexdigest()


def profile_status() -> dict:
    return {os.path.basename(p): ("current" if _sources_hash(t["sources"]) == t["sha256"] else "stale")
            for p, t in PROFILES.items()}


def traffic_per_launch(kernel: str, workload: str, full_size: bool, mean_alg: float):
    t = TRAFFIC.get((kernel, workload))
    if t is None or not full_size:
        return None
    if _sources_hash(t["sources"]) != t["sha256"]:
        return None
    return round(t["dram_bytes"] / t["algorithmic_bytes"] * mean_alg)


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default="671B-class", choices=sorted(inputs.WORKLOADS))
    ap.add_argument("--microbatches", type=int, default=None,
                    help="distinct resident microbatches cycled by the steps (default: the workload's)")
    ap.add_argument("--expert-shape", default=None,
                    help="override the expert matrices' rows x cols (e.g. 1024x512) for small profiling cases")
    ap.add_argument("--sweep", action="store_true",
                    help="rebalance latency and imbalance over the sweep grid (one JSON line per point)")
    ap.add_argument("--sweep-seeds", type=int, default=1)
    ap.add_argument("--sweep-only", default=None,
                    help="run only the sweep points TPR:N:S (comma-separated list), without the sync/grad lines")
    ap.add_argument("--stationary", action="store_true",
                    help="keep the expert popularity fixed across microbatches (no re-permutation)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-across-gpus", action="store_true",
                    help="with N > 1, skip the sharded calls across the GPUs after the timed region")
    return ap.parse_args(argv)


# ---- distributed plumbing (barrier and max over ranks only) -----------------------

class Dist:
    def __init__(self):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local_rank = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = None

    def init(self, backend: str):
        if self.world > 1:
            import datetime

            import torch.distributed as dist
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
            self.pg = dist
        return self

    def barrier(self):
        if self.pg:
            self.pg.barrier()

    def max(self, values, device=None):
        """Element-wise max over ranks of a list of floats."""
        if not self.pg:
            return list(values)
        import torch
        t = torch.tensor(list(values), dtype=torch.float64, device=device)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return t.tolist()

    def sum(self, values, device=None):
        if not self.pg:
            return list(values)
        import torch
        t = torch.tensor(list(values), dtype=torch.float64, device=device)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.SUM)
        return t.tolist()

    def close(self):
        if self.pg:
            self.pg.destroy_process_group()


# ---- clocks ---------------------------------------------------------------------

class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str, period_ms: int = 100):
        self.gpu_id, self.period_ms = gpu_id, period_ms
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", str(self.period_ms), "-f", self.path],
                stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
        except (OSError, ValueError):
            self.proc = None
        time.sleep(0.3)
        return self

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, power, reasons = [], [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 8:
                    continue
                try:
                    sm.append(float(parts[0]))
                    smax.append(float(parts[1]))
                    power.append(float(parts[2]))
                except ValueError:
                    continue
                for n, v in zip(names, parts[4:8]):
                    if v.lower().startswith("active"):
                        reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "samples": len(sm),
                "power_w_max": max(power) if power else None, "reasons": sorted(reasons)}


def measured_peaks() -> tuple[float, str]:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            v = float(json.load(f)["hbm_gbs"])
        return v, "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def workload_of(args, rank):
    """The bench's workload (rank r of a replicas run draws with base seed r)."""
    w = inputs.WORKLOADS[args.workload].with_(base_seed=rank)
    if args.stationary:
        w = w.with_(repermute=False)
    if args.expert_shape:
        rows, cols = (int(x) for x in args.expert_shape.lower().split("x"))
        w = w.with_(rows=rows, cols=cols)
    return w


def workload_config(w, n_mb, world):
    """The JSON line's config (the same for both arms)."""
    return {"workload": w.name, "E": w.E, "N": w.N, "H": w.H, "R": w.R, "K": w.K, "T": w.T,
            "P": w.P, "slot_bytes": 2 * w.P, "grad_dtype": w.grad_dtype, "zipf_s": w.s,
            "microbatches_cycled": n_mb, "parallelism": f"replicas x{world}",
            "popularity": "re-drawn every microbatch" if w.repermute else "stationary",
            "l2": "inputs larger than L2: every step streams > 1 GB (sync + grad reduce), "
                  "so each rebalance reads its ids from HBM"}


# ---- the GPU arm ------------------------------------------------------------------

NVLINK_GBS = 770.0     # measured peer copy per direction per GPU on this machine's B200s (NVLink 5)


def nvlink_model(slot_expert, w, G, slot_bytes, gbs):
    """Bytes each GPU sends and receives between GPUs in each relay round and
    in the direct form, from the plan's slot table (consumers of an expert: the
    GPUs other than its home GPU with a filled redundant slot of it, in
    increasing id; the slot cut into f parts of q = 16*ceil(slot_bytes/(16 f))
    bytes; round 0: consumer j receives part j from the home; round 1: each
    consumer receives every other part from its consumer), and the resulting
    time if every round ran at `gbs` per direction on its busiest GPU."""
    SG = w.S // G
    red = (np.arange(w.S) % (w.H + w.R)) >= w.H
    rounds = 1 if G <= 2 else 2
    eg_r, in_r = np.zeros((rounds, G)), np.zeros((rounds, G))
    eg_d, in_d = np.zeros(G), np.zeros(G)
    for e in np.unique(slot_expert[red & (slot_expert >= 0)]):
        hg = ((e // w.H) * (w.H + w.R)) // SG
        cons = sorted(set((np.nonzero(red & (slot_expert == e))[0] // SG).tolist()) - {hg})
        f = len(cons)
        if f == 0:
            continue
        q = 16 * -(-slot_bytes // (16 * f))
        part = [max(0, min(q, slot_bytes - j * q)) for j in range(f)]
        for j, c in enumerate(cons):
            eg_r[0, hg] += part[j]
            in_r[0, c] += part[j]
            eg_d[hg] += slot_bytes
            in_d[c] += slot_bytes
            for i, d in enumerate(cons):
                if i != j:
                    eg_r[1, c] += part[j]
                    in_r[1, d] += part[j]
    per_round = np.maximum(eg_r.max(axis=1), in_r.max(axis=1))
    return {"relay_us": float(per_round.sum() / (gbs * 1e9) * 1e6),
            "direct_us": float(max(eg_d.max(), in_d.max()) / (gbs * 1e9) * 1e6),
            "relay_max_egress": float(eg_r.max()), "direct_max_egress": float(eg_d.max()),
            "relay_egress": eg_r, "direct_egress": eg_d}


def run_ours(args, dist: Dist):
    import torch

    from moe_expert_load_ue_b200 import ue

    torch.cuda.set_device(dist.local_rank)
    dev = torch.device("cuda", dist.local_rank)
    dist.init("nccl")
    w = workload_of(args, dist.rank)
    n_mb = args.microbatches or w.microbatches
    cfg = ue.Config(E=w.E, N=w.N, R=w.R, K=w.K, T=w.T)
    ctx = ue.Context(dist.local_rank)
    stream = torch.cuda.Stream(device=dev)

    # Inputs: every microbatch's ids resident in HBM (and pinned on the host for the e2e leg).
    ids_host = [inputs.topk_ids(w, mb) for mb in range(n_mb)]
    ids_dev = torch.empty((n_mb, w.T, w.K), dtype=torch.int32, device=dev)
    for mb in range(n_mb):
        ids_dev[mb].copy_(torch.from_numpy(ids_host[mb]))
    counts = torch.empty((w.N, w.E), dtype=torch.int32, device=dev)
    bad = torch.empty(w.N, dtype=torch.int32, device=dev)
    plan = ue.Plan(cfg, device=dev)
    phys = torch.empty((w.T, w.K), dtype=torch.int32, device=dev)
    P = w.P
    slot_bytes = 2 * P
    gen = torch.Generator(device=dev).manual_seed(1234 + dist.rank)
    weights = torch.empty((w.S, P), dtype=torch.bfloat16, device=dev)
    for s in range(w.S):
        weights[s].normal_(0.0, 0.02, generator=gen)
    gdt = torch.bfloat16 if w.grad_dtype == "bf16" else torch.float32
    grads = torch.empty((w.N * w.R, P), dtype=gdt, device=dev)
    for r in range(w.N * w.R):
        grads[r].normal_(0.0, 1e-3, generator=gen)
    master = torch.empty((w.E, P), dtype=torch.float32, device=dev)
    for e in range(w.E):
        master[e].normal_(0.0, 1e-3, generator=gen)
    torch.cuda.synchronize(dev)

    def step(mb, ev=None):
        ids = ids_dev[mb]
        if ev:
            ev[0].record(stream)
        ue.ue_rebalance(ctx, cfg, ids, counts, bad, plan, phys, stream=stream)   # load + plan + reroute
        if ev:
            ev[1].record(stream)
        ue.ue_sync(ctx, cfg, weights, slot_bytes, plan, stream=stream)
        if ev:
            ev[2].record(stream)
        ue.ue_grad_reduce(ctx, cfg, master, grads, P, plan, stream=stream)
        if ev:
            ev[3].record(stream)

    KERNELS_PER_STEP = 5     # load, plan, reroute (one ue_rebalance call), sync, grad reduce
    with torch.cuda.stream(stream):
        for k in range(args.warmup):
            step(k % n_mb)
    stream.synchronize()

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    gpu_uuid = str(torch.cuda.get_device_properties(dev).uuid)
    gpu_id = gpu_uuid if gpu_uuid.startswith("GPU-") else f"GPU-{gpu_uuid}"
    clocks = ClockSampler(gpu_id).start()
    dist.barrier()
    torch.cuda.synchronize(dev)
    with torch.cuda.stream(stream):
        for k in range(args.steps):
            step(k % n_mb, evs[k])
    stream.synchronize()
    torch.cuda.synchronize(dev)
    dist.barrier()
    clk = clocks.stop()
    err = ctx.device_error(stream)
    if err:
        raise RuntimeError(f"a kernel gave up a bounded wait (status word {err})")

    seg = np.array([[evs[k][i].elapsed_time(evs[k][i + 1]) for i in range(3)] for k in range(args.steps)]) * 1e3
    total_ms = evs[0][0].elapsed_time(evs[-1][3])
    rebalance_us = seg[:, 0]

    # Per-kernel breakdown of the rebalance: the three steps as separate calls
    # with events between them (no launch overlap), after the timed region.
    n_bd = max(8, min(args.steps, 64))
    evb = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(n_bd)]
    with torch.cuda.stream(stream):
        for k in range(n_bd):
            ids = ids_dev[k % n_mb]
            evb[k][0].record(stream)
            ue.ue_load(ctx, cfg, ids, counts, bad, stream=stream)
            evb[k][1].record(stream)
            ue.ue_plan(ctx, cfg, counts, plan, stream=stream)
            evb[k][2].record(stream)
            ue.ue_reroute(ctx, cfg, ids, plan, phys, stream=stream)
            evb[k][3].record(stream)
            ue.ue_sync(ctx, cfg, weights, slot_bytes, plan, stream=stream)   # keeps L2 cold as in the step
    stream.synchronize()
    bd = np.array([[evb[k][i].elapsed_time(evb[k][i + 1]) for i in range(3)] for k in range(n_bd)]) * 1e3

    # The rebalance with the dispatch layout (slot offsets, per-slot source
    # indices and gates carried along), and the dispatch call alone after a
    # plan; events around each call, a weight sync between reps as in the step.
    gates_dev = torch.empty((n_mb, w.T, w.K), dtype=torch.float32, device=dev)
    for mb in range(n_mb):
        gates_dev[mb].copy_(torch.from_numpy(inputs.gates(ids_host[mb], w, mb)))
    disp = ue.Dispatch(cfg, with_gates=True, device=dev)
    n_dp = max(8, min(args.steps, 64))
    evd = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(n_dp)]
    with torch.cuda.stream(stream):
        for k in range(args.warmup + n_dp):
            mb = k % n_mb
            e = evd[k - args.warmup] if k >= args.warmup else None
            if e:
                e[0].record(stream)
            ue.ue_rebalance_dispatch(ctx, cfg, ids_dev[mb], counts, bad, plan, phys, disp, gates_dev[mb],
                                     stream=stream)
            if e:
                e[1].record(stream)
            ue.ue_sync(ctx, cfg, weights, slot_bytes, plan, stream=stream)
            if e:
                e[2].record(stream)
            ue.ue_dispatch(ctx, cfg, ids_dev[mb], plan, phys, disp, gates_dev[mb], stream=stream)
            if e:
                e[3].record(stream)
            ue.ue_sync(ctx, cfg, weights, slot_bytes, plan, stream=stream)
    stream.synchronize()
    reb_disp_us = float(np.mean([e[0].elapsed_time(e[1]) for e in evd])) * 1e3

    # Warm L2: the ids are written just before the rebalance (a device copy
    # standing in for gating's output, 8.4 MB at 262,144 tokens: well inside
    # the 126 MB L2), so the load kernel reads them from L2.
    ids_warm = torch.empty((w.T, w.K), dtype=torch.int32, device=dev)
    evw = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n_dp)]
    with torch.cuda.stream(stream):
        for k in range(args.warmup + n_dp):
            mb = k % n_mb
            ue.ue_sync(ctx, cfg, weights, slot_bytes, plan, stream=stream)    # L2 cold before the copy
            ids_warm.copy_(ids_dev[mb])
            e = evw[k - args.warmup] if k >= args.warmup else None
            if e:
                e[0].record(stream)
            ue.ue_rebalance(ctx, cfg, ids_warm, counts, bad, plan, phys, stream=stream)
            if e:
                e[1].record(stream)
    stream.synchronize()
    warm_us = float(np.mean([a.elapsed_time(b) for a, b in evw])) * 1e3
    del ids_warm
    disp_call_us = float(np.mean([e[2].elapsed_time(e[3]) for e in evd])) * 1e3
    del gates_dev

    # The rebalance of every microbatch captured once into a CUDA graph (the
    # programmatic launch edges are kept) and replayed back to back: launch
    # overhead is amortised; the ids of all microbatches together exceed L2.
    graph_us = None
    try:
        g = torch.cuda.CUDAGraph()
        cap = torch.cuda.Stream(device=dev)
        with torch.cuda.graph(g, stream=cap):
            for mb in range(n_mb):
                ue.ue_rebalance(ctx, cfg, ids_dev[mb], counts, bad, plan, phys)
        reps = 20
        with torch.cuda.stream(stream):
            g.replay()
            g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            g0.record(stream)
            for _ in range(reps):
                g.replay()
            g1.record(stream)
        stream.synchronize()
        graph_us = g0.elapsed_time(g1) * 1e3 / (reps * n_mb)
        del g
    except RuntimeError as exc:     # capture refused: report no graph figure
        print(f"# rebalance graph timing skipped: {exc}", file=sys.stderr)

    # Plans per microbatch (recomputed after the timed region) for the byte accounting.
    per_mb = []
    with torch.cuda.stream(stream):
        for mb in range(n_mb):
            ue.ue_rebalance(ctx, cfg, ids_dev[mb], counts, bad, plan, phys, stream=stream)
            stream.synchronize()
            info = plan["info"].cpu().numpy()
            per_mb.append({"Q": int(info[0]), "L": int(info[1]), "ran_out": int(info[2] & 1), "M": int(info[3]),
                           "filled": int(info[4]), "max_before": int(info[5]), "max_after": int(info[6]),
                           "slot_expert": plan["slot_expert"].cpu().numpy()})
    gsize = 2 if w.grad_dtype == "bf16" else 4
    sync_bytes = np.array([(p["M"] + p["filled"]) * slot_bytes for p in per_mb], dtype=np.float64)
    grad_bytes = np.array([p["M"] * P * 8 + p["filled"] * P * gsize for p in per_mb], dtype=np.float64)
    step_mb = np.array([k % n_mb for k in range(args.steps)])
    sync_gbs = sync_bytes[step_mb].sum() / (seg[:, 1].sum() * 1e-6) / 1e9
    grad_gbs = grad_bytes[step_mb].sum() / (seg[:, 2].sum() * 1e-6) / 1e9
    rebalance_alg_bytes = 3.0 * w.L * 4

    # Plan variants on the same microbatches: rebalance latency (events around
    # each ue_rebalance_ex) and the imbalance after the plan.
    plan_variants = {}
    for name, v in VARIANTS.items():
        evv = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n_mb)]
        after = []
        with torch.cuda.stream(stream):
            for k in range(args.warmup):        # first launches of the variant's kernels
                ue.ue_rebalance_ex(ctx, cfg, ids_dev[k % n_mb], counts, bad, plan, phys, v, stream=stream)
            for mb in range(n_mb):
                ue.ue_sync(ctx, cfg, weights, slot_bytes, plan, stream=stream)     # keeps L2 cold as in the step
                evv[mb][0].record(stream)
                ue.ue_rebalance_ex(ctx, cfg, ids_dev[mb], counts, bad, plan, phys, v, stream=stream)
                evv[mb][1].record(stream)
                stream.synchronize()
                vi = plan["info"].cpu().numpy()
                after.append(vi[6] / (vi[1] / w.N))
        plan_variants[name] = {"rebalance_us": round(float(np.mean([a.elapsed_time(b) for a, b in evv])) * 1e3, 2),
                               "imbalance_after": round(float(np.mean(after)), 4)}

    # Incremental weight sync over the microbatch sequence of one training
    # step: the first microbatch syncs in full, each later one copies only the
    # redundant slots whose expert changed; two plan buffers alternate.
    plans2 = [plan, ue.Plan(cfg, device=dev)]
    evs_d = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n_mb)]
    with torch.cuda.stream(stream):
        for mb in range(n_mb):
            cur, prv = plans2[mb % 2], plans2[(mb + 1) % 2]
            ue.ue_rebalance(ctx, cfg, ids_dev[mb], counts, bad, cur, phys, stream=stream)
            evs_d[mb][0].record(stream)
            ue.ue_sync_delta(ctx, cfg, weights, slot_bytes, cur, None if mb == 0 else prv["slot_expert"],
                             stream=stream)
            evs_d[mb][1].record(stream)
    stream.synchronize()
    red = (np.arange(w.S) % (w.H + w.R)) >= w.H
    delta_bytes = 0
    for mb in range(n_mb):
        se = per_mb[mb]["slot_expert"]
        ch = red & (se >= 0)
        if mb:
            ch &= se != per_mb[mb - 1]["slot_expert"]
        delta_bytes += (len(np.unique(se[ch])) + int(ch.sum())) * slot_bytes
    delta_full = float(sync_bytes.sum())
    delta_us = float(sum(a.elapsed_time(b) for a, b in evs_d)) * 1e3
    sync_delta = {"microbatches": n_mb, "bytes_full": int(delta_full), "bytes_delta": int(delta_bytes),
                  "saved_frac": round(1.0 - delta_bytes / delta_full, 4) if delta_full else None,
                  "us_total": round(delta_us, 1),
                  "gbs": round(delta_bytes / (delta_us * 1e-6) / 1e9, 1) if delta_us > 0 else None}
    del plans2

    # Weight restore in backward over a stack of layers sharing the redundant
    # slots (the workload's microbatches stand for the layers): forward syncs
    # the layers in order (incrementally), backward restores them last first,
    # each from the experts the slots hold then; events around each restore.
    layer_plans = [ue.Plan(cfg, device=dev) for _ in range(n_mb)]
    held_np = np.full(w.S, -1, np.int32)
    with torch.cuda.stream(stream):
        for li in range(n_mb):
            ue.ue_rebalance(ctx, cfg, ids_dev[li], counts, bad, layer_plans[li], phys, stream=stream)
            ue.ue_sync_delta(ctx, cfg, weights, slot_bytes, layer_plans[li],
                             layer_plans[li - 1]["slot_expert"] if li else None, stream=stream)
            se = per_mb[li]["slot_expert"]
            held_np = np.where(red & (se >= 0), se, held_np)
    held_seq, restore_bytes = [], 0
    for li in reversed(range(n_mb)):
        se = per_mb[li]["slot_expert"]
        held_seq.append(held_np.copy())
        ch = red & (se >= 0) & (se != held_np)
        restore_bytes += (len(np.unique(se[ch])) + int(ch.sum())) * slot_bytes
        held_np = np.where(red & (se >= 0), se, held_np)
    held_dev = torch.from_numpy(np.stack(held_seq)).to(dev)
    evr = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n_mb)]
    with torch.cuda.stream(stream):
        for k, li in enumerate(reversed(range(n_mb))):
            evr[k][0].record(stream)
            ue.ue_sync_restore(ctx, cfg, weights, slot_bytes, layer_plans[li], held_dev[k], stream=stream)
            evr[k][1].record(stream)
    stream.synchronize()
    restore_us = float(sum(a.elapsed_time(b) for a, b in evr)) * 1e3
    sync_delta["restore"] = {
        "note": "backward of a stack of layers sharing the redundant slots (the microbatches' plans as layers): "
                "ue_sync_restore, last layer first, from the experts the slots hold",
        "layers": n_mb, "bytes": int(restore_bytes), "bytes_full_sync": int(delta_full),
        "us_total": round(restore_us, 1),
        "gbs": round(restore_bytes / (restore_us * 1e-6) / 1e9, 1) if restore_us > 0 and restore_bytes else None}
    del layer_plans, held_dev

    # The calls across GPUs with G GPUs emulated as parts of this GPU's memory
    # (each GPU's slots, home-expert master rows and replica-gradient rows):
    # the relay rounds and the direct form of the weight sync, and the
    # gradient reduction on the home GPUs, events around all launches of one
    # microbatch.  Bytes that would cross NVLink are HBM traffic here.
    G = 8 if w.N % 8 == 0 else 1
    SG, EG, RG = w.S // G, w.E // G, (w.N // G) * w.R
    slot_tabs = [weights[h * SG] for h in range(G)]
    grad_tabs = [grads[h * RG] for h in range(G)] if w.R > 0 else None
    rounds = ue.ue_relay_rounds(G)
    n_sh = min(n_mb, 4)
    evs_s = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(n_sh)]
    with torch.cuda.stream(stream):
        for k in range(-1, n_sh):                # one untimed pass first
            mb = max(k, 0)
            ue.ue_rebalance(ctx, cfg, ids_dev[mb], counts, bad, plan, phys, stream=stream)
            e = evs_s[k] if k >= 0 else None
            if e:
                e[0].record(stream)
            for r in range(rounds):
                for h in range(G):
                    ue.ue_sync_shard(ctx, cfg, G, h, slot_tabs, slot_bytes, plan, r, stream=stream)
            if e:
                e[1].record(stream)
            for h in range(G):
                ue.ue_sync_shard(ctx, cfg, G, h, slot_tabs, slot_bytes, plan, -1, stream=stream)
            if e:
                e[2].record(stream)
            for h in range(G):
                ue.ue_grad_reduce_shard(ctx, cfg, G, h, master[h * EG:(h + 1) * EG], grad_tabs, gdt, P, plan,
                                        stream=stream)
            if e:
                e[3].record(stream)
    stream.synchronize()
    sh_pairs, sh_cross = [], []
    for mb in range(n_sh):
        se = per_mb[mb]["slot_expert"]
        pairs = cross = 0
        for e_ in np.unique(se[red & (se >= 0)]):
            gpus = set((np.nonzero(red & (se == e_))[0] // SG).tolist())
            hg = ((e_ // w.H) * (w.H + w.R)) // SG
            pairs += len(gpus)
            cross += len(gpus - {hg})
        sh_pairs.append((pairs + int((red & (se >= 0)).sum())) * slot_bytes)
        sh_cross.append(cross * slot_bytes)
    model = [nvlink_model(per_mb[mb]["slot_expert"], w, G, slot_bytes, NVLINK_GBS) for mb in range(n_sh)]
    t_relay = np.array([e[0].elapsed_time(e[1]) for e in evs_s]) * 1e3
    t_direct = np.array([e[1].elapsed_time(e[2]) for e in evs_s]) * 1e3
    t_grad = np.array([e[2].elapsed_time(e[3]) for e in evs_s]) * 1e3
    sh_bytes = float(np.sum(sh_pairs))
    across_gpus = {
        "G": G, "ranks_per_gpu": w.N // G, "relay_rounds": rounds, "microbatches": n_sh,
        "note": "G GPUs emulated as parts of one GPU's memory; the bytes that would cross NVLink are HBM traffic here",
        "sync_alg_bytes_mean": int(sh_bytes / n_sh), "sync_nvlink_bytes_mean": int(np.mean(sh_cross)),
        "sync_relay_us": round(float(t_relay.mean()), 1),
        "sync_relay_gbs": round(sh_bytes / (t_relay.sum() * 1e-6) / 1e9, 1),
        "sync_direct_us": round(float(t_direct.mean()), 1),
        "sync_direct_gbs": round(sh_bytes / (t_direct.sum() * 1e-6) / 1e9, 1),
        "grad_reduce_us": round(float(t_grad.mean()), 1),
        "grad_reduce_gbs": round(float(grad_bytes[:n_sh].sum()) / (t_grad.sum() * 1e-6) / 1e9, 1),
        "launches_per_microbatch": rounds * G + G + G,
        "nvlink_model": {
            "note": "time on G GPUs if each GPU's busiest direction per round ran at the measured peer-copy "
                    f"bandwidth ({NVLINK_GBS} GB/s per direction), rounds back to back; a model, not a measurement",
            "relay_us": round(float(np.mean([m["relay_us"] for m in model])), 1),
            "direct_us": round(float(np.mean([m["direct_us"] for m in model])), 1),
            "relay_max_egress_bytes_per_round": int(np.mean([m["relay_max_egress"] for m in model])),
            "direct_max_egress_bytes": int(np.mean([m["direct_max_egress"] for m in model])),
        },
    }

    # Across real GPUs (torchrun, N > 1): each rank holds one shard of the
    # resident buffers (its ranks' tokens, slots, home master rows and
    # replica-gradient rows: views, no new memory), maps the other GPUs' through
    # CUDA IPC, and runs the sharded calls with NCCL barriers between them;
    # untimed by the headline, events around each call, max over ranks.
    across_real = None
    if dist.world > 1 and not args.no_across_gpus:
        across_real = across_gpus_real(args, dist, ctx, cfg, w, ids_dev, weights, master, grads, gdt, per_mb,
                                       slot_bytes, red, n_mb)

    # Launch floor: one tiny kernel bracketed by events on the same stream,
    # queued behind a 64 MiB memset so that the host's enqueue time is hidden
    # (as it is for the rebalance inside the step loop): the device-side cost
    # of an event pair around one launch.
    tiny = torch.zeros(1, device=dev)
    busy = torch.empty(64 << 20, dtype=torch.uint8, device=dev)
    floor = []
    with torch.cuda.stream(stream):
        for _ in range(50):
            busy.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            tiny.add_(1.0)
            b.record(stream)
            stream.synchronize()
            floor.append(a.elapsed_time(b) * 1e3)
    launch_floor_us = statistics.median(floor)
    del busy


    # Max over ranks (timings) / sums (work).
    mean_reb = float(rebalance_us.mean())
    vals = dist.max([mean_reb, total_ms, float(seg[:, 1].mean()), float(seg[:, 2].mean())], device=dev)
    mean_reb_max, total_ms_max, sync_us_max, grad_us_max = vals

    # End-to-end through the public API with host buffers: every step copies
    # its ids from pinned host memory, runs ue_rebalance and copies phys and
    # every plan array back.  Pipelined over steps on three streams (H2D,
    # compute, D2H) with two sets of buffers, so one step's D2H overlaps the
    # next step's H2D; value = time per step from the first H2D to the last
    # D2H.  latency_us: the same step alone, copies one after another.
    e2e = None
    if not args.no_e2e:
        ids_pinned = [torch.from_numpy(x).pin_memory() for x in ids_host]
        n_e2e = max(8, min(args.steps, 64))
        nb = 2
        ids_b = [torch.empty((w.T, w.K), dtype=torch.int32, device=dev) for _ in range(nb)]
        phys_b = [torch.empty((w.T, w.K), dtype=torch.int32, device=dev) for _ in range(nb)]
        counts_b = [torch.empty((w.N, w.E), dtype=torch.int32, device=dev) for _ in range(nb)]
        bad_b = [torch.empty(w.N, dtype=torch.int32, device=dev) for _ in range(nb)]
        plan_b = [plan, ue.Plan(cfg, device=dev)]
        phys_h = [torch.empty((w.T, w.K), dtype=torch.int32).pin_memory() for _ in range(nb)]
        plan_h = [torch.empty(plan.buffer.shape, dtype=torch.int32).pin_memory() for _ in range(nb)]
        s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        in_done = [torch.cuda.Event() for _ in range(nb)]
        cmp_done = [torch.cuda.Event() for _ in range(nb)]
        out_done = [torch.cuda.Event() for _ in range(nb)]

        def e2e_step(k):
            b, mb = k % nb, k % n_mb
            if k >= nb:
                s_in.wait_event(out_done[b])            # buffer b's previous step fully copied out
            with torch.cuda.stream(s_in):
                ids_b[b].copy_(ids_pinned[mb], non_blocking=True)
                in_done[b].record(s_in)
            stream.wait_event(in_done[b])
            ue.ue_rebalance(ctx, cfg, ids_b[b], counts_b[b], bad_b[b], plan_b[b], phys_b[b], stream=stream)
            cmp_done[b].record(stream)
            s_out.wait_event(cmp_done[b])
            with torch.cuda.stream(s_out):
                phys_h[b].copy_(phys_b[b], non_blocking=True)
                plan_h[b].copy_(plan_b[b].buffer, non_blocking=True)     # the whole plan in one copy
                out_done[b].record(s_out)

        for k in range(args.warmup):
            e2e_step(k)
        torch.cuda.synchronize(dev)
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(s_in)
        for k in range(n_e2e):
            e2e_step(args.warmup + k)
        t1.record(s_out)
        torch.cuda.synchronize(dev)
        e2e_us = dist.max([t0.elapsed_time(t1) * 1e3 / n_e2e], device=dev)[0]
        # one step alone: copies and rebalance one after another on one stream
        ev2 = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n_e2e)]
        with torch.cuda.stream(stream):
            for k in range(n_e2e):
                mb = k % n_mb
                ev2[k][0].record(stream)
                ids_b[0].copy_(ids_pinned[mb], non_blocking=True)
                ue.ue_rebalance(ctx, cfg, ids_b[0], counts_b[0], bad_b[0], plan_b[0], phys_b[0], stream=stream)
                phys_h[0].copy_(phys_b[0], non_blocking=True)
                plan_h[0].copy_(plan_b[0].buffer, non_blocking=True)
                ev2[k][1].record(stream)
        stream.synchronize()
        lat_us = dist.max([statistics.mean(a.elapsed_time(b) * 1e3 for a, b in ev2)], device=dev)[0]
        # The host link's own floor for these bytes: the same copies, H2D and
        # D2H at once on the two copy streams, with no kernel between them.
        go = torch.cuda.Event()
        link = []
        for k in range(n_e2e + 3):
            a, b1, b2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
            go.record(stream)
            a.record(stream)
            s_in.wait_event(go)
            s_out.wait_event(go)
            with torch.cuda.stream(s_in):
                ids_b[0].copy_(ids_pinned[k % n_mb], non_blocking=True)
                b1.record(s_in)
            with torch.cuda.stream(s_out):
                phys_h[1].copy_(phys_b[1], non_blocking=True)
                plan_h[1].copy_(plan_b[1].buffer, non_blocking=True)
                b2.record(s_out)
            torch.cuda.synchronize(dev)
            if k >= 3:
                link.append(max(a.elapsed_time(b1), a.elapsed_time(b2)) * 1e3)
        link_us = dist.max([statistics.median(link)], device=dev)[0]
        h2d = w.T * w.K * 4
        d2h = w.T * w.K * 4 + plan.nbytes()
        e2e = {"value": round(e2e_us, 2), "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "latency_us": round(lat_us, 2),
               "link_floor_us": round(link_us, 2), "link_frac": round(link_us / e2e_us, 3) if e2e_us > 0 else None,
               "path": "pinned host ids -> ue_rebalance -> pinned host phys + the plan (its 11 arrays in one "
                       "buffer, one copy); steps pipelined on H2D / compute / D2H streams with two buffer sets "
                       "(latency_us: one step alone; link_floor_us: the same H2D and D2H bytes copied at once "
                       "with no kernel, the host link's bound for this leg)"}
        del ids_b, phys_b, plan_b, counts_b, bad_b

    peak, peak_kind = measured_peaks()
    dom = "grad_reduce" if seg[:, 2].sum() >= seg[:, 1].sum() else "sync"
    if dom == "grad_reduce":
        ach = grad_gbs
        per_launch = float(grad_bytes[step_mb].mean())
    else:
        ach = sync_gbs
        per_launch = float(sync_bytes[step_mb].mean())
    roofline = {"kernel": dom, "bound": "hbm", "achieved": round(ach, 1), "peak": peak, "unit": "GB/s",
                "frac": round(ach / peak, 4), "peak_source": f"{peak_kind} copy bandwidth (MEASURED_PEAKS.json hbm_gbs)"
                if peak_kind == "measured" else "fallback 6650 GB/s",
                "traffic": traffic_per_launch(dom, w.name, not args.expert_shape, per_launch),
                "traffic_source": (TRAFFIC.get((dom, w.name)) or {}).get("profile"),
                "algorithmic_bytes_per_launch": per_launch}

    cpu = None
    if dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, ids_host, P, gsize)

    result = {
        "metric": METRIC, "value": round(mean_reb_max, 2), "unit": UNIT, "n_gpus": dist.world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(total_ms_max / args.steps, 4),
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "int32",
        "data": "synthetic: seeded Zipf-popularity Gumbel-top-k routing, random bf16 weights and replica grads",
        "config": workload_config(w, n_mb, dist.world),
        "breakdown_us": {
            "load": round(float(bd[:, 0].mean()), 2), "plan": round(float(bd[:, 1].mean()), 2),
            "reroute": round(float(bd[:, 2].mean()), 2),
            "rebalance_as_separate_calls": round(float(bd.sum(axis=1).mean()), 2),
            "rebalance_p10": round(float(np.percentile(rebalance_us, 10)), 2),
            "rebalance_p50": round(float(np.percentile(rebalance_us, 50)), 2),
            "rebalance_p90": round(float(np.percentile(rebalance_us, 90)), 2),
            "sync": round(sync_us_max, 1), "grad_reduce": round(grad_us_max, 1),
            "launch_floor": round(launch_floor_us, 2),
            "rebalance_graph": None if graph_us is None else round(graph_us, 2),
            "rebalance_dispatch": round(reb_disp_us, 2),
            "rebalance_warm_l2": round(warm_us, 2),
            "dispatch_call": round(disp_call_us, 2),
        },
        "dispatch_layout": {
            "note": "ue_rebalance_dispatch: load + plan + reroute with the per-slot grouping of (t, k) and gates",
            "algorithmic_bytes": 20 * w.L,
            "hbm_floor_us": round(20 * w.L / (peak * 1e9) * 1e6, 2),
        },
        "rebalance_hbm_floor_us": round(rebalance_alg_bytes / (peak * 1e9) * 1e6, 2),
        "sync_gbs": round(sync_gbs, 1), "sync_frac": round(sync_gbs / peak, 4),
        "grad_reduce_gbs": round(grad_gbs, 1), "grad_reduce_frac": round(grad_gbs / peak, 4),
        "frac_of_8000_gbs": {"sync": round(sync_gbs / 8000, 4), "grad_reduce": round(grad_gbs / 8000, 4)},
        "sync_delta": sync_delta,
        "across_gpus_emulated": across_gpus,
        "across_gpus": across_real,
        "plan_variants": plan_variants,
        "imbalance": {
            "before": round(float(np.mean([p["max_before"] / (p["L"] / w.N) for p in per_mb])), 4),
            "after": round(float(np.mean([p["max_after"] / (p["L"] / w.N) for p in per_mb])), 4),
            "slots_ran_out_frac": round(float(np.mean([p["ran_out"] for p in per_mb])), 4),
            "replicated_experts_mean": round(float(np.mean([p["M"] for p in per_mb])), 2),
            "filled_redundant_slots_mean": round(float(np.mean([p["filled"] for p in per_mb])), 2),
        },
        "context_pages": {"rebalance_us": 300, "imbalance_before": "1.30-4.01", "imbalance_after": "1.01-1.04",
                          "hardware": "rack-scale NVL72 / Atlas 900 A3"},
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": KERNELS_PER_STEP * args.steps,
        "clocks": clk,
        "job_microbatches_per_s": round(dist.world * args.steps / (total_ms_max * 1e-3), 2),
        "profiles": profile_status(),
    }
    ctx.close()
    dist.barrier()
    dist.close()
    return result


def across_gpus_real(args, dist, ctx, cfg, w, ids_dev, weights, master, grads, gdt, per_mb, slot_bytes, red, n_mb):
    """The sharded load/plan/reroute, weight sync (relay rounds and direct form)
    and home-GPU gradient reduction on the job's GPUs, each rank one GPU."""
    if w.N % dist.world:
        return {"skipped": f"N={w.N} is not a multiple of {dist.world} GPUs"}
    return run_isolated(dist, lambda grp: _across_gpus(grp, dist, ctx, cfg, w, ids_dev, weights, master, grads,
                                                       gdt, per_mb, slot_bytes, red, n_mb))


def run_isolated(dist, fn, timeout_s: float = 60.0) -> dict:
    """fn(group) on a gloo group of its own with a short timeout: a failure on
    some ranks ends, on every rank, as an exception within the timeout (the
    others' waits in that group run out), reported as {"error": ...}; the
    job's main group is never left waiting.  Every rank calls it."""
    import datetime
    grp = dist.pg.new_group(backend="gloo", timeout=datetime.timedelta(seconds=timeout_s))
    try:
        return fn(grp)
    except Exception as exc:      # reported in the line; the replicas' numbers stand
        return {"error": repr(exc)[:300]}
    finally:
        try:
            dist.pg.destroy_process_group(grp)
        except Exception:
            pass


def _across_gpus(grp, dist, ctx, cfg, w, ids_dev, weights, master, grads, gdt, per_mb, slot_bytes, red, n_mb):
    import torch

    from moe_expert_load_ue_b200 import ue
    from moe_expert_load_ue_b200.peer import PeerBuffers
    from moe_expert_load_ue_b200.shard import DeviceOps, ShardedBalancer
    G, g = dist.world, dist.rank
    # Barriers are host-staged (stream synchronize, then a gloo barrier).
    SG, EG, RG, TG = w.S // G, w.E // G, (w.N // G) * w.R, w.T // G
    dev = weights.device
    bal = ShardedBalancer(cfg, DeviceOps(ctx, cfg, G, g), G=G, g=g, group=grp, device=dev, host_staged=True)
    pw = PeerBuffers(weights[g * SG:(g + 1) * SG], group=grp)
    pg = PeerBuffers(grads[g * RG:(g + 1) * RG], group=grp)
    counts = torch.empty((w.N, w.E), dtype=torch.int32, device=dev)
    plan = ue.Plan(cfg, device=dev)
    phys_l = torch.empty((TG, w.K), dtype=torch.int32, device=dev)
    n_sh = min(n_mb, 4)
    st = torch.cuda.current_stream(dev)
    evs = []
    for k in range(-1, n_sh):                    # one untimed pass first
        mb = max(k, 0)
        bal.rebalance(ids_dev[mb][g * TG:(g + 1) * TG], counts, None, plan, phys_l)
        e = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        e[0].record(st)
        bal.sync(pw.ptrs, slot_bytes, plan, relay=True)
        e[1].record(st)
        bal.sync(pw.ptrs, slot_bytes, plan, relay=False)
        e[2].record(st)
        bal.grad_reduce(master[g * EG:(g + 1) * EG], pg.ptrs, gdt, w.P, plan)
        e[3].record(st)
        if k >= 0:
            evs.append(e)
    torch.cuda.synchronize(dev)
    t = np.array([[e[i].elapsed_time(e[i + 1]) for i in range(3)] for e in evs]) * 1e3
    tt = torch.tensor(list(t.sum(axis=0)), dtype=torch.float64)
    dist.pg.all_reduce(tt, op=dist.pg.ReduceOp.MAX, group=grp)
    tmax = tt.tolist()
    bal.barrier()
    torch.cuda.synchronize(dev)
    pw.close()
    pg.close()
    sync_b = cross_b = grad_b = 0
    gsize = 2 if w.grad_dtype == "bf16" else 4
    for mb in range(n_sh):
        se = per_mb[mb]["slot_expert"]
        for e_ in np.unique(se[red & (se >= 0)]):
            gpus = set((np.nonzero(red & (se == e_))[0] // SG).tolist())
            hg = ((e_ // w.H) * (w.H + w.R)) // SG
            sync_b += len(gpus) * slot_bytes
            cross_b += len(gpus - {hg}) * slot_bytes
        sync_b += int((red & (se >= 0)).sum()) * slot_bytes
        grad_b += per_mb[mb]["M"] * w.P * 8 + per_mb[mb]["filled"] * w.P * gsize
    return {"G": G, "microbatches": n_sh, "relay_rounds": ue.ue_relay_rounds(G),
            "sync_alg_bytes_mean": int(sync_b / n_sh), "nvlink_bytes_mean": int(cross_b / n_sh),
            "sync_relay_us": round(tmax[0] / n_sh, 1), "sync_direct_us": round(tmax[1] / n_sh, 1),
            "grad_reduce_us": round(tmax[2] / n_sh, 1),
            "sync_relay_gbs": round(sync_b / (tmax[0] * 1e-6) / 1e9, 1),
            "sync_direct_gbs": round(sync_b / (tmax[1] * 1e-6) / 1e9, 1),
            "grad_reduce_gbs": round(grad_b / (tmax[2] * 1e-6) / 1e9, 1),
            "nvlink_gbs_relay": round(cross_b / (tmax[0] * 1e-6) / 1e9, 1),
            "note": "each rank one GPU holding its shard; peer tables by CUDA IPC; host-staged barriers "
                    "(stream synchronize + gloo) between relay rounds, inside the times; GB/s = all GPUs' "
                    "algorithmic sync / grad bytes / the slowest rank's time"}


# ---- the CPU oracle, timed on the host cores ------------------------------------

def cpu_baseline(w, ids_host, P, gsize, budget_s: float = 10.0):
    import oracle
    n_mb = len(ids_host)
    t_reb = []
    t0 = time.perf_counter()
    plans = []
    while time.perf_counter() - t0 < 0.6 * budget_s or len(t_reb) < n_mb:
        mb = len(t_reb) % n_mb
        a = time.perf_counter()
        out = oracle.rebalance(ids_host[mb], w.E, w.N, w.R)
        t_reb.append(time.perf_counter() - a)
        if len(plans) < n_mb:
            plans.append(out["plan"])
    # weight sync over a 1 MiB window of every slot; grad reduce over a 64 Ki-element window of every expert
    win = 1 << 20
    Wh = np.random.default_rng(0).integers(0, 256, size=(w.S, win), dtype=np.uint8)
    nb, ts = 0, 0.0
    gw = 1 << 16
    mh = np.random.default_rng(1).standard_normal((w.E, gw), dtype=np.float32)
    gh = (inputs.random_bf16_bits((w.N * w.R, gw), 1e-3, 2) if gsize == 2
          else inputs.random_f32((w.N * w.R, gw), 1e-3, 2))
    gb, tg = 0, 0.0
    t1 = time.perf_counter()
    i = 0
    while time.perf_counter() - t1 < 0.4 * budget_s or i < n_mb:
        pl = plans[i % n_mb]
        a = time.perf_counter()
        oracle.sync(Wh, win, w.E, w.N, w.R, pl["slot_expert"])
        ts += time.perf_counter() - a
        nb += (int(pl["info"][3]) + int(pl["info"][4])) * win
        a = time.perf_counter()
        oracle.grad_reduce(mh, gh, gw, w.E, w.N, w.R, pl)
        tg += time.perf_counter() - a
        gb += int(pl["info"][3]) * gw * 8 + int(pl["info"][4]) * gw * gsize
        i += 1
    return {"value": round(statistics.mean(t_reb) * 1e6, 1), "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": f"{len(t_reb)} full microbatches of the workload (load+plan+reroute); weight sync over a "
                      f"1 MiB window of every slot and grad reduce over a 64 Ki-element window of every "
                      f"expert, {i} plans",
            "sync_gbs": round(nb / ts / 1e9, 2), "grad_reduce_gbs": round(gb / tg / 1e9, 2),
            "threads": "single-threaded C (gcc -O2)", "nproc": os.cpu_count()}


def run_reference(args, dist: Dist):
    """The reference arm: the CPU oracle, timed as it stands on the host cores."""
    if dist.rank != 0:
        return None
    import oracle
    w = workload_of(args, 0)
    n_mb = args.microbatches or w.microbatches
    ids_host = [inputs.topk_ids(w, mb) for mb in range(n_mb)]
    for k in range(args.warmup):
        oracle.rebalance(ids_host[k % n_mb], w.E, w.N, w.R)
    times = []
    for k in range(args.steps):
        a = time.perf_counter()
        oracle.rebalance(ids_host[k % n_mb], w.E, w.N, w.R)
        times.append(time.perf_counter() - a)
    v = round(statistics.mean(times) * 1e6, 1)
    return {
        "impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(statistics.mean(times) * 1e3, 3),
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "int32",
        "data": "synthetic: seeded Zipf-popularity Gumbel-top-k routing",
        "config": workload_config(w, n_mb, args.gpus),
        "cpu_baseline": {"value": v, "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": f"each step one full microbatch (load+plan+reroute), {args.steps} steps"},
        "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }


def run_sweep(args, dist: Dist):
    """Rebalance over the sweep grid: E=256, top-8, R=1 (E + N slots), tokens per
    rank x N x Zipf s; inputs drawn on the device.  One JSON line per point."""
    import torch

    from moe_expert_load_ue_b200 import ue
    torch.cuda.set_device(dist.local_rank)
    dev = torch.device("cuda", dist.local_rank)
    ctx = ue.Context(dist.local_rank)
    stream = torch.cuda.Stream(device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    peak, _ = measured_peaks()
    only = None
    if args.sweep_only:
        only = {(int(a), int(b), float(c)) for a, b, c in (x.split(":") for x in args.sweep_only.split(","))}
    for w in inputs.sweep(seeds=args.sweep_seeds):
        if only is not None and (w.tokens_per_rank, w.N, w.s) not in only:
            continue
        cfg = ue.Config(E=w.E, N=w.N, R=w.R, K=w.K, T=w.T)
        # Inputs drawn and buffers allocated on the stream the kernels run on,
        # and the device drained before timing: no cross-stream reuse of memory.
        with torch.cuda.stream(stream):
            ids = inputs.topk_ids_device(w, 0, dev)
            counts = torch.empty((w.N, w.E), dtype=torch.int32, device=dev)
            bad = torch.empty(w.N, dtype=torch.int32, device=dev)
            plan = ue.Plan(cfg, device=dev)
            phys = torch.empty_like(ids)
        torch.cuda.synchronize(dev)
        times = []
        with torch.cuda.stream(stream):
            for k in range(args.warmup + 10):
                flush.zero_()                       # ids leave L2 between repetitions
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                ue.ue_rebalance(ctx, cfg, ids, counts, bad, plan, phys, stream=stream)
                b.record(stream)
                if k >= args.warmup:
                    times.append((a, b))
        stream.synchronize()
        info = plan["info"].cpu().tolist()
        us = [a.elapsed_time(b) * 1e3 for a, b in times]
        mean = w.L / w.N
        # The plan variants on the same ids: imbalance after and latency.
        variants = {}
        for name, v in VARIANTS.items():
            vt = []
            with torch.cuda.stream(stream):
                for k in range(args.warmup + 5):
                    flush.zero_()
                    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    a.record(stream)
                    ue.ue_rebalance_ex(ctx, cfg, ids, counts, bad, plan, phys, v, stream=stream)
                    b.record(stream)
                    if k >= args.warmup:
                        vt.append((a, b))
            stream.synchronize()
            vi = plan["info"].cpu().tolist()
            variants[name] = {"imbalance_after": round(vi[6] / mean, 4),
                              "gap_bound": round(vi[6] / vi[0] - 1.0, 4) if vi[0] > 0 else None,
                              "rebalance_us_median": round(statistics.median(a.elapsed_time(b) * 1e3 for a, b in vt),
                                                           2)}
        med = statistics.median(us)
        alg = 12 * w.L          # ids read by load and reroute, phys written
        print(json.dumps({"sweep_point": w.name, "tokens_per_rank": w.tokens_per_rank, "N": w.N, "zipf_s": w.s,
                          "seed": w.base_seed, "T": w.T, "rebalance_us_median": round(med, 2),
                          "rebalance_alg_bytes": alg, "rebalance_gbs": round(alg / (med * 1e-6) / 1e9, 1),
                          "rebalance_frac": round(alg / (med * 1e-6) / 1e9 / peak, 4),
                          "imbalance_before": round(info[5] / mean, 4), "imbalance_after": round(info[6] / mean, 4),
                          # max rank load after / Q - 1: Q = ceil(L / N) bounds every plan's busiest
                          # rank from below, so this bounds the plan's gap to the optimum from above
                          "gap_bound": round(info[6] / info[0] - 1.0, 4) if info[0] > 0 else None,
                          "slots_ran_out": bool(info[2] & 1), "replicated_experts": info[3],
                          "filled_redundant_slots": info[4], "plan_variants": variants}), flush=True)
        del ids, phys, plan, counts, bad
        torch.cuda.synchronize(dev)
    del flush
    if only is not None:
        ctx.close()
        return
    # Weight sync and gradient reduction per N at the sweep's expert shape
    # (3 x 2048 x 1024 bf16 weights, fp32 gradients), on the plan of one
    # microbatch of 4096 tokens per rank at Zipf 1.2; events around each call,
    # 10 calls after 3 (every buffer is larger than L2).
    for n in (8, 32, 64, 128, 256):
        w = inputs.Workload(f"sweep-sync-n{n}", E=256, K=8, N=n, R=1, tokens_per_rank=4096, s=1.2,
                            rows=2048, cols=1024, grad_dtype="fp32")
        cfg = ue.Config(E=w.E, N=w.N, R=w.R, K=w.K, T=w.T)
        P, slot_bytes = w.P, 2 * w.P
        with torch.cuda.stream(stream):
            ids = inputs.topk_ids_device(w, 0, dev)
            counts = torch.empty((w.N, w.E), dtype=torch.int32, device=dev)
            plan = ue.Plan(cfg, device=dev)
            ue.ue_rebalance(ctx, cfg, ids, counts, None, plan, torch.empty_like(ids), stream=stream)
            weights = torch.empty((w.S, P), dtype=torch.bfloat16, device=dev).normal_(0.0, 0.02)
            master = torch.empty((w.E, P), dtype=torch.float32, device=dev).normal_(0.0, 1e-3)
            grads = torch.empty((w.N * w.R, P), dtype=torch.float32, device=dev).normal_(0.0, 1e-3)
        stream.synchronize()
        info = plan["info"].cpu().tolist()
        sync_b = (info[3] + info[4]) * slot_bytes
        grad_b = info[3] * P * 8 + info[4] * P * 4
        ts, tg = [], []
        with torch.cuda.stream(stream):
            for k in range(13):
                a, b, c = (torch.cuda.Event(enable_timing=True) for _ in range(3))
                a.record(stream)
                ue.ue_sync(ctx, cfg, weights, slot_bytes, plan, stream=stream)
                b.record(stream)
                ue.ue_grad_reduce(ctx, cfg, master, grads, P, plan, stream=stream)
                c.record(stream)
                if k >= 3:
                    ts.append((a, b))
                    tg.append((b, c))
        stream.synchronize()
        su = statistics.median(a.elapsed_time(b) for a, b in ts) * 1e3
        gu = statistics.median(a.elapsed_time(b) for a, b in tg) * 1e3
        print(json.dumps({"sweep_sync_grad": w.name, "N": n, "slot_bytes": slot_bytes, "replicated_experts": info[3],
                          "filled_redundant_slots": info[4], "sync_bytes": sync_b, "sync_us_median": round(su, 1),
                          "sync_gbs": round(sync_b / (su * 1e-6) / 1e9, 1),
                          "sync_frac": round(sync_b / (su * 1e-6) / 1e9 / peak, 4),
                          "grad_reduce_bytes": grad_b, "grad_reduce_us_median": round(gu, 1),
                          "grad_reduce_gbs": round(grad_b / (gu * 1e-6) / 1e9, 1),
                          "grad_reduce_frac": round(grad_b / (gu * 1e-6) / 1e9 / peak, 4)}), flush=True)
        del ids, counts, plan, weights, master, grads
        torch.cuda.synchronize(dev)
    ctx.close()


def main(argv=None):
    args = parse_args(argv)
    dist = Dist()
    if args.sweep:
        run_sweep(args, dist)
        return
    if args.impl == "reference":
        res = run_reference(args, dist)
    else:
        res = run_ours(args, dist)
    if res is not None and dist.rank == 0:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
