"""Benchmark: one SCOPE attention call (scope_plan + scope_attn) per step.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl scope|reference] [--workload NAME]

A step is one pass of the whole hot path -- 3D-RoPE, key-subspace and query
k-means, lookup tables, hybrid Top-p/Top-k with the online per-head Top-k,
list emission, sparse attention -- over one synthetic batch of the
HunyuanVideo-720p-shaped workload (B=1, H=24, N=118800, d=128, bf16), inputs
resident in HBM (2.2 GB of Q/K/V, far above the 126 MB L2, so no flush is
needed between steps).  With N GPUs each rank runs its own call (weak
scaling, no collective on the data path); `value` is ms per call of the whole
job: the max-over-ranks time of K steps divided by the K*N calls made.

--impl reference times the fp64 CPU oracle on a bounded sample of the same
workload (rank 0 only) and prints its line with "impl": "reference".
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from cluster_guided_sparse_b200 import synth  # noqa: E402

METRIC = "ms per attention call (scope_plan + scope_attn) at the 720p shape"


# --------------------------------------------------------------------------- helpers
def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return p["hbm_gbs"], p["bf16_tflops"], p.get("bf16_tflops_sustained", p["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


def attn_traffic(heads: int):
    """DRAM bytes of one sparse-attention launch, from the committed ncu capture
    (profiles/attn_tc_traffic.json) scaled from its heads to `heads`; None if the
    kernel source changed since the capture."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", "attn_tc_traffic.json")) as f:
            rec = json.load(f)
        with open(os.path.join(ROOT, "cluster_guided_sparse_b200", "csrc", "attn_tc.cu"), "rb") as f:
            sha = hashlib.sha256(f.read()).hexdigest()
    except Exception:
        return None
    if sha != rec.get("kernel_source_sha256"):
        return None
    return rec["sparse_dram_bytes_per_launch_captured"] * heads / rec["captured_heads"]


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled while the timed region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device: int):
        self.dev = device
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            uuid = str(torch.cuda.get_device_properties(self.dev).uuid)
            sel = ["-i", uuid if uuid.startswith("GPU-") else "GPU-" + uuid]
            self.proc = subprocess.Popen(["nvidia-smi", *sel, f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for nm, val in zip(names, parts[3:7]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """Max of a per-rank scalar over all ranks (a device tensor under NCCL, a
    host tensor under gloo)."""
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_ms_per_call(rank_ms: float, steps: int, world: int) -> float:
    """Whole-job ms per call: every rank made `steps` calls inside its timed
    region; the job's time is the slowest rank's."""
    return max_over_ranks(rank_ms, world) / (steps * world)


def tile_flops(sizes: torch.Tensor, n: torch.Tensor, d: int, bm: int = 128, bn: int = 128,
               item_rows: int = 256) -> float:
    """Flops of the tiles the attention kernel issues: each cluster's queries
    in work items of up to `item_rows`, each item's rows padded to `bm`-row Q
    tiles, its key list padded to `bn`-key tiles (Q.K^T plus P.V)."""
    s = sizes.to(torch.int64)
    full, rem = s // item_rows, s % item_rows
    qtiles = full * (item_rows // bm) + (rem + bm - 1) // bm
    ktiles = (n.to(torch.int64) + bn - 1) // bn
    return 4.0 * d * bm * bn * float((qtiles * ktiles).sum())


# --------------------------------------------------------------------------- oracle sample
def oracle_sample(w, budget_rows=1024, clusters=2, queries=8):
    """Times the fp64 oracle on a bounded slice of head 0 of workload `w` and
    extrapolates to one whole call (all heads, all rows, all clusters).
    Returns (ms per call extrapolated, sample description, seconds spent)."""
    import oracle

    t0 = time.perf_counter()
    qh, kh, vh, _ = synth.make_head(w, 0, 0, 0, synth.grid_field(w))
    q, k, v = (oracle._round_bf16(x.astype(np.float64)) for x in (qh, kh, vh))
    N, D, I = w.N, w.D, w.iters
    rng = np.random.default_rng(0)
    rows = np.sort(rng.choice(N, min(budget_rows, N), replace=False))
    tm = {}
    s = time.perf_counter()
    qr = oracle.rope3d(q, w.grid, w.d_split, w.theta)
    kr = oracle.rope3d(k, w.grid, w.d_split, w.theta)
    tm["rope"] = time.perf_counter() - s
    offs = np.cumsum((0,) + tuple(w.d_split))
    # key-subspace and query assignment: per-row cost on the sampled rows
    t_assign = 0.0
    kcent = []
    for si in range(3):
        a, b = int(offs[si]), int(offs[si + 1])
        C = w.c_sub[si]
        cent = kr[np.arange(C) * (N // C), a:b]
        s = time.perf_counter()
        lab = oracle.kmeans_assign(kr[rows, a:b], cent)
        t_assign += (time.perf_counter() - s) * N / len(rows) * (I + 1)
        full = oracle.kmeans_assign(kr[:, a:b], cent) if b > a else np.zeros(N, np.int32)
        s = time.perf_counter()
        cent, _ = oracle.kmeans_update(kr[:, a:b], full, cent)
        t_assign += (time.perf_counter() - s) * I
        kcent.append((cent, full))
        del lab
    qcent = qr[np.arange(w.c_q) * (N // w.c_q)]
    s = time.perf_counter()
    oracle.kmeans_assign(qr[rows], qcent)
    t_assign += (time.perf_counter() - s) * N / len(rows) * (I + 1)
    qlab = oracle.kmeans_assign(qr, qcent)
    s = time.perf_counter()
    qcent, _ = oracle.kmeans_update(qr, qlab, qcent)
    t_assign += (time.perf_counter() - s) * I
    tm["kmeans"] = t_assign
    s = time.perf_counter()
    luts = [oracle.lut(qcent[:, int(offs[si]):int(offs[si + 1])], kcent[si][0]) for si in range(3)]
    tm["lut"] = time.perf_counter() - s
    scale = 1.0 / np.sqrt(D)
    s = time.perf_counter()
    lists = []
    for c in range(clusters):
        sc = oracle.proxy_scores([L[c] for L in luts], [kc[1] for kc in kcent])
        r = oracle.retained_count(sc, w.top_p, w.k_min, scale)
        lists.append(oracle.emit(sc, r))
    tm["select"] = (time.perf_counter() - s) * w.c_q / clusters
    s = time.perf_counter()
    for i in range(queries):
        oracle.attention_rows(qr[i:i + 1], kr, v, lists[i % clusters], scale)
    tm["attn"] = (time.perf_counter() - s) * N / queries
    per_head = sum(tm.values())
    ms = per_head * w.H * w.B * 1e3
    desc = (f"head 0 of {w.name}: full RoPE, k-means assign on {len(rows)} rows x (iters+1) and full updates, "
            f"LUT, selection for {clusters} clusters, attention for {queries} queries; extrapolated x rows, "
            f"x clusters, x queries, x {w.B * w.H} heads (1 thread)")
    return ms, desc, time.perf_counter() - t0


# --------------------------------------------------------------------------- arms
def run_reference(args, world, rank):
    if rank != 0:
        return
    w = synth.WORKLOADS[args.workload]
    vals = []
    spent = 0.0
    for i in range(args.warmup + args.steps):
        ms, desc, sec = oracle_sample(w, budget_rows=256, clusters=1, queries=4)
        spent += sec
        if i >= args.warmup:
            vals.append(ms)
    val = statistics.median(vals)
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": "ms", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": val, "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "sample": "bounded oracle sample per step, extrapolated"},
            "cpu_baseline": {"value": val, "unit": "ms", "cores": 1, "kind": "oracle", "sample": desc},
            "e2e": {"value": val, "unit": "ms", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_scope(args, world, rank, local):
    import cluster_guided_sparse_b200 as scope

    w = synth.WORKLOADS[args.workload]
    dev = torch.device("cuda", local if world > 1 else 0)
    q, k, v = synth.make_inputs(w)
    qh, kh, vh = (t.pin_memory() for t in (q, k, v))
    qd, kd, vd = (t.to(dev) for t in (q, k, v))
    params, grid = scope.make_params(w)
    ws = torch.empty(scope.workspace_bytes(qd, params, grid), dtype=torch.uint8, device=dev)
    o = torch.empty(qd.shape, dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        pl = scope.plan(qd, kd, params, grid, workspace=ws)
        scope.attn(qd, kd, vd, pl, out=o)
        return pl

    for _ in range(args.warmup):
        pl = step()
    torch.cuda.synchronize()
    pl.sync_status()

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    L0 = scope.lib().scope_kernel_launches()
    with ClockSampler(dev.index) as clocks:
        barrier(world)
        torch.cuda.synchronize()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for i in range(args.steps):
            ev[i][0].record(stream)
            pl = scope.plan(qd, kd, params, grid, workspace=ws)
            ev[i][1].record(stream)
            scope.attn(qd, kd, vd, pl, out=o)
            ev[i][2].record(stream)
        t1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
    launches = scope.lib().scope_kernel_launches() - L0
    ms_per_call = job_ms_per_call(t0.elapsed_time(t1), args.steps, world)
    total_ms = ms_per_call * args.steps * world
    plan_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in ev)
    attn_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in ev)
    call_median_ms = statistics.median(e[0].elapsed_time(e[2]) for e in ev)

    # algorithmic attention flops of one launch: 4 d sum_c |c| n_c
    sizes = pl.view("q_sizes").to(torch.int64)
    n = pl.view("n").to(torch.int64)
    pairs = int((sizes * n).sum())
    attn_flops = 4.0 * w.D * pairs
    density = pairs / (w.B * w.H * float(w.N) ** 2)
    hbm, bf16, bf16_sus, src = peaks()
    achieved = attn_flops / (attn_ms * 1e-3) / 1e12
    tile_tf = tile_flops(sizes.flatten(), n.flatten(), w.D) / (attn_ms * 1e-3) / 1e12

    # this build's dense attention (RoPE + all keys) at the same shape, for context
    od = torch.empty_like(o)
    dense = []
    for i in range(1 + args.steps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        scope.dense_attn(qd, kd, vd, params, grid, out=od)
        b.record(stream)
        torch.cuda.synchronize()
        if i > 0:
            dense.append(a.elapsed_time(b))
    dense_ms = statistics.mean(dense)
    del od

    # end to end through the public API with host buffers: Q and K go first
    # (scope_plan reads them); V is only read by scope_attn, so its copy runs
    # on a side stream while the plan computes.
    e2e = []
    oh = torch.empty(qd.shape, dtype=torch.bfloat16).pin_memory()
    side = torch.cuda.Stream(dev)
    for i in range(args.warmup + args.steps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        qk_in, v_in = torch.cuda.Event(), torch.cuda.Event()
        barrier(world)
        torch.cuda.synchronize()
        a.record(stream)
        qd.copy_(qh, non_blocking=True)
        kd.copy_(kh, non_blocking=True)
        qk_in.record(stream)
        side.wait_event(qk_in)
        with torch.cuda.stream(side):
            vd.copy_(vh, non_blocking=True)
            v_in.record(side)
        pl = scope.plan(qd, kd, params, grid, workspace=ws)
        stream.wait_event(v_in)
        scope.attn(qd, kd, vd, pl, out=o)
        oh.copy_(o, non_blocking=True)
        b.record(stream)
        torch.cuda.synchronize()
        if i >= args.warmup:
            e2e.append(a.elapsed_time(b))
    e2e_ms = max_over_ranks(statistics.mean(e2e), world) / world
    h2d = sum(t.numel() * t.element_size() for t in (qh, kh, vh))
    d2h = oh.numel() * oh.element_size()

    if rank != 0:
        return
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        ms, desc, _ = oracle_sample(w)
        cpu = {"value": ms, "unit": "ms", "cores": 1, "kind": "oracle", "sample": desc}
    eff = w.dense_flops() / (ms_per_call * 1e-3) / 1e12
    line = {
        "metric": METRIC, "value": ms_per_call, "unit": "ms", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "global_batch": w.B * world, "seq_len": w.N, "heads": w.H,
                   "head_dim": w.D, "top_p": w.top_p, "online_topk": bool(w.online_topk),
                   "l2": "inputs 2.2 GB >> 126 MB L2, no flush", "parallelism": f"replicas x{world}"},
        "effective_tflops": eff, "plan_ms": plan_ms, "attn_ms": attn_ms, "call_median_ms": call_median_ms,
        "density": density, "tile_tflops": tile_tf, "tile_frac_of_sustained": tile_tf / bf16_sus,
        "own_dense_ms": dense_ms, "speedup_vs_own_dense": dense_ms / ms_per_call,
        "roofline": {"kernel": "sparse attention (scope_attn)", "bound": "tensor", "achieved": achieved,
                     "peak": bf16_sus, "unit": "TFLOP/s", "frac": achieved / bf16_sus,
                     "traffic": attn_traffic(w.B * w.H),
                     "peak_source": f"{src} bf16 sustained"},
        "e2e": {"value": e2e_ms, "unit": "ms", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": launches,
        "clocks": clocks.summary(),
        "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="scope", choices=["scope", "reference"])
    ap.add_argument("--workload", default="hunyuan720p", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        run_reference(args, world, rank)
        return
    world, rank, local = dist_setup(args.gpus)
    try:
        run_scope(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
