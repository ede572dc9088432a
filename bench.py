#!/usr/bin/env python
"""Benchmark of the routed-expert MoE layer with intra-expert activation sparsity.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload olmoe] [--T 16] [--sparsity 0.9] [--sweep full|quick|none]

One step is one forward of the whole layer (router + bucketing, gate
projection, threshold mask and compaction, gathered up/down projection,
shared experts, combine) over one batch of T synthetic tokens already
resident in HBM.  The default workload is the OLMoE-shaped decode layer
(d_model 2048, 64 experts, d_ff 1024, top-8, no shared expert) at T = 16 with
tau calibrated on the GPU for 90% sparsity.  L2 is flushed (a write of twice
its size) before every timed step, outside the step's CUDA events.

Prints ONE JSON line on rank 0.  Under torchrun each rank runs an independent
replica of the layer on its own GPU ("replicas only": the layer has no
exchange step); the step time is the max over ranks.

The JSON line's ``sweep`` holds one row per (workload, batch size, sparsity):
the sparse path, the dense path and AUTO each timed the same way, with the
expert kernel's roofline fraction and AUTO's choice.  It covers the tiny
layer, the OLMoE-shaped layer at T = 1, 4, 16, 64, the DeepSeek-V2-Lite-shaped
layer at T = 1, 8, 32, 128 and sparsity 0/50/80/90/95 %, the large layer at
T = 1, 16, 64 and a 2 % keep rate, and the crossover sweep T = 1 ... 4096.

``--impl reference`` times the CPU oracle (the plain fp64 definition of the
layer) on the host cores instead -- rank 0 only -- on the same inputs (drawn
on the GPU when there is one, as the GPU arm does, then copied to the host).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, HERE)

METRIC = "routed-MoE layer tokens/s and HBM GB/s (% roofline) at 90% intra-expert sparsity"
FALLBACK_HBM_GBS = 6650.0
WORKLOAD_TEXT = {
    "olmoe": "OLMoE-shaped decode layer: d_model=2048, 64 routed SwiGLU experts, d_ff=1024, "
             "top-8 softmax router, no shared expert, bf16 weights ~N(0,1/fan_in)",
    "dsv2lite": "DeepSeek-V2-Lite-shaped decode layer: d_model=2048, 64 routed experts d_ff=1408, "
                "top-6, 2 dense shared experts d_ff=1408",
    "large": "large sparse-routed decode layer: d_model=4096, 256 routed experts d_ff=1024, top-8, "
             "1 dense shared expert d_ff=1024 (6.44 GB of expert weights)",
    "tiny": "tiny MoE layer: d_model=256, 8 experts d_ff=512, top-2, 1 shared expert",
    "crossover": "OLMoE shapes for the sparse/dense crossover sweep",
}


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=100)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default="olmoe")
    p.add_argument("--T", type=int, default=16)
    p.add_argument("--sparsity", type=float, default=0.9)
    p.add_argument("--path", choices=["auto", "sparse", "dense"], default="auto")
    p.add_argument("--router", choices=["fused", "one_launch", "kernel"], default="fused",
                   help="decode batches: route inside the expert kernel (default), also combine there "
                        "(one launch), or route with the router kernel")
    p.add_argument("--budget", type=int, default=-1,
                   help="per-pair rank budget for the timed layer (keep each routed pair's r best neurons); "
                        "-1: the threshold at --sparsity")
    p.add_argument("--sweep", choices=["full", "quick", "none"], default="full")
    p.add_argument("--no-sweep", action="store_true", help="same as --sweep none")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-seconds", type=float, default=10.0)
    return p.parse_args()


def measured_peaks():
    try:
        with open(os.path.join(HERE, "MEASURED_PEAKS.json")) as fh:
            return json.load(fh), "measured"
    except (OSError, ValueError):
        return {"hbm_gbs": FALLBACK_HBM_GBS}, "fallback"


def recorded_traffic(kernel, workload_key):
    """DRAM bytes per launch from a committed ncu summary, if its source hash still matches."""
    path = os.path.join(HERE, "profiles", "dram_traffic.txt")
    try:
        lines = open(path).read().splitlines()
    except OSError:
        return None
    want_sha = kernel_source_sha()
    for ln in lines:
        parts = ln.split()
        if len(parts) == 4 and parts[0] == kernel and parts[1] == workload_key and parts[2] == want_sha:
            return float(parts[3])
    return None


def kernel_source_sha():
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(HERE, "intra_expert_activation_router_b200", "csrc")
    for fn in sorted(os.listdir(csrc)):
        if fn.endswith((".cu", ".cuh", ".h")):
            h.update(open(os.path.join(csrc, fn), "rb").read())
    return h.hexdigest()[:12]


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(self.gpu_id)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for ln in self.proc.stdout:
            self.lines.append(ln.strip())

    def __exit__(self, *exc):
        if self.proc:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.t.join(timeout=2)

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def gpu_uuid(dev):
    import torch
    try:
        u = str(torch.cuda.get_device_properties(dev).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:  # noqa: BLE001
        return str(dev)


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(value, device=None):
    """The largest of each rank's `value` over the default process group
    (the value itself when there is none or it has one rank)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(world, units_per_rank, seconds):
    """Units all ranks processed per second of the slowest rank (weak scaling)."""
    return world * units_per_rank / seconds


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def bench_config(args, world):
    """The workload description both arms print (identical dicts)."""
    cfg = {"workload": WORKLOAD_TEXT.get(args.workload, args.workload), "T": args.T,
           "sparsity": args.sparsity, "parallelism": f"replicas{world}",
           "l2": "flushed before every timed step (2x L2 written, then read back, outside the step events)"}
    if args.budget >= 0:
        cfg["rank_budget"] = args.budget   # each routed pair keeps its `budget` best neurons; no threshold
    return cfg


def draw_inputs(shape, T, device):
    """The workload's weights and batch, drawn on `device` from the seeded
    generators (the GPU arm draws on its GPU; the reference arm draws the
    same values there too when a GPU is present, then copies them)."""
    import moe_inputs as mi
    return mi.make_weights(shape, device=device), mi.make_x(shape, T, device=device)


def oracle_step(o, inputs, shape, tau, budget, nthreads):
    """One forward of the CPU oracle: the threshold tau, or the per-pair rank
    budget when budget >= 0."""
    if budget >= 0:
        return o.forward_budget(**inputs, top_k=shape.top_k, budget=budget, nthreads=nthreads)
    return o.forward(**inputs, top_k=shape.top_k, tau=tau, want_scores=False, nthreads=nthreads)


def oracle_time_sample(shape, W_host, x_host, tau, target_s, nthreads, budget=-1):
    """The CPU oracle at threshold tau (or the rank budget) on repeats of the
    batch for about target_s seconds (rank 0, N = 1).  Returns (tokens/s,
    repeats, seconds)."""
    import oracle
    o = oracle.Oracle()
    inputs = oracle.layer_inputs(W_host, x_host)
    T = x_host.shape[0]
    t0 = time.perf_counter()
    oracle_step(o, inputs, shape, tau, budget, nthreads)
    one = time.perf_counter() - t0
    reps = max(1, min(500, int(math.ceil(target_s / max(one, 1e-6)))))
    t0 = time.perf_counter()
    for _ in range(reps):
        oracle_step(o, inputs, shape, tau, budget, nthreads)
    el = time.perf_counter() - t0
    return reps * T / el, reps, el


def run_reference(args):
    world, rank, local = dist_setup()
    if rank != 0:
        return
    import torch
    import moe_inputs as mi
    import oracle
    shape = mi.SHAPES[args.workload]
    gen_dev = "cuda" if torch.cuda.is_available() else "cpu"
    W, x = draw_inputs(shape, args.T, gen_dev)
    W, x = W.to("cpu"), x.cpu()
    o = oracle.Oracle()
    inputs = oracle.layer_inputs(W, x)
    cores = cpu_cores()
    # tau of the batch, then size each step's token sample so the run stays short
    r = o.forward(**inputs, top_k=shape.top_k, tau=math.inf, nthreads=cores)
    tau = o.calibrate_tau(r.score, args.sparsity)
    t0 = time.perf_counter()
    oracle_step(o, inputs, shape, tau, args.budget, cores)
    full = time.perf_counter() - t0
    budget = 150.0
    n_tok = args.T
    if (args.steps + args.warmup) * full > budget:
        n_tok = max(1, int(args.T * budget / ((args.steps + args.warmup) * full)))
    sub = dict(inputs)
    sub["x"] = inputs["x"][:n_tok]
    for _ in range(args.warmup):
        oracle_step(o, sub, shape, tau, args.budget, cores)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle_step(o, sub, shape, tau, args.budget, cores)
        times.append(time.perf_counter() - t0)
    ms = 1000 * statistics.mean(times)
    value = n_tok / (ms / 1000)
    sample = (f"{n_tok} of the {args.T} tokens per step, {args.steps} steps; inputs drawn on "
              f"{'the GPU' if gen_dev == 'cuda' else 'the CPU'} and copied to the host")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": bench_config(args, world), "tau": tau,
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def l2_flush(buf):
    """Write a 2x-L2 buffer, then read it back, so L2 ends up full of clean
    lines: the next step neither hits in L2 nor pays for write-backs."""
    buf.zero_()
    buf.sum()


def time_steps(layer, x, tau, out, flush, steps, graph=True):
    """Per-step CUDA-event timing with an L2 flush before each step (outside the events).

    graph=True (the default): the K steps -- flush, start event, forward, end
    event -- are captured into one CUDA graph and replayed once, so the host's
    enqueue cost cannot leave the GPU idle inside a step; the device does
    exactly the same work.  A second graph of the same K steps also records
    the library's launch events (before the first kernel, before the expert
    kernel, after the last kernel) for the per-kernel split; each event node
    adds about a microsecond of its own, so the step times come from the first
    graph, which has only the two events per step.  graph=False enqueues the
    steps one by one from Python (eager), with the launch events.

    Returns (step_ms, router_ms, expert_ms) per step."""
    import torch
    from intra_expert_activation_router_b200 import moe_set_launch_events

    def ev():
        return torch.cuda.Event(enable_timing=True, external=True)

    st = torch.cuda.current_stream()

    def run(with_kernel_events):
        starts = [ev() for _ in range(steps)]
        ends = [ev() for _ in range(steps)]
        kev = [[ev() for _ in range(3)] for _ in range(steps)] if with_kernel_events else None
        for e in starts + ends + [e for trio in (kev or []) for e in trio]:
            e.record(st)   # create the CUDA events before the graph (or the library) records them
        torch.cuda.synchronize()

        def body():
            for i in range(steps):
                l2_flush(flush)
                starts[i].record()
                if kev:
                    moe_set_launch_events(layer.h, kev[i])
                layer.forward(x, tau, out=out)
                ends[i].record()
            if kev:
                moe_set_launch_events(layer.h, None)

        if graph:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                body()
            torch.cuda.synchronize()
            g.replay()
            torch.cuda.synchronize()
            del g
        else:
            body()
            torch.cuda.synchronize()
        step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
        if not kev:
            return step_ms, None, None
        return step_ms, [t[0].elapsed_time(t[1]) for t in kev], [t[1].elapsed_time(t[2]) for t in kev]

    if not graph:
        return run(True)
    step_ms, _, _ = run(False)
    _, router_ms, expert_ms = run(True)
    return step_ms, router_ms, expert_ms


# (workload, batch sizes, sparsities) of the sweep; "quick" keeps one point per workload
SWEEP_FULL = [
    ("tiny", (16,), (0.9,)),
    ("olmoe", (1, 4, 16, 64), (0.9,)),
    ("dsv2lite", (1, 8, 32, 128), (0.0, 0.5, 0.8, 0.9, 0.95)),
    ("large", (1, 16, 64), (0.98,)),
    ("crossover", (1, 2, 4, 8, 16, 24, 32, 48, 64, 128, 256, 512, 1024, 2048, 4096), (0.9,)),
]
SWEEP_QUICK = [("tiny", (16,), (0.9,)), ("olmoe", (1, 16), (0.9,)), ("dsv2lite", (8,), (0.9,)),
               ("large", (1,), (0.98,))]


def sweep_rows(dev, kind, peak, flush, steps=20):
    """One row per (workload, T, sparsity): sparse, dense and AUTO timed alike."""
    import torch
    import moe_inputs as mi
    import intra_expert_activation_router_b200 as m
    rows = []
    plan = SWEEP_FULL if kind == "full" else SWEEP_QUICK
    for name, Ts, qs in plan:
        shape = mi.SHAPES[name]
        W = mi.make_weights(shape, device=dev)
        layer = m.MoESparseLayer.from_weights(W, shape.top_k, max_tokens=max(Ts))
        del W
        x_max = mi.make_x(shape, max(Ts), device=dev)
        for q in qs:
            # AUTO's switch point for this layer and sparsity, measured on the device
            t_star = layer.tune_t_star(x_max, layer.calibrate_tau(x_max, q))
            for T in Ts:
                x = mi.make_x(shape, T, device=dev)
                out = torch.empty_like(x)
                tau = layer.calibrate_tau(x, q)
                row = {"workload": name, "T": T, "sparsity": q, "tau": tau, "t_star": t_star}
                for mode, path in (("sparse", m.MOE_PATH_SPARSE), ("dense", m.MOE_PATH_DENSE),
                                   ("auto", m.MOE_PATH_AUTO)):
                    try:
                        layer.set_path(path)
                    except m.MoeError:
                        row[f"{mode}_us"] = None
                        continue
                    for _ in range(3):
                        layer.forward(x, tau, out=out)
                    sm_, rm_, em_ = time_steps(layer, x, tau, out, flush, steps)
                    st = layer.stats()
                    if st["device_error"]:
                        row[f"{mode}_device_error"] = st["device_error"]
                    used = "sparse" if st["path"] == m.MOE_PATH_SPARSE else "dense"
                    b = st["alg_bytes"] if used == "sparse" else st["dense_bytes"]
                    us = 1000 * statistics.mean(sm_)
                    kus = 1000 * statistics.mean(em_)
                    kb = b - (0 if st["fused_router"] else shape.n_experts * shape.d_model * 2 + T * shape.d_model * 2)
                    row[f"{mode}_us"] = us
                    row[f"{mode}_tokens_per_s"] = T / (us * 1e-6)
                    if mode == "auto":
                        row["auto_path"] = used
                        continue
                    row[f"{mode}_kernels_us"] = kus
                    row[f"{mode}_alg_bytes"] = b
                    row[f"{mode}_gbs"] = b / (us * 1e-6) / 1e9
                    row[f"{mode}_kernel_frac"] = kb / (kus * 1e-6) / 1e9 / peak
                    if mode == "sparse":
                        row["n_active"], row["n_union"], row["n_touched"] = (
                            st["n_active"], st["n_union"], st["n_touched"])
                best = min(v for v in (row.get("sparse_us"), row.get("dense_us")) if v is not None)
                row["auto_over_best"] = row["auto_us"] / best
                layer.set_path(m.MOE_PATH_AUTO)
                rows.append(row)
                log(json.dumps({k: (round(v, 2) if isinstance(v, float) else v) for k, v in row.items()}))
        layer.close()
        torch.cuda.empty_cache()
    return rows


def launch_mode_rows(dev, flush, steps=20):
    """Decode batches of the OLMoE-shaped layer in the three launch
    structures: router kernel + expert kernel + conversion (3 launches),
    routing inside the expert kernel (2), routing and combine inside (1)."""
    import torch
    import moe_inputs as mi
    import intra_expert_activation_router_b200 as m
    shape = mi.SHAPES["olmoe"]
    W = mi.make_weights(shape, device=dev)
    layer = m.MoESparseLayer.from_weights(W, shape.top_k, max_tokens=16)
    del W
    layer.set_path(m.MOE_PATH_SPARSE)
    rows = []
    for T in (1, 4, 16):
        x = mi.make_x(shape, T, device=dev)
        out = torch.empty_like(x)
        tau = layer.calibrate_tau(x, 0.9)
        row = {"workload": "olmoe", "T": T, "sparsity": 0.9}
        for name, fused, one in (("launches3_us", False, False), ("launches2_us", True, False),
                                 ("launches1_us", True, True)):
            layer.set_fused_router(fused, one_launch=one)
            for _ in range(3):
                layer.forward(x, tau, out=out)
            sm_, _, _ = time_steps(layer, x, tau, out, flush, steps)
            row[name] = 1000 * statistics.mean(sm_)
            if layer.stats()["device_error"]:
                row[name + "_device_error"] = True
        rows.append(row)
        log(json.dumps({k: (round(v, 2) if isinstance(v, float) else v) for k, v in row.items()}))
    layer.close()
    torch.cuda.empty_cache()
    return rows


def rank_budget_rows(dev, flush, steps=20):
    """The per-pair rank budget (each routed pair keeps its r = 10 % of d_ff
    highest-scoring neurons) beside the threshold at 90 % sparsity, on the
    OLMoE-shaped layer's decode batches.  The budget runs two sparse passes
    (the routed gates, then the masked up/down) around a per-pair selection."""
    import torch
    import moe_inputs as mi
    import intra_expert_activation_router_b200 as m
    shape = mi.SHAPES["olmoe"]
    W = mi.make_weights(shape, device=dev)
    layer = m.MoESparseLayer.from_weights(W, shape.top_k, max_tokens=16)
    del W
    layer.set_path(m.MOE_PATH_SPARSE)
    r = shape.d_ff // 10
    rows = []
    for T in (1, 4, 16):
        x = mi.make_x(shape, T, device=dev)
        out = torch.empty_like(x)
        tau = layer.calibrate_tau(x, 0.9)
        row = {"workload": "olmoe", "T": T, "budget": r, "tau": tau}
        for name, budget in (("threshold", -1), ("budget", r)):
            layer.set_rank_budget(budget)
            for _ in range(3):
                layer.forward(x, tau, out=out)
            sm_, _, _ = time_steps(layer, x, tau, out, flush, steps)
            st = layer.stats()
            row[name + "_us"] = 1000 * statistics.mean(sm_)
            row[name + "_alg_bytes"] = st["alg_bytes"]
            row[name + "_n_active"] = st["n_active"]
            if st["device_error"]:
                row[name + "_device_error"] = st["device_error"]
        layer.set_rank_budget(-1)
        rows.append(row)
        log(json.dumps({k: (round(v, 2) if isinstance(v, float) else v) for k, v in row.items()}))
    layer.close()
    torch.cuda.empty_cache()
    return rows


def capacity_rows(dev, flush, steps=20):
    """Capacity-aware token drop (each expert keeps at most ceil(gamma T k / E)
    pairs, the best by routing weight) beside the plain layer, on the
    OLMoE-shaped layer at 90 % sparsity, both branches where each runs."""
    import torch
    import moe_inputs as mi
    import intra_expert_activation_router_b200 as m
    shape = mi.SHAPES["olmoe"]
    W = mi.make_weights(shape, device=dev)
    layer = m.MoESparseLayer.from_weights(W, shape.top_k, max_tokens=512)
    del W
    rows = []
    for T, path in ((16, m.MOE_PATH_SPARSE), (64, m.MOE_PATH_DENSE), (512, m.MOE_PATH_DENSE)):
        x = mi.make_x(shape, T, device=dev)
        out = torch.empty_like(x)
        tau = layer.calibrate_tau(x, 0.9)
        layer.set_path(path)
        row = {"workload": "olmoe", "T": T, "path": "sparse" if path == m.MOE_PATH_SPARSE else "dense"}
        for name, gamma in (("plain", 0.0), ("gamma1", 1.0), ("gamma1_25", 1.25)):
            layer.set_capacity(gamma)
            for _ in range(3):
                layer.forward(x, tau, out=out)
            sm_, _, _ = time_steps(layer, x, tau, out, flush, steps)
            st = layer.stats()
            row[name + "_us"] = 1000 * statistics.mean(sm_)
            row[name + "_capacity"] = st["capacity"]
            row[name + "_alg_bytes"] = st["alg_bytes"] if row["path"] == "sparse" else st["dense_bytes"]
            if st["device_error"]:
                row[name + "_device_error"] = st["device_error"]
        layer.set_capacity(0.0)
        layer.set_path(m.MOE_PATH_AUTO)
        rows.append(row)
        log(json.dumps({k: (round(v, 2) if isinstance(v, float) else v) for k, v in row.items()}))
    layer.close()
    torch.cuda.empty_cache()
    return rows


def deterministic_rows(dev, flush, steps=20):
    """The deterministic combine (each contribution in a row of its own,
    summed in one fixed order) beside the default fp32-atomic one, on the
    OLMoE-shaped layer at 90 % sparsity: decode batches on the sparse branch
    and a larger one on the dense branch."""
    import torch
    import moe_inputs as mi
    import intra_expert_activation_router_b200 as m
    shape = mi.SHAPES["olmoe"]
    W = mi.make_weights(shape, device=dev)
    layer = m.MoESparseLayer.from_weights(W, shape.top_k, max_tokens=256)
    del W
    rows = []
    for T, path in ((1, m.MOE_PATH_SPARSE), (16, m.MOE_PATH_SPARSE), (256, m.MOE_PATH_DENSE)):
        x = mi.make_x(shape, T, device=dev)
        out = torch.empty_like(x)
        tau = layer.calibrate_tau(x, 0.9)
        layer.set_path(path)
        row = {"workload": "olmoe", "T": T, "path": "sparse" if path == m.MOE_PATH_SPARSE else "dense"}
        for name, det in (("atomic", False), ("deterministic", True)):
            layer.set_deterministic(det)
            for _ in range(3):
                layer.forward(x, tau, out=out)
            sm_, _, _ = time_steps(layer, x, tau, out, flush, steps)
            st = layer.stats()
            row[name + "_us"] = 1000 * statistics.mean(sm_)
            if st["device_error"]:
                row[name + "_device_error"] = st["device_error"]
        layer.set_deterministic(False)
        layer.set_path(m.MOE_PATH_AUTO)
        rows.append(row)
        log(json.dumps({k: (round(v, 2) if isinstance(v, float) else v) for k, v in row.items()}))
    layer.close()
    torch.cuda.empty_cache()
    return rows


def run_ours(args):
    import torch
    world, rank, local = dist_setup()
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(local)
    import moe_inputs as mi
    import intra_expert_activation_router_b200 as m
    dev = torch.device("cuda", local)
    shape = mi.SHAPES[args.workload]
    T = args.T
    sweep_kind = "none" if args.no_sweep or world > 1 else args.sweep
    W, x = draw_inputs(shape, T, dev)
    layer = m.MoESparseLayer.from_weights(W, shape.top_k, max_tokens=max(T, 64))
    if args.path != "auto":
        layer.set_path({"sparse": m.MOE_PATH_SPARSE, "dense": m.MOE_PATH_DENSE}[args.path])
    layer.set_fused_router(args.router != "kernel", one_launch=args.router == "one_launch")
    if args.budget >= 0:
        layer.set_rank_budget(args.budget)
    out = torch.empty_like(x)
    tau = layer.calibrate_tau(x, args.sparsity)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = torch.empty(2 * l2 // 4, dtype=torch.float32, device=dev)

    for _ in range(args.warmup):
        layer.forward(x, tau, out=out)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(gpu_uuid(dev)) as clk:
        step_ms, router_ms, expert_ms = time_steps(layer, x, tau, out, flush, args.steps)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    total_ms = max_over_ranks(sum(step_ms), dev)
    ms = total_ms / args.steps
    value = whole_job_rate(world, T * args.steps, total_ms / 1000)
    st = layer.stats()
    # the same steps enqueued one by one from Python, for comparison
    eager_ms, _, _ = time_steps(layer, x, tau, out, flush, args.steps, graph=False)
    eager_ms = max_over_ranks(sum(eager_ms), dev) / args.steps
    path = "sparse" if st["path"] == m.MOE_PATH_SPARSE else "dense"
    alg = st["alg_bytes"] if path == "sparse" else st["dense_bytes"]
    # the router's bytes belong to the expert kernel when it routes the batch itself
    router_bytes = 0 if st["fused_router"] else shape.n_experts * shape.d_model * 2 + T * shape.d_model * 2
    expert_bytes = alg - router_bytes
    expert_ms_mean = statistics.mean(expert_ms)
    peaks, peak_kind = measured_peaks()
    peak = float(peaks["hbm_gbs"])
    achieved = expert_bytes / (expert_ms_mean / 1000) / 1e9
    kname = "k_expert_sparse" if path == "sparse" else "k_dense"
    traffic = recorded_traffic(kname, f"{args.workload}:T={T}")

    # end to end through the host-pointer entry: pinned x in, pinned out back, every step
    xh = x.cpu().pin_memory()
    oh = torch.empty_like(xh).pin_memory()
    e2e_steps = min(args.steps, 50)
    e2e_t = []
    for _ in range(e2e_steps):
        l2_flush(flush)
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        m.moe_sparse_forward_host(layer.h, xh, T, tau, oh)
        e2e_t.append(time.perf_counter() - t0)
    e2e_total = max_over_ranks(sum(e2e_t), dev)
    e2e_value = whole_job_rate(world, T * e2e_steps, e2e_total)
    layer.close()

    sweep = sweep_rows(dev, sweep_kind, peak, flush) if rank == 0 and sweep_kind != "none" else []
    modes = launch_mode_rows(dev, flush) if rank == 0 and sweep_kind != "none" else []
    budget_rows = rank_budget_rows(dev, flush) if rank == 0 and sweep_kind != "none" else []
    cap_rows = capacity_rows(dev, flush) if rank == 0 and sweep_kind != "none" else []
    det_rows = deterministic_rows(dev, flush) if rank == 0 and sweep_kind != "none" else []

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cores = cpu_cores()
        W_host, x_host = W.to("cpu"), x.cpu()
        tps, reps, el = oracle_time_sample(shape, W_host, x_host, tau, args.cpu_seconds, cores, args.budget)
        tps1, reps1, el1 = oracle_time_sample(shape, W_host, x_host[:4], tau, args.cpu_seconds / 2, 1, args.budget)
        cpu = {"value": tps, "unit": "tokens/s", "cores": cores, "kind": "oracle",
               "sample": f"{reps} repeats of the {T}-token batch ({el:.1f} s, fp64 oracle at the bench's "
                         f"tau, OpenMP over tokens on {cores} threads)",
               "single_thread": {"value": tps1, "unit": "tokens/s", "cores": 1,
                                 "sample": f"{reps1} repeats of the batch's first 4 tokens ({el1:.1f} s)"}}

    if rank == 0:
        clocks = clk.summary()
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic", "config": bench_config(args, world), "tau": tau, "path": path,
            "hbm_gbs": alg / (ms / 1000) / 1e9,
            "latency_us": 1000 * ms,
            "timing": "K steps captured in one CUDA graph and replayed once (device work identical; "
                      "no host enqueue gaps); eager_latency_us: the same steps enqueued one by one",
            "eager_latency_us": 1000 * eager_ms,
            "device_error": st["device_error"],
            "fused_router": st["fused_router"],
            "alg_bytes_per_step": alg,
            "kernels_us": {"router": 1000 * statistics.mean(router_ms), kname: 1000 * expert_ms_mean},
            "roofline": {"bound": "hbm", "kernel": kname, "achieved": achieved, "peak": peak,
                         "unit": "GB/s", "frac": achieved / peak, "traffic": traffic,
                         "peak_source": f"{peak_kind} copy bandwidth (MEASURED_PEAKS.json hbm_gbs)"
                         if peak_kind == "measured" else "fallback 6.65 TB/s (MEASURED_PEAKS.json absent)",
                         "alg_bytes_per_launch": expert_bytes},
            "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": T * shape.d_model * 2,
                    "d2h_bytes_per_step": T * shape.d_model * 2},
            # sparse: router (unless routed in the expert kernel), expert kernel, y conversion;
            # dense: router, gather, GEMM1 and GEMM2 per routed/shared group, convert
            "gpu_launches": ({0: 3, 1: 2, 2: 1}[st["fused_router"]] if path == "sparse"
                             else 5 + 2 * shape.n_shared) * args.steps,
            "clocks": {"sm_mhz": clocks["sm_mhz"], "sm_max_mhz": clocks["sm_max_mhz"],
                       "reasons": clocks["reasons"]},
            "stats": {"n_touched": st["n_touched"], "n_active": st["n_active"], "n_union": st["n_union"]},
            "sweep": sweep,
            "launch_modes": modes,
            "rank_budget": budget_rows,
            "capacity_drop": cap_rows,
            "deterministic_combine": det_rows,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
