#!/usr/bin/env python
"""Throughput of the Muon / MuonGS optimizer step on B200.

One step = one pass of the whole step (momentum, normalisation, 5 Newton-Schulz
iterations, [equilibration], scale, projection / decay, update) over every matrix of
a shape set, with weights, momenta and gradients resident in HBM. Prints one JSON
line. The default shape set is the largest one that fits a GPU, the 1.5B dense set;
the line also carries `per_set`, the same measurement for the other shape sets,
`sharded`, the ZeRO-1 sharded step over a one-rank NCCL group, and `next_rows`: the
MuonH and two-sided steps on the 400M shapes and the QK-Clip rescale.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload dense_1p5b]
  python bench.py --impl reference ...   # the float64 CPU oracle on host cores
  python bench.py --impl torch ...       # the same step in eager PyTorch on the GPU
                                         # (cuBLAS bf16 batched matmuls), for comparison

Multi-GPU (torchrun, one process per GPU), `--dist sharded` (default): the ZeRO-1
step of distributed.ShardedMuon over NCCL. Every rank holds its local gradients of
every matrix; one reduce-scatter brings each matrix's averaged gradient to its owner,
the owner runs the libmuon step on the matrices it owns, one all-gather shares the
updated weights. One job step is one step of the whole shape set (strong scaling).
`--dist replica`: every rank steps its own copy of the shape set with no collective
on the data path (weak scaling). At N = 1 the headline is the plain plan step.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_BYTES = 126 * 2 ** 20


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference", "torch"])
    ap.add_argument("--workload", default="dense_1p5b")
    ap.add_argument("--dist", default="sharded", choices=["sharded", "replica"],
                    help="multi-GPU mode: ZeRO-1 sharded step over NCCL, or independent replicas")
    ap.add_argument("--no-per-set", action="store_true", help="skip the other shape sets")
    ap.add_argument("--no-next", action="store_true",
                    help="skip the MuonH, two-sided and QK-Clip measurements")
    ap.add_argument("--no-sharded", action="store_true",
                    help="skip the one-rank NCCL sharded measurement at N = 1")
    ap.add_argument("--run", type=int, default=0,
                    help="which hyper-parameter setting of the workload (e.g. gpt400m: 0 MuonGS, 1 Muon+wd)")
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="budget of the oracle CPU-baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--slice-every", type=int, default=1,
                    help="profiling: keep every k-th matrix of the shape set (all classes in proportion)")
    ap.add_argument("--slice-class", type=int, default=-1,
                    help="profiling: keep only shape class i (in order of first appearance)")
    ap.add_argument("--slice-count", type=int, default=0,
                    help="profiling: with --slice-class, keep its first n matrices")
    return ap.parse_args()


def sliced(w, args):
    """The matrices of shape set w that a profiling slice keeps (all of them by default)."""
    specs = w.matrices()
    if args.slice_every > 1:
        specs = [s for s in specs if s.index % args.slice_every == 0]
    if args.slice_class >= 0:
        shapes = []
        for s in specs:
            if (s.rows, s.cols) not in shapes:
                shapes.append((s.rows, s.cols))
        specs = [s for s in specs if (s.rows, s.cols) == shapes[args.slice_class]]
        if args.slice_count > 0:
            specs = specs[:args.slice_count]
    return specs


def is_sliced(args) -> bool:
    return args.slice_every > 1 or args.slice_class >= 0


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,utilization.gpu,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.tmp = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", gpu_id, "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-lms", "20"], stdout=self.tmp, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        self.tmp.flush()
        rows = []
        with open(self.tmp.name) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) != 9:
                    continue
                try:
                    rows.append(dict(sm=float(parts[1]), smax=float(parts[2]), util=float(parts[4]),
                                     reasons=[n for n, v in zip(
                                         ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                                          "sw_power_cap"], parts[5:]) if v.lower() == "active"]))
                except ValueError:
                    continue
        os.unlink(self.tmp.name)
        load = [r for r in rows if r["util"] > 0] or rows
        if not load:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        reasons = sorted({x for r in load for x in r["reasons"]})
        return {"sm_mhz": statistics.median(r["sm"] for r in load),
                "sm_max_mhz": max(r["smax"] for r in load), "reasons": reasons,
                "samples": len(load)}


def gpu_id_for(torch, dev: int) -> str:
    try:
        u = str(torch.cuda.get_device_properties(dev).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        return vis.split(",")[dev] if vis else str(dev)


# ------------------------------------------------------------------ roofline traffic record
def traffic_record(kernel: str, workload: str):
    """Per-launch DRAM bytes of `kernel` from the committed ncu summary, valid only
    while the kernel's source is unchanged (sha256 of the sources listed there)."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(path):
        return None
    for line in open(path):
        parts = dict(p.split("=", 1) for p in line.split() if "=" in p)
        if parts.get("kernel") != kernel or parts.get("workload") != workload:
            continue
        h = hashlib.sha256()
        for src in parts.get("sources", "").split(","):
            with open(os.path.join(ROOT, src), "rb") as f:
                h.update(f.read())
        if h.hexdigest()[:16] != parts.get("sha"):
            return None
        return float(parts["bytes_per_launch"])
    return None


# ------------------------------------------------------------------ CPU oracle
def oracle_sample(w, run, budget_s: float, rotate: int = 0, smallest_only: bool = False):
    """Times the float64 oracle on a stratified sample of the shape set and extrapolates
    to one full step: sum over shape classes of count x mean seconds per matrix. With
    `smallest_only` (warm-up) it runs one matrix of the smallest shape class."""
    from matrix_orthogonalising_optimizer_03_b200 import workloads as wl
    from oracle import muon_oracle as orc
    hp = orc.HParams(lr=w.lr, momentum=w.momentum, weight_decay=run.weight_decay, mode=run.mode,
                     equilibrate=run.equilibrate)
    specs = w.matrices()
    by_class = {}
    for s in specs:
        by_class.setdefault((s.rows, s.cols), []).append(s)
    if smallest_only:
        key = min(by_class, key=lambda k: k[0] * k[1])
        by_class = {key: by_class[key]}
    t_start = time.perf_counter()
    per_class, sampled = {}, 0
    rounds = 0
    while True:
        for key, lst in by_class.items():
            s = lst[(rotate + rounds) % len(lst)]
            W = wl.weight(w, s).astype("float64")
            G = wl.grad(w, s, 0).astype("float64")
            M = __import__("numpy").zeros_like(W)
            t0 = time.perf_counter()
            orc.muon_step(W, G, M, hp)
            per_class.setdefault(key, []).append(time.perf_counter() - t0)
            sampled += 1
        rounds += 1
        if time.perf_counter() - t_start >= budget_s or rounds >= 64:
            break
    est = sum(len(by_class[k]) * statistics.mean(v) for k, v in per_class.items())
    return est, sampled, rounds


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def run_reference(args, rank: int, world: int):
    if rank != 0:
        return 0
    from matrix_orthogonalising_optimizer_03_b200 import workloads as wl
    w = wl.WORKLOADS[args.workload]
    run = w.runs[args.run]
    per_step = max(1.0, min(10.0, 150.0 / max(1, args.steps + args.warmup)))
    for i in range(args.warmup):  # untimed; one small matrix pages the code in
        oracle_sample(w, run, 0.0, rotate=i, smallest_only=True)
    times, sampled = [], 0
    for i in range(args.steps):
        est, n, _ = oracle_sample(w, run, per_step, rotate=args.warmup + i)
        times.append(est)
        sampled += n
    mean_s = statistics.mean(times)
    value = 1.0 / mean_s
    cores = blas_threads()
    sample = (f"each step: float64 oracle on a stratified sample of the {w.name} shape set "
              f"(>= 1 matrix per shape class, about {per_step:.0f} s), extrapolated by class counts; "
              f"{sampled} matrices timed in total")
    line = {"metric": "muon_steps_per_s", "value": value, "unit": "steps/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": mean_s * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": {"workload": w.name, "matrices": w.n_matrices, "params": w.n_params,
                       "mode": run.mode, "weight_decay": run.weight_decay,
                       "equilibrate": run.equilibrate},
            "cpu_baseline": {"value": value, "unit": "steps/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "steps/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ eager PyTorch arm
def run_torch(args, rank: int, world: int, local: int):
    """The same optimizer step written as eager PyTorch on the GPU, the usual way to run
    Muon: per shape class one batched tensor, momentum and Nesterov by in-place ops,
    the quintic Newton-Schulz iteration with bf16 batched matmuls (cuBLAS), the
    Moonlight scale, the MuonGS projection and the update. No libmuon code runs."""
    import torch
    import torch.distributed as dist
    from datetime import timedelta

    from matrix_orthogonalising_optimizer_03_b200 import workloads as wl

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=dev)
    w = wl.WORKLOADS[args.workload]
    run = w.runs[args.run]
    if run.equilibrate or run.mode not in ("muon", "muongs") or w.ns_fp32:
        if rank == 0:
            print(json.dumps({"impl": "torch", "unavailable": "the eager arm covers bf16 Muon and "
                              "MuonGS without equilibration"}), flush=True)
        return 0
    specs = w.matrices()
    Ws, G_src = wl.device_inputs(w, dev, seed=rank)
    gdt = torch.bfloat16 if w.grad_dtype == "bf16" else torch.float32
    classes = {}
    for s, W, G in zip(specs, Ws, G_src):
        classes.setdefault((s.rows, s.cols), []).append((W, G))
    batches = []
    for (r, c), lst in classes.items():
        W = torch.stack([x[0] for x in lst])
        G = torch.stack([x[1] for x in lst]).to(gdt)
        batches.append((W, G, torch.zeros_like(W), r > c, 0.2 * max(r, c) ** 0.5))
    del Ws, G_src
    a, b, c = 3.4445, -4.7750, 2.0315
    mu, lr, wd, eps = w.momentum, w.lr, run.weight_decay, 1e-7

    def step():
        for W, G, M, tall, scale in batches:
            M.mul_(mu).add_(G)
            U = torch.add(G, M, alpha=mu)
            X = (U / (U.norm(dim=(1, 2), keepdim=True) + eps)).to(torch.bfloat16)
            if tall:
                X = X.mT
            for _ in range(5):
                A = torch.bmm(X, X.mT)
                Bm = torch.baddbmm(A, A, A, beta=b, alpha=c)
                X = torch.baddbmm(X, Bm, X, beta=a, alpha=1.0)
            O = (X.mT if tall else X).float() * scale
            cw = torch.full((W.shape[0], 1, 1), 1.0 - lr * wd, device=W.device)
            if run.mode == "muongs":
                cw = cw + lr * (W * O).sum(dim=(1, 2), keepdim=True) / (
                    W * W).sum(dim=(1, 2), keepdim=True).clamp_min(1e-30)
            W.mul_(cw).add_(O, alpha=-lr)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = rank_max(e0.elapsed_time(e1), world, dev)
    if rank == 0:
        value = throughput(args.steps, world, ms)
        print(json.dumps({
            "metric": "muon_steps_per_s", "value": value, "unit": "steps/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic", "impl": "torch",
            "config": {"workload": w.name, "matrices": w.n_matrices, "params": w.n_params,
                       "mode": run.mode, "weight_decay": run.weight_decay,
                       "ns_path": "torch.bmm / baddbmm bf16 (cuBLAS)",
                       "parallelism": f"replica x{world}"}}), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


# ------------------------------------------------------------------ multi-rank timing
def rank_max(x: float, world: int, device="cpu") -> float:
    """The maximum of x over all ranks of the default process group (x itself at
    world 1). Every rank must call it at the same point."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def throughput(steps: int, world: int, ms_max: float, scaling: str = "weak") -> float:
    """Whole-job shape-set steps per second, timed by the slowest rank. Weak scaling:
    every rank steps its own copy of the shape set `steps` times. Strong scaling: the
    ranks share one shape set, so a job step is one shape-set step."""
    copies = world if scaling == "weak" else 1
    return steps * copies / (ms_max / 1e3)


# ------------------------------------------------------------------ per-kernel summaries
ELEMENTWISE = ("ingest", "post_reduce", "post_apply")


def elementwise_rates(prof, peaks):
    """Achieved algorithmic GB/s of the memory-bound kernels and their fraction of the
    measured HBM copy bandwidth."""
    out = {}
    for k in ELEMENTWISE:
        v = prof.get(k)
        if not v or not v["launches"] or v["total_ms"] <= 0:
            continue
        gbs = v["bytes"] / (v["total_ms"] / 1e3) / 1e9
        out[k] = {"gb_s": gbs, "frac": gbs / peaks["hbm_gbs"],
                  "bytes_per_launch": v["bytes"] / v["launches"],
                  "ms_per_launch": v["total_ms"] / v["launches"]}
    return out


def ns_rates(prof, w, steps: int, ms_total: float, peaks, specs=None):
    """Newton-Schulz throughput in algorithmic flops (symmetric Gram and polynomial
    counted once), over the whole step time and over the summed time of the
    Newton-Schulz launches, each as a fraction of the burst and sustained bf16 peaks."""
    from matrix_orthogonalising_optimizer_03_b200 import workloads as wl
    per_step = (wl.workload_ns_flops(w) if specs is None
                else sum(wl.ns_flops(s.rows, s.cols) for s in specs))
    flops = per_step * steps
    ns_ms = sum(v["total_ms"] for k, v in prof.items() if k.startswith("ns_"))
    step_tf = flops / (ms_total / 1e3) / 1e12
    phase_tf = flops / (ns_ms / 1e3) / 1e12 if ns_ms > 0 else None

    def fr(x):
        if x is None or w.ns_fp32:
            return None
        return {"burst": x / peaks["bf16_tflops"], "sustained": x / peaks["bf16_tflops_sustained"]}
    return {"ns_tflops_step": step_tf, "ns_frac_step": fr(step_tf),
            "ns_tflops_phases": phase_tf, "ns_frac_phases": fr(phase_tf),
            "ns_ms_per_step": ns_ms / steps}


# ------------------------------------------------------------------ one shape set on one GPU
def set_inputs(w, dev, seed: int, specs=None):
    """Resident inputs of a shape set (or of the matrices `specs` of it): W (fp32), M
    (fp32, zero) and one flat gradient buffer with a view per matrix, drawn on the
    device (seeded)."""
    import torch
    from matrix_orthogonalising_optimizer_03_b200 import workloads as wl
    all_specs = w.matrices()
    specs = all_specs if specs is None else specs
    gdt = torch.bfloat16 if w.grad_dtype == "bf16" else torch.float32
    numel = sum(s.rows * s.cols for s in specs)
    subset = None if len(specs) == len(all_specs) else {s.index for s in specs}
    Ws, G_src = wl.device_inputs(w, dev, seed=seed, only=subset)
    g_flat = torch.empty(numel, dtype=gdt, device=dev)
    Ms, Gs = [], []
    off = 0
    for s, g in zip(specs, G_src):
        Ms.append(torch.zeros(s.rows, s.cols, dtype=torch.float32, device=dev))
        gv = g_flat[off:off + s.rows * s.cols].view(s.rows, s.cols)
        gv.copy_(g)
        Gs.append(gv)
        off += s.rows * s.cols
    del G_src
    return Ws, Gs, Ms, g_flat, numel, gdt


def time_steps(step, steps: int, world: int, dev, stream, after_start=None):
    """CUDA-event time (ms, max over ranks) of `steps` calls of step(), bracketed by a
    barrier and a device synchronisation on both sides. after_start() runs right after
    the start event is recorded (e.g. to order another stream behind it)."""
    import torch
    import torch.distributed as dist

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    e0.record(stream)
    if after_start is not None:
        after_start()
    for _ in range(steps):
        step()
    e1.record(stream)
    barrier()
    return rank_max(e0.elapsed_time(e1), world, dev)


def measure_plan(B, w, run, args, dev, world: int, peaks, peak_src, seed: int, full: bool,
                 specs=None):
    """The plain plan step of one shape set (or of the matrices `specs` of it): warm-up,
    K timed steps, K profiled steps (per-kernel CUDA events), and with `full` the
    end-to-end feed. Returns a summary dict and the live weights and momenta."""
    import torch
    from matrix_orthogonalising_optimizer_03_b200 import workloads as wl
    Ws, Gs, Ms, g_flat, numel, gdt = set_inputs(w, dev, seed, specs)
    gsz = 2 if w.grad_dtype == "bf16" else 4
    hp = B.hparams(lr=w.lr, momentum=w.momentum, weight_decay=run.weight_decay, mode=run.mode,
                   equilibrate=run.equilibrate, ns_fp32=w.ns_fp32)
    plan = B.Plan(Ws, Gs, Ms, hp)
    stats = B.new_stats(len(Ws), dev)
    stream = torch.cuda.current_stream()
    torch.cuda.synchronize()
    local = dev.index if dev.index is not None else 0
    sampler = ClockSampler(gpu_id_for(torch, local))
    for _ in range(args.warmup):
        plan.step(stats=stats)
    torch.cuda.synchronize()
    if plan.query_device_status() != 0:
        raise RuntimeError(f"device-side error during warm-up ({w.name})")
    ms = time_steps(lambda: plan.step(stats=stats), args.steps, world, dev, stream)
    clocks = sampler.stop()
    # profiled pass over the same K steps: per-kernel device times on the launching stream
    B.load().muon_plan_profile_enable(plan._plan, 1)
    torch.cuda.synchronize()
    for _ in range(args.steps):
        plan.step(stats=stats)
    prof = plan_profile(B, plan)
    B.load().muon_plan_profile_enable(plan._plan, 0)
    launches = sum(p["launches"] for p in prof.values())
    out = {
        "value": throughput(args.steps, world, ms, "weak"), "unit": "steps/s",
        "ms_per_step": ms / args.steps,
        "matrices": w.n_matrices if specs is None else len(specs),
        "params": w.n_params if specs is None else sum(s.rows * s.cols for s in specs),
        "mode": run.mode, "weight_decay": run.weight_decay, "equilibrate": run.equilibrate,
        "ns_path": ("none (two-sided normalisation)" if run.mode == "twosided"
                    else "fp32 CUDA cores" if w.ns_fp32 else "bf16 tcgen05"),
        **(ns_rates(prof, w, args.steps, ms, peaks, specs) if run.mode != "twosided" else
           {"ns_tflops_step": None, "ns_frac_step": None, "ns_tflops_phases": None,
            "ns_frac_phases": None, "ns_ms_per_step": 0.0}),
        "roofline": roofline(prof, w, peaks, peak_src, w.name if specs is None else None, ms,
                             clocks),
        "elementwise": elementwise_rates(prof, peaks),
        "kernels": {k: {"launches_per_step": v["launches"] / args.steps,
                        "ms_per_step": v["total_ms"] / args.steps} for k, v in prof.items()
                    if v["launches"]},
        "gpu_launches": int(round(launches)),
        "clocks": clocks,
        "l2": "inputs larger than L2 (W+M+G = %.0f MB vs 126 MB)" % (numel * (8 + gsz) / 1e6),
    }
    if full:
        # a learning-rate schedule: new hyper-parameters before every step (the plan
        # updates its captured graph in place)
        lrs = [w.lr * (0.5 + 0.5 * ((t * 7) % 10) / 10.0) for t in range(args.steps)]
        it = iter(lrs)

        def sched_step():
            plan.set_hparams(B.hparams(lr=next(it), momentum=w.momentum,
                                       weight_decay=run.weight_decay, mode=run.mode,
                                       equilibrate=run.equilibrate, ns_fp32=w.ns_fp32))
            plan.step(stats=stats)
        ms_sched = time_steps(sched_step, args.steps, world, dev, stream)
        out["lr_schedule"] = {"value": throughput(args.steps, world, ms_sched, "weak"),
                              "unit": "steps/s", "ms_per_step": ms_sched / args.steps,
                              "what": "muon_plan_set_hparams (new lr) before every step"}
        # end to end through the public API (binding.StreamedSteps): every step copies
        # its gradients from pinned host memory and reads the per-matrix statistics
        # back; the copy of step t+1 overlaps step t on a second stream
        g_host = torch.empty(numel, dtype=gdt, pin_memory=True)
        g_host.copy_(g_flat)
        feed = B.StreamedSteps(Ws, Ms, hp, grad_dtype=gdt)
        for _ in range(2):
            feed.step(g_host)

        def fed_step():
            feed.step(g_host)
        # every copy starts inside the timed region: the copy stream waits for the start
        ms_e2e = time_steps(fed_step, args.steps, world, dev, stream,
                            after_start=lambda: feed.copy_stream.wait_stream(stream))
        torch.cuda.synchronize()
        feed.close()
        del feed, g_host
        out["e2e"] = {"value": throughput(args.steps, world, ms_e2e, "weak"), "unit": "steps/s",
                      "h2d_bytes_per_step": numel * gsz, "d2h_bytes_per_step": stats.numel() * 4,
                      "overlap": "H2D of step t+1 on a copy stream during step t (two buffers)"}
    if plan.query_device_status() != 0:
        raise RuntimeError(f"device-side error in the timed region ({w.name})")
    plan.close()
    del plan, Gs, g_flat, stats
    return out, Ws, Ms


def measure_sharded(B, w, run, args, dev, world: int, rank: int, peaks, peak_src, seed: int,
                    e2e: bool):
    """The ZeRO-1 sharded step (distributed.ShardedMuon) over the current NCCL process
    group: reduce-scatter of the gradients to their owners, the owners' libmuon plan
    step, all-gather of the updated weights. Every rank holds its own local gradients
    of every matrix. One job step is one shape-set step (strong scaling)."""
    import torch
    from matrix_orthogonalising_optimizer_03_b200 import distributed as D
    from matrix_orthogonalising_optimizer_03_b200 import workloads as wl
    specs = w.matrices()
    gdt = torch.bfloat16 if w.grad_dtype == "bf16" else torch.float32
    gsz = 2 if w.grad_dtype == "bf16" else 4
    Ws, Gs = wl.device_inputs(w, dev, seed=seed)
    opt = D.ShardedMuon([(s.rows, s.cols) for s in specs], dev, init=Ws, grad_dtype=gdt,
                        lr=w.lr, momentum=w.momentum, weight_decay=run.weight_decay,
                        mode=run.mode, equilibrate=run.equilibrate, ns_fp32=w.ns_fp32)
    for gv, g in zip(opt.grads, Gs):
        gv.copy_(g)
    del Ws, Gs
    n_mine = len(opt.mine)
    stats = B.new_stats(max(n_mine, 1), dev)
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        opt.step(stats=stats if n_mine else None)
    torch.cuda.synchronize()
    local = dev.index if dev.index is not None else 0
    sampler = ClockSampler(gpu_id_for(torch, local))
    ms = time_steps(lambda: opt.step(stats=stats if n_mine else None), args.steps, world, dev,
                    stream)
    clocks = sampler.stop()
    prof = {}
    if opt.plan is not None:
        B.load().muon_plan_profile_enable(opt.plan._plan, 1)
        torch.cuda.synchronize()
    for _ in range(args.steps):   # every rank takes part in the collectives
        opt.step(stats=stats if n_mine else None)
    if opt.plan is not None:
        prof = plan_profile(B, opt.plan)
        B.load().muon_plan_profile_enable(opt.plan._plan, 0)
    launches = rank_max(float(sum(p["launches"] for p in prof.values())), world, dev)
    out = {"value": throughput(args.steps, world, ms, "strong"), "unit": "steps/s",
           "ms_per_step": ms / args.steps, "world": world, "backend": opt.backend,
           "scaling": "strong", "owned_matrices": n_mine,
           "collectives": "reduce_scatter_tensor (avg, bf16 grads) + all_gather_into_tensor "
                          "(fp32 W), in place",
           "kernels": {k: {"launches_per_step": v["launches"] / args.steps,
                           "ms_per_step": v["total_ms"] / args.steps} for k, v in prof.items()
                       if v["launches"]},
           "gpu_launches_max_rank": int(round(launches)),
           "clocks": clocks}
    if prof:
        out["roofline"] = roofline(prof, w, peaks, peak_src, w.name, ms, clocks)
    if e2e:
        # end to end: each step copies this rank's local gradients from pinned host
        # memory (on the compute stream, not overlapped) and reads the statistics back
        numel = opt.flat_g.numel()
        g_host = torch.empty(numel, dtype=gdt, pin_memory=True)
        g_host.copy_(opt.flat_g)
        st_host = torch.empty_like(stats, device="cpu").pin_memory()

        def fed_step():
            opt.flat_g.copy_(g_host, non_blocking=True)
            opt.step(stats=stats if n_mine else None)
            st_host.copy_(stats, non_blocking=True)
        ms_e2e = time_steps(fed_step, args.steps, world, dev, stream)
        out["e2e"] = {"value": throughput(args.steps, world, ms_e2e, "strong"), "unit": "steps/s",
                      "h2d_bytes_per_step": numel * gsz, "d2h_bytes_per_step": stats.numel() * 4,
                      "overlap": "none (copy, step and read-back in order on one stream)"}
        del g_host, st_host
    if opt.plan is not None:
        if opt.plan.query_device_status() != 0:
            raise RuntimeError("device-side error in the sharded step")
        opt.plan.close()
    del opt
    torch.cuda.synchronize()
    return out


PER_SET = [("gpt160m", 0), ("gpt400m", 0), ("gpt400m", 1), ("moe_1b", 0), ("single_128x256", 0),
           ("single_128x256", 1)]

# The follow-on features that run as kernels of their own, each timed like a shape set:
# the MuonH retraction and the two-sided normalisation on the 400M shapes (MuonW is the
# Muon + weight-decay run of the same set, and the ZeRO-1 step is the "sharded" record).
NEXT_RUNS = [("gpt400m", "muonh", 0.0), ("gpt400m", "twosided", 0.0)]


def measure_qk_clip(B, args, dev, peaks):
    """QK-Clip: the per-head rescale of the query and key weights (the Moonlight review's
    MuonClip; the loss-spike page's QK-Clip section) on the attention shapes of the 1.5B
    dense set: 24 layers of W_q and W_k, 2048 x 2048 fp32, 16 heads of 128 rows, with the
    caller's S_max drawn so that half of the heads exceed tau = 100 (gamma = 2/3,
    power 1/2 on each side). Algorithmic bytes: 8 per rescaled element (read and write);
    heads at or below tau are not touched. Timed with CUDA events on the launching
    stream over K calls of a QkClipPlan (descriptors marshalled once) after W warm-up
    calls."""
    import torch
    layers, heads, d, hd = 24, 16, 2048, 128
    g = torch.Generator(device=dev)
    g.manual_seed(20)
    wq = [torch.randn(d, d, device=dev, generator=g) * 0.02 for _ in range(layers)]
    wk = [torch.randn(d, d, device=dev, generator=g) * 0.02 for _ in range(layers)]
    hot = torch.rand(layers * heads, device=dev, generator=g) < 0.5
    s_max = torch.where(hot, torch.full_like(hot, 150.0, dtype=torch.float32),
                        torch.full_like(hot, 50.0, dtype=torch.float32))
    slices = []
    for li in range(layers):
        for h in range(heads):
            slices.append((wq[li], h * hd, hd, li * heads + h, 0.5))
            slices.append((wk[li], h * hd, hd, li * heads + h, 0.5))
    clip = B.QkClipPlan(slices, s_max, tau=100.0)  # the descriptors marshalled once
    for _ in range(args.warmup):
        clip.apply()
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(args.steps):
        clip.apply()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    scaled = int(hot.sum().item()) * 2 * hd * d
    gbs = 8.0 * scaled / (ms / 1e3) / 1e9
    return {"ms_per_call": ms, "heads_clipped": int(hot.sum().item()),
            "heads": layers * heads, "rescaled_elements": scaled,
            "gb_s": gbs, "frac": gbs / peaks["hbm_gbs"], "bound": "hbm",
            "what": "24 layers x (W_q, W_k) 2048 x 2048 fp32, 16 heads of 128 rows, "
                    "half of the heads above tau"}


# ------------------------------------------------------------------ GPU arm
def main():
    args = parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank, world)
    if args.impl == "torch":
        return run_torch(args, rank, world, local)

    import torch
    import torch.distributed as dist
    from datetime import timedelta

    from matrix_orthogonalising_optimizer_03_b200 import binding as B
    from matrix_orthogonalising_optimizer_03_b200 import workloads as wl

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=dev)
    B.load()
    w = wl.WORKLOADS[args.workload]
    run = w.runs[args.run]
    peaks, peak_src = load_peaks()
    sharded_job = world > 1 and args.dist == "sharded"
    gsz = 2 if w.grad_dtype == "bf16" else 4

    if is_sliced(args):
        # a profiling slice of the shape set: the plan step only, no comparison legs
        if world != 1:
            raise SystemExit("profiling slices run on one GPU")
        specs = sliced(w, args)
        res, _, _ = measure_plan(B, w, run, args, dev, 1, peaks, peak_src, 0, full=False,
                                 specs=specs)
        print(json.dumps({"profiling_slice": {"workload": w.name, "every": args.slice_every,
                                              "class": args.slice_class, "count": len(specs)},
                          **res}), flush=True)
        return 0
    if sharded_job:
        res = measure_sharded(B, w, run, args, dev, world, rank, peaks, peak_src, 0, e2e=True)
        line_core = {"value": res["value"], "ms_per_step": res["ms_per_step"],
                     "scaling": "strong", "roofline": res.get("roofline"),
                     "kernels": res["kernels"], "gpu_launches": res["gpu_launches_max_rank"],
                     "e2e": res["e2e"], "clocks": res["clocks"]}
        parallelism = f"zero1-sharded x{world} (nccl)"
        extra = {"sharded": {k: v for k, v in res.items() if k not in ("e2e",)}}
        cpu = None
    else:
        res, _, _ = measure_plan(B, w, run, args, dev, world, peaks, peak_src, rank, full=True)
        line_core = {"value": res["value"], "ms_per_step": res["ms_per_step"],
                     "scaling": "weak" if world > 1 else "strong", "roofline": res["roofline"],
                     "kernels": res["kernels"], "gpu_launches": res["gpu_launches"],
                     "e2e": res["e2e"], "clocks": res["clocks"]}
        parallelism = f"replica x{world}" if world > 1 else "single GPU"
        extra = {k: res[k] for k in ("ns_tflops_step", "ns_frac_step", "ns_tflops_phases",
                                     "ns_frac_phases", "ns_ms_per_step", "elementwise",
                                     "lr_schedule")}
        cpu = None
        if world == 1 and rank == 0 and not args.no_cpu_baseline:
            est, n, rounds = oracle_sample(w, run, args.cpu_seconds)
            cpu = {"value": 1.0 / est, "unit": "steps/s", "cores": blas_threads(), "kind": "oracle",
                   "sample": f"float64 oracle on {n} matrices ({rounds} per shape class) of the "
                             f"{w.name} shape set, extrapolated to one full step by class counts"}
        torch.cuda.empty_cache()
        if world == 1 and not args.no_sharded:
            # the sharded step at world 1: a one-rank NCCL group, in-place collectives
            dist.init_process_group("nccl", store=dist.HashStore(), rank=0, world_size=1,
                                    device_id=dev)
            try:
                sh = measure_sharded(B, w, run, args, dev, 1, 0, peaks, peak_src, 0, e2e=False)
            finally:
                dist.destroy_process_group()
            extra["sharded"] = {k: sh[k] for k in ("value", "unit", "ms_per_step", "world",
                                                   "backend", "scaling", "collectives",
                                                   "gpu_launches_max_rank")}
            torch.cuda.empty_cache()
        if world == 1 and not args.no_per_set:
            per = {}
            for name, ridx in PER_SET:
                if name == w.name and ridx == args.run:
                    continue
                ws = wl.WORKLOADS[name]
                r, _, _ = measure_plan(B, ws, ws.runs[ridx], args, dev, 1, peaks, peak_src, 0,
                                       full=False)
                per[f"{name}/{ws.runs[ridx].mode}" + ("+wd" if ws.runs[ridx].weight_decay else "")] = r
                torch.cuda.empty_cache()
            extra["per_set"] = per
        if world == 1 and not args.no_next:
            nxt = {}
            for name, mode, wd in NEXT_RUNS:
                ws = wl.WORKLOADS[name]
                r, _, _ = measure_plan(B, ws, wl.Run(mode, wd), args, dev, 1, peaks, peak_src, 0,
                                       full=False)
                nxt[f"{mode}/{name}"] = r
                torch.cuda.empty_cache()
            nxt["qk_clip"] = measure_qk_clip(B, args, dev, peaks)
            torch.cuda.empty_cache()
            extra["next_rows"] = nxt

    if rank == 0:
        line = {
            "metric": "muon_steps_per_s", "value": line_core["value"], "unit": "steps/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": line_core["ms_per_step"], "higher_is_better": True,
            "scaling": line_core["scaling"], "vs_baseline": None,
            "dtype": "f32" if w.ns_fp32 else "bf16", "data": "synthetic",
            "config": {"workload": w.name, "matrices": w.n_matrices, "params": w.n_params,
                       "mode": run.mode, "weight_decay": run.weight_decay,
                       "equilibrate": run.equilibrate, "ns_steps": 5, "grad_dtype": w.grad_dtype,
                       "ns_path": "fp32 CUDA cores" if w.ns_fp32 else "bf16 tcgen05",
                       "ns_tflops_per_step": wl.workload_ns_flops(w) / 1e12,
                       "l2": "inputs larger than L2 (W+M+G = %.0f MB vs 126 MB)" % (
                           w.n_params * (8 + gsz) / 1e6),
                       "parallelism": parallelism},
            "ns_tflops": extra.get("ns_tflops_step"),
            "roofline": line_core["roofline"],
            "kernels": line_core["kernels"],
            "gpu_launches": line_core["gpu_launches"],
            "e2e": line_core["e2e"],
            "clocks": line_core["clocks"],
            "cpu_baseline": cpu,
            **extra,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def plan_profile(B, plan):
    import ctypes

    class Entry(ctypes.Structure):
        _fields_ = [("name", ctypes.c_char * 32), ("launches", ctypes.c_int32),
                    ("total_ms", ctypes.c_float), ("flops", ctypes.c_double),
                    ("bytes", ctypes.c_double)]
    lib = B.load()
    lib.muon_plan_profile_read.restype = ctypes.c_int
    lib.muon_plan_profile_read.argtypes = [ctypes.c_void_p, ctypes.POINTER(Entry), ctypes.c_int]
    arr = (Entry * 16)()
    n = lib.muon_plan_profile_read(plan._plan, arr, 16)
    if n < 0:
        raise RuntimeError("muon_plan_profile_read failed")
    return {arr[i].name.decode(): {"launches": arr[i].launches, "total_ms": arr[i].total_ms,
                                    "flops": arr[i].flops, "bytes": arr[i].bytes} for i in range(n)}


def roofline(prof, w, peaks, peak_src, workload, region_ms: float, clocks=None):
    ns = {k: v for k, v in prof.items() if k.startswith("ns_") and v["launches"]}
    if not ns:
        return None
    name, v = max(ns.items(), key=lambda kv: kv[1]["total_ms"])
    per_launch_s = v["total_ms"] / 1e3 / v["launches"]
    flops = v["flops"] / v["launches"]
    achieved = flops / per_launch_s / 1e12
    if w.ns_fp32:
        alu_peak = 148 * 128 * 2 * 1.965e9 / 1e12
        return {"bound": "alu", "kernel": name, "achieved": achieved, "unit": "TFLOP/s",
                "peak": alu_peak, "frac": achieved / alu_peak, "traffic": None,
                "peak_source": "fp32 FMA: 148 SMs x 128 lanes x 2 flops x 1965 MHz"}
    # a kernel that ran under the power cap (the clock record shows sw_power_cap), or
    # inside a timed region of a second or more, is in the sustained regime: compare it
    # with the sustained figure; otherwise with the burst figure. Both are reported.
    capped = clocks is not None and "sw_power_cap" in (clocks.get("reasons") or [])
    sustained = region_ms >= 1000.0 or capped
    peak = peaks["bf16_tflops_sustained" if sustained else "bf16_tflops"]
    traffic = traffic_record(name, workload)
    return {"bound": "tensor", "kernel": name, "achieved": achieved, "peak": peak,
            "unit": "TFLOP/s", "frac": achieved / peak, "traffic": traffic,
            "frac_burst": achieved / peaks["bf16_tflops"],
            "frac_sustained": achieved / peaks["bf16_tflops_sustained"],
            "flops_per_launch": flops, "launch_ms": per_launch_s * 1e3,
            "peak_source": f"{peak_src} bf16 ({'sustained' if sustained else 'burst'}"
                           f"{': sw_power_cap in the timed region' if capped else ''})"}


if __name__ == "__main__":
    sys.exit(main())
