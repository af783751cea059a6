#!/usr/bin/env python
"""Benchmark of the LittleBit factorised binary layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

One step = one token (batch 1) through a decoder stack of factorised linears
(every linear: both contractions of both branches, all three scales, and the
decoder glue), i.e. one call of lb_stack_forward.  Rank 0 prints one JSON line.

Workloads (seeded synthetic weights; no dataset or trained checkpoint exists here):
  stack70b-1.0 (default), stack70b-0.55, stack13b-0.55, stack13b-0.1,
  mlp7b-{1.0,0.55,0.3,0.1}

Multi-GPU: the layer does not shard at batch 1, so N GPUs run N independent
replicas (one process per GPU under torchrun); the job's tokens/s is the sum,
timed as the max over ranks.
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
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

WORKLOADS = {
    "stack70b-1.0": ("llama2-70b", 1.0, "stack"),
    "stack70b-0.55": ("llama2-70b", 0.55, "stack"),
    "stack13b-0.55": ("llama2-13b", 0.55, "stack"),
    "stack13b-0.1": ("llama2-13b", 0.1, "stack"),
    "mlp7b-1.0": ("llama2-7b", 1.0, "mlp"),
    "mlp7b-0.55": ("llama2-7b", 0.55, "mlp"),
    "mlp7b-0.3": ("llama2-7b", 0.3, "mlp"),
    "mlp7b-0.1": ("llama2-7b", 0.1, "mlp"),
}
METRIC = "batch-1 layer-stack tokens/s"
L2_BYTES = 126 * 1024 * 1024


def describe(name: str) -> str:
    model, bpw, kind = WORKLOADS[name]
    if kind == "mlp":
        return f"{model} MLP block (gate, up 4096->11008, down 11008->4096), {bpw} bits/weight, batch 1"
    return f"{model} decoder linear stack, all layers, {bpw} bits/weight, 2 branches, batch 1"


# ---------------------------------------------------------------- distributed plumbing
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(value: float, world: int, device=None) -> float:
    """Max of a per-rank float over all ranks (identity when world == 1)."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int, device=None):
    if world > 1:
        import torch.distributed as dist
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clocks and throttle reasons with nvidia-smi while running."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.thread.join(timeout=5)

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------- workloads
def build_workload(name: str, device, seed: int):
    from binary_rank_linear_lb_b200.configs import MODELS, linear_bytes
    from binary_rank_linear_lb_b200.model import build_mlp_block, build_stack
    model_name, bpw, kind = WORKLOADS[name]
    model = MODELS[model_name]
    if kind == "mlp":
        st = build_mlp_block(model, bpw, base=seed, device=device, signs="bits")
        nbytes = sum(linear_bytes(*model.shapes()[p], model.ranks(bpw)[p]) for p in (4, 5, 6))
    else:
        st = build_stack(model, bpw, base=seed, device=device, signs="bits")
        nbytes = model.bytes_per_token(bpw)
    return st, model, bpw, kind, nbytes


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(path))
        return float(d["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return 6650.0, "fallback"


def cpu_oracle_rate(name: str, budget_s: float = 12.0):
    """Oracle tokens/s on a bounded sample: a few whole layers of one token, scaled."""
    import numpy as np
    import oracle
    from oracle import stack as ostack
    from binary_rank_linear_lb_b200.configs import MODELS
    model_name, bpw, kind = WORKLOADS[name]
    model = MODELS[model_name]
    rk = model.ranks(bpw)
    rng = np.random.default_rng(0)

    def lin(p):
        i, o = model.shapes()[p]
        r = rk[p]
        brs = []
        for _ in range(2):
            Vp = rng.integers(0, 2 ** 32, size=(r, (i + 31) // 32), dtype=np.uint64).astype(np.uint32)
            Up = rng.integers(0, 2 ** 32, size=(o, (r + 31) // 32), dtype=np.uint64).astype(np.uint32)
            sc = lambda n: np.abs(1 + 0.1 * rng.standard_normal(n))
            brs.append(oracle.Branch(Vp, Up, sc(o), sc(i), sc(r)))
        return ostack.Linear(brs, i, o, r)

    x = rng.standard_normal(model.hidden)
    t0 = time.perf_counter()
    layers_done = 0
    if kind == "mlp":
        g, u, d = lin(4), lin(5), lin(6)
        t0 = time.perf_counter()
        reps = 0
        while True:
            ostack.mlp_block(x, g, u, d)
            reps += 1
            if time.perf_counter() - t0 > budget_s or reps >= 50:
                break
        dt = (time.perf_counter() - t0) / reps
        return 1.0 / dt, oracle.threads(), f"{reps} full MLP-block tokens"
    elapsed = 0.0
    while elapsed < budget_s and layers_done < model.n_layers:
        L = {n: lin(p) for p, n in enumerate(("q", "k", "v", "o", "gate", "up", "down"))}
        t0 = time.perf_counter()
        ostack.decoder_stack(x, [L], model.n_heads, model.n_kv_heads, model.head_dim)
        elapsed += time.perf_counter() - t0
        layers_done += 1
    per_token = elapsed / layers_done * model.n_layers
    return 1.0 / per_token, oracle.threads(), (
        f"{layers_done} of {model.n_layers} decoder layers of one token, time scaled to all layers")


# ---------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="stack70b-1.0", choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    world, rank, local = dist_env()
    if args.warmup < 3:
        args.warmup = 3

    if args.impl == "reference":
        # The reference arm is the oracle itself (no installable reference exists),
        # run on the host cores by rank 0 only.
        if rank != 0:
            return 0
        rate, cores, sample = cpu_oracle_rate(args.workload,
                                              budget_s=max(5.0, 20.0 / max(1, args.steps)))
        line = {"impl": "reference", "metric": METRIC, "value": rate, "unit": "tokens/s",
                "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": 1e3 / rate, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": {"workload": describe(args.workload)},
                "cpu_baseline": {"value": rate, "unit": "tokens/s", "cores": cores,
                                 "kind": "oracle", "sample": sample},
                "e2e": {"value": rate, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return 0

    import torch
    import binary_rank_linear_lb_b200 as lb
    from binary_rank_linear_lb_b200 import synth

    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    device = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(device)

    st, model, bpw, kind, nbytes = build_workload(args.workload, device, args.seed + rank)
    x = synth.activation(model.hidden, 1234 + rank, torch.bfloat16, device)
    y = torch.empty(model.hidden, dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream(device)
    flush = None
    if nbytes < 2 * L2_BYTES:
        flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=device)

    for _ in range(args.warmup):
        st.forward(x, y)
    torch.cuda.synchronize(device)
    if st.status() != lb.LB_OK:
        raise RuntimeError("device-side wait timed out during warm-up")

    uuid = str(torch.cuda.get_device_properties(device).uuid)
    gpu_id = uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    stops = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    barrier(world, device)
    torch.cuda.synchronize(device)
    with ClockSampler(gpu_id) as clocks:
        t_wall = time.perf_counter()
        for i in range(args.steps):
            if flush is not None:
                flush.fill_(i & 0xFF)
            starts[i].record(stream)
            st.forward(x, y)
            stops[i].record(stream)
        torch.cuda.synchronize(device)
        t_wall = time.perf_counter() - t_wall
    barrier(world, device)
    if st.status() != lb.LB_OK:
        raise RuntimeError("device-side wait timed out")
    step_ms = [a.elapsed_time(b) for a, b in zip(starts, stops)]
    total_ms = max_over_ranks(sum(step_ms), world, device)
    ms_per_step = total_ms / args.steps
    value = world * args.steps / (total_ms / 1e3)

    # End to end through the public host-buffer entry point (copies inside the timing).
    xh = x.cpu().pin_memory()
    yh = torch.empty(model.hidden, dtype=torch.float32).pin_memory()
    for _ in range(3):
        st.forward_host(xh, yh)
    barrier(world, device)
    e2e_steps = max(3, args.steps)
    t0 = time.perf_counter()
    for i in range(e2e_steps):
        st.forward_host(xh, yh)
    e2e_s = max_over_ranks(time.perf_counter() - t0, world, device)
    e2e_value = world * e2e_steps / e2e_s

    hbm_peak, peak_kind = peaks()
    achieved = nbytes / (ms_per_step / 1e3) / 1e9
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "data": "synthetic",
        "config": {"workload": describe(args.workload), "bits_per_weight": bpw,
                   "bytes_per_token": nbytes, "parallelism": f"replicas{world}",
                   "l2": "flushed between steps" if flush is not None
                   else "working set larger than L2", "signs": "uniform random bits"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                     "frac": achieved / hbm_peak, "traffic": None,
                     "peak_source": peak_kind, "kernel": "stack_program_kernel"},
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": 2 * model.hidden,
                "d2h_bytes_per_step": 4 * model.hidden},
        "gpu_launches": args.steps,
        "clocks": clocks.summary(),
        "wall_s": t_wall,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, cores, sample = cpu_oracle_rate(args.workload)
        line["cpu_baseline"] = {"value": rate, "unit": "tokens/s", "cores": cores,
                                "kind": "oracle", "sample": sample}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
