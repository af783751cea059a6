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
import hashlib
import json
import os
import statistics
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
    # single linears through lb_linear_forward: (in, out), bits/weight, M rows of x
    "prefill-gate7b-1.0-M4096": ((4096, 11008), 1.0, "linear", 4096),
    "prefill-gate7b-0.1-M4096": ((4096, 11008), 0.1, "linear", 4096),
    "prefill-gate7b-1.0-M512": ((4096, 11008), 1.0, "linear", 512),
    "decode-gate70b-1.0-M1": ((8192, 28672), 1.0, "linear", 1),
}
METRIC = "batch-1 layer-stack tokens/s"
L2_BYTES = 126 * 1024 * 1024


# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of one launch of
# a workload's dominant kernel, from the ncu captures summarised in profiles/.
# A figure is reported only while the kernel's sources hash to the value it
# was captured with (otherwise the line carries null).  Stack figures come
# from a capture of a shorter stack of the same layers and are scaled by the
# layer count: every layer reads its own weights once, so traffic grows in
# proportion.  workload: (sources hash, bytes per captured launch, layers
# captured, or 0 for a single linear).
MEASURED_TRAFFIC = {
    "stack70b-1.0": ("2038467ba1b45bad", 214971136 + 3177984, 2),
    "prefill-gate7b-1.0-M4096": ("1504e09a31a2c770", 53246208 + 144017664, 0),
    "prefill-gate7b-0.1-M4096": ("1504e09a31a2c770", 34988544 + 138443776, 0),
}
KERNEL_SOURCES = {
    "stack_program_kernel": ("lb_decode.cu", "lb_internal.cuh"),
    "linear_program_kernel": ("lb_decode.cu", "lb_internal.cuh"),
    "prefill_gemm_kernel": ("lb_prefill.cu", "lb_internal.cuh"),
}


def kernel_hash(kernel: str) -> str:
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "binary_rank_linear_lb_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def measured_traffic(workload: str, kernel: str, n_layers: int):
    rec = MEASURED_TRAFFIC.get(workload)
    if rec is None or rec[0] != kernel_hash(kernel):
        return None
    src, nbytes, layers = rec
    return nbytes * n_layers / layers if layers else float(nbytes)


def describe(name: str, n_layers: int = 0) -> str:
    model, bpw, kind = WORKLOADS[name][:3]
    if kind == "linear":
        (i, o), M = model, WORKLOADS[name][3]
        return f"one factorised linear {i}->{o}, {bpw} bits/weight, 2 branches, M={M} rows of x"
    if kind == "mlp":
        return f"{model} MLP block (gate, up 4096->11008, down 11008->4096), {bpw} bits/weight, batch 1"
    layers = f"{n_layers} layers" if n_layers else "all layers"
    return f"{model} decoder linear stack, {layers}, {bpw} bits/weight, 2 branches, batch 1"


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
    """Samples SM clocks and throttle reasons through NVML while the timed loop runs."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, device_index: int, period_s: float = 0.002):
        self.index = device_index
        self.period = period_s
        self.samples = []
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None

    def _handle(self, nv):
        import torch
        props = torch.cuda.get_device_properties(self.index)
        uuid = str(getattr(props, "uuid", ""))
        for cand in (uuid, "GPU-" + uuid):
            try:
                return nv.nvmlDeviceGetHandleByUUID(cand)
            except Exception:
                pass
        bus = "%08x:%02x:%02x.0" % (getattr(props, "pci_domain_id", 0), props.pci_bus_id,
                                    props.pci_device_id)
        return nv.nvmlDeviceGetHandleByPciBusId(bus)

    def __enter__(self):
        try:
            import pynvml as nv
            nv.nvmlInit()
            h = self._handle(nv)
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)

            def run():
                while not self._stop.is_set():
                    try:
                        sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                        rs = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                        self.samples.append((sm, rs))
                    except Exception:
                        pass
                    time.sleep(self.period)
            self._thread = threading.Thread(target=run, daemon=True)
            self._thread.start()
        except Exception:
            self._thread = None
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._thread is not None:
            self._thread.join(timeout=5)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        reasons = set()
        for _, rs in self.samples:
            for bit, name in self.REASONS.items():
                if rs & bit:
                    reasons.add(name)
        return {"sm_mhz": statistics.median(s for s, _ in self.samples),
                "sm_max_mhz": self.max_mhz, "reasons": sorted(reasons),
                "samples": len(self.samples)}


# ---------------------------------------------------------------- workloads
class LinearStep:
    """One lb_linear_forward call on M rows, shaped like a stack for the timing loop."""

    def __init__(self, in_f, out_f, r, M, device, seed):
        import torch
        import binary_rank_linear_lb_b200 as lb
        from binary_rank_linear_lb_b200 import synth
        from binary_rank_linear_lb_b200.model import build_linear
        self.lb, self.in_f, self.out_f, self.r, self.M = lb, in_f, out_f, r, M
        self.brs = build_linear(in_f, out_f, r, base=seed, device=device, signs="bits")
        self.x = synth.activation((M, in_f), seed + 1, torch.bfloat16, device)
        self.y = torch.empty((M, out_f), dtype=torch.float32, device=device)
        self.ws = torch.empty(lb.linear_workspace_size(M, in_f, out_f, r, 2), dtype=torch.uint8,
                              device=device)
        self.hidden = in_f

    def forward(self, x=None, y=None):
        return self.lb.linear_forward(self.x, self.brs, self.in_f, self.out_f, self.r, y=self.y,
                                      workspace=self.ws)

    def forward_host(self, xh, yh):
        import torch
        self.x.copy_(xh.view(self.M, self.in_f), non_blocking=True)
        self.forward()
        yh.view(self.M, self.out_f).copy_(self.y, non_blocking=True)
        torch.cuda.current_stream().synchronize()

    def status(self):
        return self.lb.workspace_status(self.ws)


def build_workload(name: str, device, seed: int, n_layers: int = 0):
    from binary_rank_linear_lb_b200.configs import MODELS, linear_bytes, linear_flops, rank_for
    from binary_rank_linear_lb_b200.model import build_mlp_block, build_stack
    model_name, bpw, kind = WORKLOADS[name][:3]
    if kind == "linear":
        (i, o), M = model_name, WORKLOADS[name][3]
        r = rank_for(bpw, i, o)
        st = LinearStep(i, o, r, M, device, seed)
        nbytes = linear_bytes(i, o, r) + M * i * 2 + M * o * 4
        st.flops = linear_flops(M, i, o, r)
        return st, st, bpw, kind, nbytes
    model = MODELS[model_name]
    if kind == "mlp":
        st = build_mlp_block(model, bpw, base=seed, device=device, signs="bits")
        nbytes = sum(linear_bytes(*model.shapes()[p], model.ranks(bpw)[p]) for p in (4, 5, 6))
    else:
        nl = n_layers or model.n_layers
        st = build_stack(model, bpw, base=seed, n_layers=nl, device=device, signs="bits")
        nbytes = model.bytes_per_token(bpw, nl)
    return st, model, bpw, kind, nbytes


def peaks():
    """(HBM GB/s, dense bf16 TFLOP/s, source) from the measured peaks file."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(path))
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    except (OSError, KeyError, ValueError):
        return 6650.0, 1590.0, "fallback"


def oracle_sampler(name: str):
    """One bounded sample of a workload for the oracle on the host cores.

    Returns (step, tokens per step, what one step is): a stack step is one decoder
    layer of one token (1/n_layers of a token), an MLP-block step one whole token, a
    single-linear step one row of x.  The packed words and scales are drawn once
    (uniform bits, |N(1, 0.1)| scales), outside the steps."""
    import numpy as np
    import oracle
    from oracle import stack as ostack
    from binary_rank_linear_lb_b200.configs import MODELS, rank_for
    model_name, bpw, kind = WORKLOADS[name][:3]
    rng = np.random.default_rng(0)

    def branches(i, o, r):
        brs = []
        for _ in range(2):
            Vp = rng.integers(0, 2 ** 32, size=(r, (i + 31) // 32), dtype=np.uint64).astype(np.uint32)
            Up = rng.integers(0, 2 ** 32, size=(o, (r + 31) // 32), dtype=np.uint64).astype(np.uint32)
            sc = lambda n: np.abs(1 + 0.1 * rng.standard_normal(n))
            brs.append(oracle.Branch(Vp, Up, sc(o), sc(i), sc(r)))
        return brs

    if kind == "linear":
        (i, o), M = model_name, WORKLOADS[name][3]
        r = rank_for(bpw, i, o)
        brs = branches(i, o, r)
        xs = rng.standard_normal((1, i))
        return (lambda: oracle.forward(xs, brs, i, o, r)), 1.0, (
            f"one row of x through the {i}->{o} layer (r={r}, 2 branches)")
    model = MODELS[model_name]
    rk = model.ranks(bpw)

    def lin(p):
        i, o = model.shapes()[p]
        return ostack.Linear(branches(i, o, rk[p]), i, o, rk[p])

    x = rng.standard_normal(model.hidden)
    if kind == "mlp":
        g, u, d = lin(4), lin(5), lin(6)
        return (lambda: ostack.mlp_block(x, g, u, d)), 1.0, "one token through the MLP block"
    L = {n: lin(p) for p, n in enumerate(("q", "k", "v", "o", "gate", "up", "down"))}
    return ((lambda: ostack.decoder_stack(x, [L], model.n_heads, model.n_kv_heads,
                                          model.head_dim)),
            1.0 / model.n_layers,
            f"one decoder layer of one token (1/{model.n_layers} of a token)")


def cpu_oracle_rate(name: str, budget_s: float = 12.0):
    """Oracle tokens/s from repeated bounded samples, about budget_s seconds in all."""
    import oracle
    step, tokens, what = oracle_sampler(name)
    step()
    n, t0 = 0, time.perf_counter()
    while True:
        step()
        n += 1
        if time.perf_counter() - t0 > budget_s or n >= 1000:
            break
    dt = (time.perf_counter() - t0) / n
    return tokens / dt, oracle.threads(), f"{n} timed samples, each {what}"


# ---------------------------------------------------------------- sweeps
def _time_events(fn, iters, flush=None):
    """Median device time (ms) of fn() over iters runs, L2 flushed before each."""
    import torch
    ts = []
    for _ in range(iters):
        if flush is not None:
            flush.fill_(1)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        b.synchronize()
        ts.append(a.elapsed_time(b))
    return statistics.median(ts)


def sweep_prefill(device, flush, tflops_peak, fp8_peak=None):
    """The 7B gate projection (4096 -> 11008) over the token batch M, both paths."""
    import torch
    import binary_rank_linear_lb_b200 as lb
    from binary_rank_linear_lb_b200 import synth
    from binary_rank_linear_lb_b200.configs import linear_bytes, linear_flops, rank_for
    from binary_rank_linear_lb_b200.model import build_linear
    in_f, out_f = 4096, 11008
    out = []
    for bpw in (1.0, 0.1):
        r = rank_for(bpw, in_f, out_f)
        brs = build_linear(in_f, out_f, r, base=77, device=device, signs="bits")
        for M in (1, 8, 64, 512, 4096):
            x = synth.activation((M, in_f), 5, torch.bfloat16, device)
            y = torch.empty((M, out_f), dtype=torch.float32, device=device)
            ws = torch.empty(lb.linear_workspace_size(M, in_f, out_f, r, 2), dtype=torch.uint8,
                             device=device)
            fn = lambda: lb.linear_forward(x, brs, in_f, out_f, r, y=y, workspace=ws)
            for _ in range(3):
                fn()
            ms = _time_events(fn, 10, flush)
            fl = linear_flops(M, in_f, out_f, r)
            by = linear_bytes(in_f, out_f, r) + M * in_f * 2 + M * out_f * 4
            out.append({"bits_per_weight": bpw, "r": r, "M": M,
                        "path": "tcgen05" if lb.linear_path(M, in_f, out_f, r) else "lut-decode",
                        "ms": ms, "tflops": fl / ms / 1e9, "gbs": by / ms / 1e6,
                        "tensor_frac_fp16": fl / ms / 1e9 / tflops_peak,
                        "tensor_frac_fp8": fl / ms / 1e9 / fp8_peak if fp8_peak else None})
            del x, y, ws
    return out


def measure_fp8_peak(device):
    """Dense FP8 (e4m3) matmul rate of the library GEMM, 8192^3, best of 10 (TFLOP/s).

    Plain library timing (torch._scaled_mm), the denominator of the FP8 tensor-core
    fraction; None with the reason if the call is not available."""
    import torch
    n = 8192
    try:
        a = torch.randn(n, n, device=device).to(torch.float8_e4m3fn)
        b = torch.randn(n, n, device=device).to(torch.float8_e4m3fn).t()
        one = torch.tensor(1.0, device=device)
        f = lambda: torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
        for _ in range(3):
            f()
        best = min(_time_events(f, 1) for _ in range(10))
        del a, b
        return {"fp8_tflops": 2 * n ** 3 / best / 1e9, "how": "torch._scaled_mm e4m3 8192^3, "
                "bf16 out, best of 10 (CUDA events)"}
    except Exception as e:   # pragma: no cover - depends on the library build
        return {"fp8_tflops": None, "how": f"torch._scaled_mm failed: {type(e).__name__}: {e}"}


def sweep_layer70b_vs_dense(device, flush, hbm_peak):
    """One 8192 -> 28672 factorised linear at batch 1 for each bits/weight, and a dense
    bf16 matrix-vector product of the same shape (torch.matmul over 470 MB of weights;
    a library call, context only).  L2 flushed before every timed call."""
    import torch
    import binary_rank_linear_lb_b200 as lb
    from binary_rank_linear_lb_b200 import synth
    from binary_rank_linear_lb_b200.configs import linear_bytes, rank_for
    from binary_rank_linear_lb_b200.model import build_linear
    in_f, out_f = 8192, 28672
    W = torch.randn(out_f, in_f, device=device, dtype=torch.bfloat16)
    xd = torch.randn(in_f, 1, device=device, dtype=torch.bfloat16)
    for _ in range(3):
        torch.matmul(W, xd)
    dense_ms = _time_events(lambda: torch.matmul(W, xd), 20, flush)
    dense_bytes = W.numel() * 2
    del W
    torch.cuda.empty_cache()
    rows = []
    for bpw in (1.0, 0.55, 0.3, 0.1):
        r = rank_for(bpw, in_f, out_f)
        brs = build_linear(in_f, out_f, r, base=31, device=device, signs="bits")
        x = synth.activation((1, in_f), 5, torch.bfloat16, device)
        y = torch.empty((1, out_f), dtype=torch.float32, device=device)
        ws = torch.empty(lb.linear_workspace_size(1, in_f, out_f, r, 2), dtype=torch.uint8,
                         device=device)
        fn = lambda: lb.linear_forward(x, brs, in_f, out_f, r, y=y, workspace=ws)
        for _ in range(3):
            fn()
        ms = _time_events(fn, 20, flush)
        # the bit-serial (XOR / popcount) variant of the same layer, 16 bit-planes
        xws = torch.empty(lb.lib().lb_linear_xor_workspace_size(1, in_f, out_f, r, 2, 16),
                          dtype=torch.uint8, device=device)
        fx = lambda: lb.linear_forward_xor(x, brs, in_f, out_f, r, bits=16, y=y, workspace=xws)
        for _ in range(3):
            fx()
        xor_ms = _time_events(fx, 20, flush)
        by = linear_bytes(in_f, out_f, r)
        rows.append({"bits_per_weight": bpw, "r": r, "ms": ms, "bytes": by,
                     "gbs": by / ms / 1e6, "hbm_frac": by / ms / 1e6 / hbm_peak,
                     "speedup_vs_dense_bf16": dense_ms / ms, "xor_popcount_ms": xor_ms})
        del brs, x, y, ws, xws
    return {"dense_bf16_ms": dense_ms, "dense_bf16_gbs": dense_bytes / dense_ms / 1e6,
            "layers": rows,
            "pages": "A100, same layer shape: speed-up grows as bits/weight fall, up to 11.6x"}


def sweep_small_m(device, flush):
    """The 7B gate projection at M = 1..16, 24, 32, 48, 64 rows on both kernel paths
    (LB_LINEAR_PATH forces one), and the path lb_linear_forward picks by itself."""
    import torch
    import binary_rank_linear_lb_b200 as lb
    from binary_rank_linear_lb_b200 import synth
    from binary_rank_linear_lb_b200.configs import rank_for
    from binary_rank_linear_lb_b200.model import build_linear
    in_f, out_f = 4096, 11008
    out = []
    for bpw in (1.0, 0.1):
        r = rank_for(bpw, in_f, out_f)
        brs = build_linear(in_f, out_f, r, base=78, device=device, signs="bits")
        for M in list(range(1, 17)) + [24, 32, 48, 64]:
            x = synth.activation((M, in_f), 6, torch.bfloat16, device)
            y = torch.empty((M, out_f), dtype=torch.float32, device=device)
            rec = {"bits_per_weight": bpw, "r": r, "M": M}
            for path, key in ((None, "default_ms"), ("0", "lut_ms"), ("1", "tensor_ms")):
                if path is None:
                    os.environ.pop("LB_LINEAR_PATH", None)
                    rec["default_path"] = "tcgen05" if lb.linear_path(M, in_f, out_f, r) else "lut"
                else:
                    os.environ["LB_LINEAR_PATH"] = path
                ws = torch.empty(lb.linear_workspace_size(M, in_f, out_f, r, 2),
                                 dtype=torch.uint8, device=device)
                fn = lambda: lb.linear_forward(x, brs, in_f, out_f, r, y=y, workspace=ws)
                for _ in range(3):
                    fn()
                rec[key] = _time_events(fn, 10, flush)
                del ws
            os.environ.pop("LB_LINEAR_PATH", None)
            rec["default_over_best"] = rec["default_ms"] / min(rec["lut_ms"], rec["tensor_ms"])
            out.append(rec)
    return out


def sweep_dual_svid(device):
    """Dual-SVID initialisation (lb_dual_svid) of the 7B gate shape (11008 x 4096) from a
    seeded N(0, 0.02^2) dense weight, at 1.0 and 0.1 bits/weight: seconds, and the
    initialised layer's output error against the dense layer on 64 N(0, 1) rows,
    ||y - W x|| / ||W x||."""
    import torch
    import binary_rank_linear_lb_b200 as lb
    from binary_rank_linear_lb_b200.configs import rank_for
    out_f, in_f = 11008, 4096
    g = torch.Generator(device=device)
    g.manual_seed(2024)
    W = 0.02 * torch.randn((out_f, in_f), generator=g, device=device)
    x = torch.randn((64, in_f), generator=g, device=device)
    y_ref = x @ W.T
    rows = []
    for bpw in (1.0, 0.1):
        r = rank_for(bpw, in_f, out_f)
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        brs = lb.dual_svid(W, r, 2)
        torch.cuda.synchronize()
        dt = time.perf_counter() - t0
        y = lb.linear_forward(x, brs, in_f, out_f, r)
        err = (torch.linalg.norm(y - y_ref) / torch.linalg.norm(y_ref)).item()
        rows.append({"bits_per_weight": bpw, "r": r, "seconds": dt, "layer_output_rel_err": err})
        del brs
    return {"shape": [out_f, in_f], "weight": "N(0, 0.02^2), seed 2024", "runs": rows}


def sweep_stacks(device, skip: str, hbm_peak):
    """tokens/s of the other stack workloads (fewer steps; same timing rules)."""
    import torch
    from binary_rank_linear_lb_b200 import synth
    out = {}
    for name in ("stack70b-1.0", "stack70b-0.55", "stack13b-0.55", "stack13b-0.1", "mlp7b-1.0",
                 "mlp7b-0.55", "mlp7b-0.3", "mlp7b-0.1"):
        if name == skip:
            continue
        st, model, bpw, kind, nbytes = build_workload(name, device, 99)
        x = synth.activation(model.hidden, 3, torch.bfloat16, device)
        y = torch.empty(model.hidden, dtype=torch.float32, device=device)
        flush = None
        if nbytes < 2 * L2_BYTES:
            flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=device)
        for _ in range(3):
            st.forward(x, y)
        ms = _time_events(lambda: st.forward(x, y), 10, flush)
        out[name] = {"tokens_per_s": 1e3 / ms, "ms_per_token": ms, "bytes_per_token": nbytes,
                     "gbs": nbytes / ms / 1e6, "hbm_frac": nbytes / ms / 1e6 / hbm_peak}
        del st, flush
        torch.cuda.empty_cache()
    return out


# ---------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="stack70b-1.0", choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--layers", type=int, default=0,
                    help="decoder layers (default: all); fewer only for profiling captures")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-sweep", action="store_true",
                    help="skip the extra sweeps (prefill M sweep, other stacks) on rank 0")
    args = ap.parse_args()
    world, rank, local = dist_env()
    if args.warmup < 3:
        args.warmup = 3

    if args.impl == "reference":
        # The reference arm is the oracle itself (no installable reference exists),
        # run on the host cores by rank 0 only.  Each step is one bounded sample of
        # the workload (see oracle_sampler); value is tokens/s from the timed steps.
        if rank != 0:
            return 0
        import oracle
        step, tokens, what = oracle_sampler(args.workload)
        for _ in range(args.warmup):
            step()
        t0 = time.perf_counter()
        for _ in range(args.steps):
            step()
        ms_per_step = (time.perf_counter() - t0) * 1e3 / args.steps
        rate = tokens / (ms_per_step / 1e3)
        sample = f"each step is {what}; value = tokens per step / time per step"
        line = {"impl": "reference", "metric": METRIC, "value": rate, "unit": "tokens/s",
                "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": ms_per_step, "tokens_per_step": tokens,
                "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": {"workload": describe(args.workload)},
                "cpu_baseline": {"value": rate, "unit": "tokens/s", "cores": oracle.threads(),
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

    st, model, bpw, kind, nbytes = build_workload(args.workload, device, args.seed + rank,
                                                  args.layers)
    if kind == "linear":
        x, y, tokens = st.x, st.y, st.M
    else:
        x = synth.activation(model.hidden, 1234 + rank, torch.bfloat16, device)
        y = torch.empty(model.hidden, dtype=torch.float32, device=device)
        tokens = 1
    stream = torch.cuda.current_stream(device)
    flush = None
    if nbytes < 2 * L2_BYTES:
        flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=device)

    for _ in range(args.warmup):
        st.forward(x, y)
    torch.cuda.synchronize(device)
    if st.status() != lb.LB_OK:
        raise RuntimeError("device-side wait timed out during warm-up")

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    stops = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    barrier(world, device)
    torch.cuda.synchronize(device)
    with ClockSampler(device.index) as clocks:
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
    value = world * args.steps * tokens / (total_ms / 1e3)

    # End to end through the public host-buffer entry point (copies inside the timing).
    xh = x.cpu().pin_memory()
    yh = torch.empty(tuple(y.shape), dtype=torch.float32).pin_memory()
    for _ in range(3):
        st.forward_host(xh, yh)
    barrier(world, device)
    e2e_steps = max(3, args.steps)
    t0 = time.perf_counter()
    for i in range(e2e_steps):
        st.forward_host(xh, yh)
    e2e_s = max_over_ranks(time.perf_counter() - t0, world, device)
    e2e_value = world * e2e_steps * tokens / e2e_s

    hbm_peak, tflops_peak, peak_kind = peaks()
    achieved = nbytes / (ms_per_step / 1e3) / 1e9
    roof = {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
            "frac": achieved / hbm_peak, "traffic": None, "peak_source": peak_kind,
            "kernel": "stack_program_kernel"}
    launches = args.steps                    # stacks: one cooperative launch per token
    if kind == "linear":
        # the tensor-core path launches lmax, pre-pass and GEMM kernels; the lookup-table
        # path one kernel per chunk of up to 8 rows
        launches = args.steps * (3 if lb.linear_path(st.M, st.in_f, st.out_f, st.r)
                                 else (st.M + 7) // 8)
        if lb.linear_path(st.M, st.in_f, st.out_f, st.r):
            tf = st.flops / (ms_per_step / 1e3) / 1e12
            roof = {"bound": "tensor", "achieved": tf, "peak": tflops_peak, "unit": "TFLOP/s",
                    "frac": tf / tflops_peak, "traffic": None,
                    "peak_source": peak_kind + " (bf16 dense; fp16 runs at the same rate)",
                    "kernel": "prefill_gemm_kernel"}
            fp8 = measure_fp8_peak(device)
            if fp8["fp8_tflops"]:
                roof["fp8_frac"] = tf / fp8["fp8_tflops"]
                roof["fp8_peak"] = fp8
        else:
            roof["kernel"] = "linear_program_kernel"
    roof["traffic"] = measured_traffic(args.workload, roof["kernel"],
                                       getattr(st, "n_layers", 0))
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "data": "synthetic",
        "config": {"workload": describe(args.workload, args.layers), "bits_per_weight": bpw,
                   "bytes_per_token": nbytes, "parallelism": f"replicas{world}",
                   "l2": "flushed between steps" if flush is not None
                   else "working set larger than L2", "signs": "uniform random bits"},
        "roofline": roof,
        "e2e": {"value": e2e_value, "unit": "tokens/s",
                "h2d_bytes_per_step": xh.numel() * xh.element_size(),
                "d2h_bytes_per_step": yh.numel() * yh.element_size()},
        "gpu_launches": launches,
        "clocks": clocks.summary(),
        "wall_s": t_wall,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, cores, sample = cpu_oracle_rate(args.workload)
        line["cpu_baseline"] = {"value": rate, "unit": "tokens/s", "cores": cores,
                                "kind": "oracle", "sample": sample}
    if rank == 0 and world == 1 and not args.no_sweep:
        del st
        torch.cuda.empty_cache()
        flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=device)
        fp8 = measure_fp8_peak(device)
        line["sweeps"] = {
            "peaks": {"hbm_gbs": hbm_peak, "fp16_tflops": tflops_peak, "source": peak_kind,
                      "fp8_tflops_measured": fp8["fp8_tflops"], "fp8_how": fp8["how"]},
            "prefill_gate7b": sweep_prefill(device, flush, tflops_peak, fp8["fp8_tflops"]),
            "small_m_gate7b": sweep_small_m(device, flush),
            "layer70b_vs_dense": sweep_layer70b_vs_dense(device, flush, hbm_peak),
            "dual_svid_gate7b": sweep_dual_svid(device),
            "stacks": sweep_stacks(device, args.workload, hbm_peak),
        }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
