"""lb_linear_forward against the oracle (GPU).

Bar: max|y - y_ref| <= 2e-3 * max|y_ref| per output tensor (fp32 outputs).
"""
import numpy as np
import pytest
import torch

import oracle
import binary_rank_linear_lb_b200 as lb
from binary_rank_linear_lb_b200 import synth
from binary_rank_linear_lb_b200.configs import SINGLE, rank_for
from binary_rank_linear_lb_b200.model import build_linear

from helpers import assert_close, oracle_linear, to_f64

pytestmark = pytest.mark.gpu


def run_case(in_f, out_f, r, M, dtype, nb=2, base=0, rows=None, layout=lb.LB_LAYOUT_SLICES):
    brs = build_linear(in_f, out_f, r, base=base, n_branches=nb, layout=layout)
    x = synth.activation((M, in_f), synth.tensor_seed(base, 0, 0, 0, synth.KIND_X), dtype, "cuda")
    y = lb.linear_forward(x, brs, in_f, out_f, r)
    torch.cuda.synchronize()
    ob = oracle_linear(in_f, out_f, r, base, 0, 0, nb)
    y_ref = oracle.forward(to_f64(x), ob, in_f, out_f, r, rows=rows)
    got = y.cpu().numpy().astype(np.float64)
    if rows is not None:
        got = got[:, rows]
    return got, y_ref


def test_single_linear_config():
    """in 512, out 256, r 32, two branches, M = 1, fp16 x."""
    got, ref = run_case(SINGLE["in_f"], SINGLE["out_f"], SINGLE["r"], 1, torch.float16)
    assert_close(got, ref, what="single")


@pytest.mark.parametrize("shape", [(1, 1, 1), (32, 32, 32), (100, 33, 7), (1000, 300, 70),
                                   (1024, 1024, 1024), (1100, 2100, 1088), (300, 5000, 2100)])
@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16, torch.float32])
@pytest.mark.parametrize("layout", [lb.LB_LAYOUT_SLICES, lb.LB_LAYOUT_ROWS])
def test_ragged_shapes(shape, dtype, layout):
    got, ref = run_case(*shape, M=1, dtype=dtype, layout=layout)
    assert_close(got, ref, what=str(shape))


def test_rows_layout_unpadded_pitch():
    """Row-major weights with the unpadded pitch ceil(k/32) (odd and 2-word pitches)."""
    for in_f, out_f, r in ((1000, 300, 70), (640, 2100, 60), (96, 64, 33)):
        brs = [b for b in build_linear(in_f, out_f, r, base=9, layout=lb.LB_LAYOUT_ROWS, pad=False)]
        x = synth.activation((1, in_f), 90, torch.bfloat16, "cuda")
        y = lb.linear_forward(x, brs, in_f, out_f, r)
        torch.cuda.synchronize()
        ref = oracle.forward(to_f64(x), oracle_linear(in_f, out_f, r, 9, 0, 0), in_f, out_f, r)
        assert_close(y.cpu().numpy(), ref, what=f"unpadded {in_f, out_f, r}")


@pytest.mark.parametrize("M", [2, 3, 8, 11])
def test_small_batches(M):
    got, ref = run_case(777, 513, 96, M, torch.bfloat16)
    for m in range(M):
        assert_close(got[m], ref[m], what=f"row {m}")


def test_one_branch():
    got, ref = run_case(640, 320, 64, 1, torch.bfloat16, nb=1)
    assert_close(got, ref, what="one branch")


@pytest.mark.parametrize("bpw", [1.0, 0.55, 0.3, 0.1])
@pytest.mark.parametrize("shape", [(4096, 11008), (11008, 4096)])
def test_7b_mlp_shapes(shape, bpw):
    r = rank_for(bpw, *shape)
    got, ref = run_case(shape[0], shape[1], r, 1, torch.bfloat16, base=1)
    assert_close(got, ref, what=f"{shape} @ {bpw}")


@pytest.mark.parametrize("shape", [(8192, 28672, 3136), (28672, 8192, 3136), (8192, 1024, 448)])
def test_70b_shapes_sampled_rows(shape):
    """Full-size 70B linears; the oracle evaluates 96 sampled output rows."""
    rng = np.random.default_rng(shape[1])
    rows = np.sort(rng.choice(shape[1], size=96, replace=False)).tolist()
    rows[-1] = shape[1] - 1
    got, ref = run_case(*shape, M=1, dtype=torch.bfloat16, base=2, rows=rows)
    # the tolerance is relative to max|y_ref| over the sampled rows
    assert_close(got, ref, what=f"70B {shape}")


def test_workspace_reports_ok_and_repeat_calls_agree():
    in_f, out_f, r = 2048, 1536, 256
    brs = build_linear(in_f, out_f, r)
    x = synth.activation((1, in_f), 7, torch.bfloat16, "cuda")
    ws = torch.empty(lb.linear_workspace_size(1, in_f, out_f, r, 2), dtype=torch.uint8,
                     device="cuda")
    y1 = lb.linear_forward(x, brs, in_f, out_f, r, workspace=ws).clone()
    y2 = lb.linear_forward(x, brs, in_f, out_f, r, workspace=ws)
    assert lb.workspace_status(ws) == lb.LB_OK
    torch.testing.assert_close(y1, y2, rtol=1e-5, atol=1e-4 * y1.abs().max().item())


# ---------------------------------------------------------------- tensor-core path
@pytest.mark.parametrize("shape", [(512, 256, 64), (640, 1000, 192), (1024, 1001, 128),
                                   (4096, 11008, 128)])
@pytest.mark.parametrize("M", [17, 100, 256])
@pytest.mark.parametrize("layout", [lb.LB_LAYOUT_SLICES, lb.LB_LAYOUT_ROWS])
def test_prefill_path_shapes(shape, M, layout):
    in_f, out_f, r = shape
    assert lb.linear_path(M, in_f, out_f, r) == 1
    got, ref = run_case(in_f, out_f, r, M, torch.bfloat16, base=3, layout=layout)
    for m in (0, M // 2, M - 1):
        assert_close(got[m], ref[m], what=f"{shape} M={M} row {m}")
    assert_close(got, ref, what=f"{shape} M={M}")


@pytest.mark.parametrize("subtiles", ["1", "2"])
@pytest.mark.parametrize("M", [129, 300, 520])
@pytest.mark.parametrize("shape", [(640, 1000, 192), (1024, 1001, 128)])
def test_prefill_subtile_shapes(shape, M, subtiles, monkeypatch):
    """Both tile shapes of the tensor-core GEMMs (one or two 128-row M sub-tiles per
    expanded sign tile), with M ragged inside the first or second sub-tile."""
    monkeypatch.setenv("LB_PREFILL_SUBTILES", subtiles)
    in_f, out_f, r = shape
    got, ref = run_case(in_f, out_f, r, M, torch.bfloat16, base=7, layout=lb.LB_LAYOUT_SLICES)
    assert_close(got, ref, what=f"{shape} M={M} sub-tiles={subtiles}")


@pytest.mark.parametrize("split2", ["1", "2", "3", "4"])
@pytest.mark.parametrize("subtiles", ["1", "2"])
@pytest.mark.parametrize("M,shape", [(64, (640, 1000, 192)), (300, (1024, 1001, 128)),
                                     (100, (512, 256, 64))])
def test_prefill_stage2_k_split(M, shape, subtiles, split2, monkeypatch):
    """The second GEMM split along K into 1-4 parts that add into y (vector and scalar
    reductions: out = 1001 is not a multiple of 4), with both tile shapes."""
    monkeypatch.setenv("LB_PREFILL_SUBTILES", subtiles)
    monkeypatch.setenv("LB_PREFILL_SPLIT2", split2)
    in_f, out_f, r = shape
    got, ref = run_case(in_f, out_f, r, M, torch.bfloat16, base=9, layout=lb.LB_LAYOUT_SLICES)
    assert_close(got, ref, what=f"{shape} M={M} sub-tiles={subtiles} split2={split2}")


@pytest.mark.parametrize("dtype", [torch.float16, torch.float32])
def test_prefill_path_dtypes_and_one_branch(dtype):
    got, ref = run_case(768, 512, 128, 64, dtype, nb=1, base=4)
    assert_close(got, ref, what=f"one branch {dtype}")


@pytest.mark.parametrize("bpw", [1.0, 0.1])
def test_prefill_7b_gate_sampled_rows(bpw):
    """7B gate projection at M = 512; the oracle evaluates all rows of 8 sampled tokens."""
    in_f, out_f = 4096, 11008
    r = rank_for(bpw, in_f, out_f)
    M = 512
    brs = build_linear(in_f, out_f, r, base=5)
    x = synth.activation((M, in_f), 55, torch.bfloat16, "cuda")
    y = lb.linear_forward(x, brs, in_f, out_f, r)
    torch.cuda.synchronize()
    ob = oracle_linear(in_f, out_f, r, 5, 0, 0, 2)
    toks = [0, 1, 127, 128, 255, 300, 510, 511]
    ref = oracle.forward(to_f64(x[toks]), ob, in_f, out_f, r)
    assert_close(y[toks].cpu().numpy(), ref, what=f"7B gate M=512 @ {bpw}")


def test_prefill_large_activations_do_not_overflow():
    """Rows of very different magnitude: the per-row powers of two keep fp16 in range."""
    in_f, out_f, r = 512, 512, 128
    brs = build_linear(in_f, out_f, r, base=6)
    x = synth.activation((32, in_f), 66, torch.float32, "cuda")
    x = x * torch.logspace(-20, 30, 32, base=2.0, device="cuda")[:, None]
    y = lb.linear_forward(x, brs, in_f, out_f, r)
    torch.cuda.synchronize()
    assert torch.isfinite(y).all()
    ob = oracle_linear(in_f, out_f, r, 6, 0, 0, 2)
    ref = oracle.forward(to_f64(x), ob, in_f, out_f, r)
    for m in range(32):
        assert_close(y[m].cpu().numpy(), ref[m], what=f"row {m}")


@pytest.mark.parametrize("bpw", [1.0, 0.1])
@pytest.mark.parametrize("M", [64, 4096])
def test_prefill_timed_7b_gate_every_m_block(M, bpw):
    """The 7B gate projection (4096 -> 11008) exactly as bench.py times it: seed 0, sign
    words drawn directly, the sliced layout, bf16 x from seed 1, one lb_linear_forward call
    (at M = 4096: 32 M blocks of 128 rows, no K split, stage-2 tiles waiting per block on
    their stage-1 rows).  The oracle evaluates every output feature of the first, a middle
    and the last row of every 128-row M block."""
    from helpers import oracle_branch_bits
    in_f, out_f = 4096, 11008
    r = rank_for(bpw, in_f, out_f)
    assert lb.linear_path(M, in_f, out_f, r) == 1
    brs = build_linear(in_f, out_f, r, base=0, signs="bits")
    x = synth.activation((M, in_f), 1, torch.bfloat16, "cuda")
    y = lb.linear_forward(x, brs, in_f, out_f, r)
    torch.cuda.synchronize()
    toks = sorted({t for b0 in range(0, M, 128)
                   for t in (b0, b0 + min(64, M - b0 - 1), min(b0 + 127, M - 1))})
    ob = [oracle_branch_bits(in_f, out_f, r, 0, 0, 0, b) for b in range(2)]
    ref = oracle.forward(to_f64(x[toks]), ob, in_f, out_f, r)
    got = y[toks].cpu().numpy().astype(np.float64)
    for i, t in enumerate(toks):
        assert_close(got[i], ref[i], what=f"7B gate M={M} @ {bpw}, token {t}")
    assert_close(got, ref, what=f"7B gate M={M} @ {bpw}")


@pytest.mark.parametrize("path", ["0", "1"])
@pytest.mark.parametrize("M", [1, 5, 8, 14, 15, 16, 24, 64])
def test_forced_paths_small_m(M, path, monkeypatch):
    """Both kernel paths at the token counts where lb_linear_forward switches between them
    (LB_LINEAR_PATH forces one: the tensor-core kernels also below 16 rows, the lookup-table
    kernels also above), on a 64-aligned shape with a ragged output width."""
    monkeypatch.setenv("LB_LINEAR_PATH", path)
    in_f, out_f, r = 1024, 1001, 192
    assert lb.linear_path(M, in_f, out_f, r) == int(path)
    got, ref = run_case(in_f, out_f, r, M, torch.bfloat16, base=12)
    for m in range(M):
        assert_close(got[m], ref[m], what=f"M={M} path={path} row {m}")


@pytest.mark.parametrize("M", [15, 16, 17])
def test_dispatch_threshold(M):
    """lb_linear_forward switches to the tensor cores at 16 rows (the measured crossover
    on the 7B gate shape); either side of the switch matches the oracle."""
    in_f, out_f, r = 4096, 11008, 128
    assert lb.linear_path(M, in_f, out_f, r) == (1 if M >= 16 else 0)
    assert lb.linear_path(M, 4000, out_f, r) == 0          # in not a multiple of 64
    got, ref = run_case(in_f, out_f, r, M, torch.bfloat16, base=13)
    for m in (0, M // 2, M - 1):
        assert_close(got[m], ref[m], what=f"M={M} row {m}")
