"""lb_stack_forward (decoder stacks and the 7B MLP block) against the oracle (GPU).

The oracle runs the whole stack itself from the same seeded inputs; no GPU
intermediate ever enters it.
"""
import time

import numpy as np
import pytest
import torch

import oracle
from oracle import stack as ostack
import binary_rank_linear_lb_b200 as lb
from binary_rank_linear_lb_b200 import synth
from binary_rank_linear_lb_b200.configs import LLAMA2_13B, LLAMA2_7B, LLAMA2_70B, Model
from binary_rank_linear_lb_b200.model import build_mlp_block, build_stack

from helpers import assert_close, oracle_branch_bits, oracle_linear, to_f64

pytestmark = pytest.mark.gpu


def oracle_layers(model: Model, ranks, n_layers, base):
    layers = []
    for li in range(n_layers):
        L = {}
        for p, name in enumerate(ostack_names()):
            i, o = model.shapes()[p]
            L[name] = ostack.Linear(oracle_linear(i, o, ranks[p], base, li, p), i, o, ranks[p])
        layers.append(L)
    return layers


def ostack_names():
    return ("q", "k", "v", "o", "gate", "up", "down")


def run_stack(model, bpw, n_layers, base, ranks=None, layout=lb.LB_LAYOUT_SLICES):
    rk = ranks or model.ranks(bpw)
    st = build_stack(model, bpw, base=base, n_layers=n_layers, ranks=rk, layout=layout)
    x = synth.activation(model.hidden, synth.tensor_seed(base, 0, 0, 0, synth.KIND_X),
                         torch.bfloat16, "cuda")
    y = st.forward(x)
    torch.cuda.synchronize()
    assert st.status() == lb.LB_OK
    layers = oracle_layers(model, rk, n_layers, base)
    h_ref, outs = ostack.decoder_stack(to_f64(x), layers, model.n_heads, model.n_kv_heads,
                                       model.head_dim, keep=True)
    return st, x, y, h_ref, outs


SMALL = Model("small", hidden=256, inter=512, n_layers=3, n_heads=4, n_kv_heads=2, head_dim=64)


def prefix_output(st, model, n_layers, x):
    """The residual stream after the first n_layers layers of GPU stack st: the same
    device-resident weights run as a stack of n_layers layers (x itself for 0)."""
    if n_layers == 0:
        return to_f64(x)
    rk = [[int(st._ranks[li * 7 + p]) for p in range(7)] for li in range(n_layers)]
    pre = lb.Stack(st._keep[:n_layers], rk, model.hidden, model.inter, model.n_heads,
                   model.n_kv_heads, model.head_dim)
    h = to_f64(pre.forward(x))
    torch.cuda.synchronize()
    assert pre.status() == lb.LB_OK
    return h


def check_layer_teacher_forced(st, model, li, h_in, h_out, L, what):
    """Every linear of layer li of a GPU stack run, each against the oracle fed with the
    GPU's own input to that linear (teacher-forced): q, k, v from rmsnorm(h_in); o from the
    GPU's v; gate, up from rmsnorm(h_in + o); down from the GPU's gate and up.  o and down
    add into the residual stream, so their sum is checked as h_out - h_in."""
    a = ostack.rmsnorm(h_in)
    got = {p: to_f64(st.output(li, i)) for i, p in ((0, "q"), (1, "k"), (2, "v"), (4, "gate"),
                                                      (5, "up"))}
    for name in ("q", "k", "v"):
        assert_close(got[name], L[name](a), what=f"{what} layer {li} {name}")
    o_ref = L["o"](ostack.gqa_broadcast(got["v"], model.n_heads, model.n_kv_heads,
                                        model.head_dim))
    a2 = ostack.rmsnorm(h_in + o_ref)
    for name in ("gate", "up"):
        assert_close(got[name], L[name](a2), what=f"{what} layer {li} {name}")
    down_ref = L["down"](ostack.silu(got["gate"]) * got["up"])
    assert_close(h_out - h_in, o_ref + down_ref, what=f"{what} layer {li} o + down")


@pytest.mark.parametrize("layout", [lb.LB_LAYOUT_SLICES, lb.LB_LAYOUT_ROWS])
def test_small_decoder_stack_and_intermediates(layout):
    st, x, y, h_ref, outs = run_stack(SMALL, 1.0, 3, base=3, ranks=[64, 32, 32, 64, 96, 96, 96],
                                      layout=layout)
    assert_close(y.cpu().numpy(), h_ref, what="small stack")
    for li in range(3):
        for p, name in ((0, "q"), (1, "k"), (2, "v"), (4, "gate"), (5, "up")):
            got = st.output(li, p).cpu().numpy()
            assert_close(got, outs[li][name], what=f"layer {li} {name}")


def test_forward_host_matches_device():
    st = build_stack(SMALL, 1.0, base=4, n_layers=2, ranks=[64, 32, 32, 64, 96, 96, 96])
    x = synth.activation(SMALL.hidden, 11, torch.bfloat16, "cuda")
    y = st.forward(x).cpu()
    xh = x.cpu().pin_memory()
    yh = torch.empty(SMALL.hidden, dtype=torch.float32).pin_memory()
    st.forward_host(xh, yh)
    torch.testing.assert_close(yh, y, rtol=1e-4, atol=1e-4 * y.abs().max().item())


def test_bounded_wait_gives_up_and_workspace_recovers():
    """A grid-wide wait that is never met ends in an error status, not a hang.  The
    arrival counter in the workspace header is preset so that phase 0's arrivals wrap it
    to zero, short of the first wait's target; each CTA gives up after its ~2 s bound, the
    call ends and the workspace reports LB_ERR_TIMEOUT.  The error is sticky (the next
    call returns at once) until the plan is prepared again, after which the stack gives
    the same result as before."""
    ranks = [64, 32, 32, 64, 96, 96, 96]
    st = build_stack(SMALL, 1.0, base=4, n_layers=2, ranks=ranks)
    x = synth.activation(SMALL.hidden, 11, torch.bfloat16, "cuda")
    y_ok = st.forward(x).clone()
    assert st.status() == lb.LB_OK
    grid = torch.cuda.get_device_properties(0).multi_processor_count
    st.workspace[:4].view(torch.int32)[0] = -grid          # 2^32 - G arrivals so far
    t0 = time.perf_counter()
    st.forward(x)
    assert st.status() == lb.LB_ERR_TIMEOUT
    assert time.perf_counter() - t0 < 30.0
    t0 = time.perf_counter()
    st.forward(x)                                           # sticky: returns at once
    assert st.status() == lb.LB_ERR_TIMEOUT
    assert time.perf_counter() - t0 < 1.0
    st.prepare()
    y = st.forward(x)
    assert st.status() == lb.LB_OK
    torch.testing.assert_close(y, y_ok, rtol=1e-5, atol=1e-5 * y_ok.abs().max().item())


def check_two_layer_stack(model, bpw, base, what):
    st, x, y, h_ref, _ = run_stack(model, bpw, 2, base=base)
    assert_close(y.cpu().numpy(), h_ref, what=what)
    layers = oracle_layers(model, model.ranks(bpw), 2, base)
    h1 = prefix_output(st, model, 1, x)
    check_layer_teacher_forced(st, model, 0, to_f64(x), h1, layers[0], what)
    check_layer_teacher_forced(st, model, 1, h1, to_f64(y), layers[1], what)


@pytest.mark.parametrize("bpw", [0.55, 0.1])
def test_13b_stack_two_layers_full_width(bpw):
    """The final hidden state, and every linear of both layers teacher-forced."""
    check_two_layer_stack(LLAMA2_13B, bpw, 5, f"13B x2 @ {bpw}")


@pytest.mark.slow
def test_13b_stack_full_depth_0p1():
    _, _, y, h_ref, _ = run_stack(LLAMA2_13B, 0.1, LLAMA2_13B.n_layers, base=6)
    assert_close(y.cpu().numpy(), h_ref, what="13B x40 @ 0.1")


@pytest.mark.slow
def test_70b_stack_two_layers_full_width():
    """The final hidden state, and every linear of both layers teacher-forced."""
    check_two_layer_stack(LLAMA2_70B, 0.55, 7, "70B x2 @ 0.55")


@pytest.mark.slow
def test_70b_stack_full_depth_bench_workload():
    """bench.py's default workload as it times it: all 80 layers of the 70B-shaped stack at
    1.0 bits/weight, two branches, sign words drawn directly, the sliced layout, one
    cooperative launch; the oracle runs the same seeded layers one at a time."""
    model, base = LLAMA2_70B, 0
    st = build_stack(model, 1.0, base=base, signs="bits")
    x = synth.activation(model.hidden, 1234, torch.bfloat16, "cuda")
    y = st.forward(x).cpu().numpy()
    torch.cuda.synchronize()
    assert st.status() == lb.LB_OK
    rk = model.ranks(1.0)

    def layer(li):
        L = {}
        for p, name in enumerate(ostack_names()):
            i, o = model.shapes()[p]
            L[name] = ostack.Linear([oracle_branch_bits(i, o, rk[p], base, li, p, b)
                                     for b in range(2)], i, o, rk[p])
        return L

    # every linear of the first and the last layer, teacher-forced
    last = model.n_layers - 1
    h_first = prefix_output(st, model, 1, x)
    h_last = prefix_output(st, model, last, x)
    what = "70B x80 @ 1.0, bench workload"
    check_layer_teacher_forced(st, model, 0, to_f64(x), h_first, layer(0), what)
    check_layer_teacher_forced(st, model, last, h_last, y.astype(np.float64), layer(last), what)
    del st
    torch.cuda.empty_cache()
    # and the final hidden state against the oracle run free from x
    h = to_f64(x)
    for li in range(model.n_layers):
        h = ostack.decoder_stack(h, [layer(li)], model.n_heads, model.n_kv_heads, model.head_dim)
    assert_close(y, h, what=what)


@pytest.mark.parametrize("bpw", [1.0, 0.55, 0.3, 0.1])
def test_7b_mlp_block(bpw):
    base = 8
    st = build_mlp_block(LLAMA2_7B, bpw, base=base)
    x = synth.activation(LLAMA2_7B.hidden, 13, torch.bfloat16, "cuda")
    y = st.forward(x)
    torch.cuda.synchronize()
    rk = LLAMA2_7B.ranks(bpw)
    mk = lambda p: ostack.Linear(oracle_linear(*LLAMA2_7B.shapes()[p], rk[p], base, 0, p),
                                 *LLAMA2_7B.shapes()[p], rk[p])
    ref = ostack.mlp_block(to_f64(x), mk(4), mk(5), mk(6))
    assert_close(y.cpu().numpy(), ref, what=f"7B MLP @ {bpw}")
