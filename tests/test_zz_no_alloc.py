"""lb_linear_forward_noalloc (GPU): the allocation-free entry point.

It exists for callers that cannot allocate device memory, so it takes its
scratch from a fixed array inside liblb.so.  Its results must match
lb_linear_forward's on the same inputs, call after call, even though every call
reuses (and leaves behind) the same array.  Collected last on purpose.
"""
import ctypes

import pytest
import torch

pytestmark = pytest.mark.gpu

TOL = 2e-3   # the bar every forward test uses: max|y - y_ref| <= TOL * max|y_ref|


def _rel(a, b):
    return ((a - b).abs().max() / b.abs().max()).item()


# (in, out, r, M): lookup-table shapes, and shapes lb_linear_forward runs on the tensor
# cores: the first two fit the fixed array there (stage 1 unsplit), the last one does not
# and runs the lookup-table kernels instead.
SHAPES = [(512, 256, 32, 1), (4096, 11008, 1472, 1), (777, 513, 96, 3),
          (512, 256, 64, 17), (4096, 11008, 1472, 17), (4096, 11008, 128, 64)]


@pytest.mark.parametrize("shape", SHAPES)
def test_noalloc_matches_workspace_entry_point_twice(shape):
    import binary_rank_linear_lb_b200 as lb
    from binary_rank_linear_lb_b200 import synth
    from binary_rank_linear_lb_b200.model import build_linear

    in_f, out_f, r, M = shape
    if M >= 16:
        assert lb.linear_path(M, in_f, out_f, r) == 1     # lb_linear_forward uses the tensor cores
    brs = build_linear(in_f, out_f, r, base=21, device="cuda")
    L = lb.lib()
    arr = (lb.lb_branch * 2)(*[b.c_struct() for b in brs])
    stream = torch.cuda.current_stream().cuda_stream
    outs = []
    for call in range(2):
        x = synth.activation((M, in_f), 100 + call, torch.bfloat16, "cuda")
        ref = lb.linear_forward(x, brs, in_f, out_f, r)
        y = torch.full((M, out_f), float("nan"), dtype=torch.float32, device="cuda")
        st = L.lb_linear_forward_noalloc(x.data_ptr(), lb.LB_BF16, M, in_f, out_f, r,
                                         ctypes.addressof(arr), 2, y.data_ptr(), stream)
        assert st == lb.LB_OK, lb.status_string(st)
        torch.cuda.synchronize()
        assert torch.isfinite(y).all()
        assert _rel(y, ref) <= TOL
        outs.append(y)
    assert not torch.equal(outs[0], outs[1])     # different inputs gave different outputs


def test_noalloc_rejects_sizes_beyond_its_scratch():
    import binary_rank_linear_lb_b200 as lb
    L = lb.lib()
    cap = L.lb_noalloc_scratch_bytes()
    r_too_big = cap // (4 * 2) + 64        # one row of x, two branches
    arr = (lb.lb_branch * 2)(lb.lb_branch(256, 256, 256, 256, 256),
                             lb.lb_branch(256, 256, 256, 256, 256))
    st = L.lb_linear_forward_noalloc(256, lb.LB_BF16, 1, 64, 64, r_too_big,
                                     ctypes.addressof(arr), 2, 256, None)
    assert st == lb.LB_ERR_WORKSPACE
