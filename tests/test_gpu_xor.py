"""lb_linear_forward_xor (the bit-serial XOR / popcount variant) against the oracle (GPU).

Both sides quantise the activations with the same fp32 decisions and sum integers
exactly, so the GPU result equals the oracle's up to the final fp32 rounding of
h * D2 * Z (bar: 1e-5 * max|y_ref|); against the float layer the quantisation
error stays inside the layer's 2e-3 bound at 16 bit-planes.
"""
import numpy as np
import pytest
import torch

import oracle
import binary_rank_linear_lb_b200 as lb
from binary_rank_linear_lb_b200 import synth
from binary_rank_linear_lb_b200.configs import rank_for
from binary_rank_linear_lb_b200.model import build_linear

from helpers import assert_close, oracle_linear, to_f64

pytestmark = pytest.mark.gpu


def run(in_f, out_f, r, M, dtype, bits, layout, nb=2, base=40):
    brs = build_linear(in_f, out_f, r, base=base, n_branches=nb, layout=layout)
    x = synth.activation((M, in_f), synth.tensor_seed(base, 0, 0, 0, synth.KIND_X), dtype, "cuda")
    y = lb.linear_forward_xor(x, brs, in_f, out_f, r, bits=bits)
    torch.cuda.synchronize()
    ob = oracle_linear(in_f, out_f, r, base, 0, 0, nb)
    xr = to_f64(x)
    return y.cpu().numpy().astype(np.float64), oracle.forward_xor(xr, ob, in_f, out_f, r, bits), \
        oracle.forward(xr, ob, in_f, out_f, r)


@pytest.mark.parametrize("shape,M,dtype", [((512, 256, 32), 1, torch.float16),
                                           ((1000, 300, 70), 3, torch.bfloat16),
                                           ((777, 513, 96), 2, torch.float32),
                                           ((4096, 11008, rank_for(1.0, 4096, 11008)), 1, torch.bfloat16)])
@pytest.mark.parametrize("layout", [lb.LB_LAYOUT_SLICES, lb.LB_LAYOUT_ROWS])
def test_xor_variant_matches_its_oracle(shape, M, dtype, layout):
    got, ref_xor, ref = run(*shape, M, dtype, 16, layout)
    for m in range(M):
        assert_close(got[m], ref_xor[m], tol=1e-5, what=f"{shape} row {m} vs bit-serial oracle")
        assert_close(got[m], ref[m], tol=2e-3, what=f"{shape} row {m} vs float oracle")


@pytest.mark.parametrize("bits", [1, 4, 8, 12, 24])
def test_xor_variant_other_bit_widths(bits):
    got, ref_xor, _ = run(640, 320, 64, 2, torch.bfloat16, bits, lb.LB_LAYOUT_SLICES, nb=1)
    for m in range(2):
        assert_close(got[m], ref_xor[m], tol=1e-5, what=f"bits={bits} row {m}")


def test_xor_variant_rejects_bad_bit_widths():
    brs = build_linear(64, 64, 32, base=41)
    x = torch.zeros((1, 64), dtype=torch.bfloat16, device="cuda")
    for bits in (0, 25):
        with pytest.raises(lb.LbError):
            lb.linear_forward_xor(x, brs, 64, 64, 32, bits=bits)
