"""lb_dual_svid (Dual-SVID initialisation on the GPU) against the oracle (GPU).

The SVD is unique only up to the signs of its singular-vector pairs, and the GPU's
is a randomized truncated one, so the tests compare what is unique: the branch a
set of signs and scales represents (diag(h) sign(U) diag(l) sign(V)^T diag(g)), the
signs after aligning each column pair, the scales, and the approximation error.
Weights with a clear spectral gap keep the leading singular vectors well defined.
"""
import numpy as np
import pytest
import torch

import binary_rank_linear_lb_b200 as lb
from oracle import dual_svid as ds

pytestmark = pytest.mark.gpu


def gapped_weight(out_f, in_f, r, seed):
    """Singular values 1 .. 0.1 for the first r, then a 30x drop (0.003 .. 0.001), plus
    a little noise: the rank-r subspace is well separated from the rest."""
    g = np.random.default_rng(seed)
    k = 2 * r
    A, _ = np.linalg.qr(g.standard_normal((out_f, k)))
    B, _ = np.linalg.qr(g.standard_normal((in_f, k)))
    sig = np.concatenate([np.geomspace(1.0, 0.1, r), np.geomspace(0.003, 0.001, k - r)])
    return (A * sig) @ B.T + 1e-5 * g.standard_normal((out_f, in_f)) / np.sqrt(in_f)




def signs_of(P, n, k, layout):
    w = P if layout == lb.LB_LAYOUT_ROWS else lb.unslice_words(P, n, k)
    bits = np.unpackbits(w.cpu().numpy().view(np.uint8).reshape(n, -1), axis=1,
                         bitorder="little")[:, :k]
    return np.where(bits == 1, -1.0, 1.0)


def gpu_branch(b, out_f, in_f, r):
    SU = signs_of(b.Up, out_f, r, b.layout)             # out x r
    SV = signs_of(b.Vp, r, in_f, b.layout).T            # in x r
    f = lambda t: t.float().cpu().numpy().astype(np.float64)
    return SU, SV, f(b.h), f(b.g), f(b.l)


@pytest.mark.parametrize("out_f,in_f,r", [(512, 384, 32), (384, 768, 48), (1024, 1024, 64)])
@pytest.mark.parametrize("layout", [lb.LB_LAYOUT_SLICES, lb.LB_LAYOUT_ROWS])
def test_dual_svid_matches_oracle(out_f, in_f, r, layout):
    W = gapped_weight(out_f, in_f, r, seed=out_f + in_f + r)
    brs = lb.dual_svid(torch.tensor(W, dtype=torch.float32, device="cuda"), r, 2, layout)
    torch.cuda.synchronize()
    W32 = W.astype(np.float32).astype(np.float64)
    ref = ds.dual_svid(W32, r, 2)
    got = [gpu_branch(b, out_f, in_f, r) for b in brs]
    # first branch: signs (each column pair aligned), scales and the branch itself
    SU, SV, h, g, l = got[0]
    rSU, rSV, rh, rg, rl = ref[0]
    flip = np.where((SU * rSU).sum(axis=0) < 0, -1.0, 1.0)
    assert np.mean(SU * flip != rSU) < 1e-3 and np.mean(SV * flip != rSV) < 1e-3
    for a, b_, what in ((h, rh, "h"), (g, rg, "g"), (l, rl, "l")):
        assert np.abs(a - b_).max() <= 1e-2 * np.abs(b_).max(), what
    W1, rW1 = ds.reconstruct(*got[0]), ds.reconstruct(*ref[0])
    assert np.linalg.norm(W1 - rW1) <= 1e-2 * np.linalg.norm(rW1)
    # both branches: the approximation error is the oracle's to within 5%, and the
    # residual branch lowers it
    e1 = np.linalg.norm(W32 - W1)
    e = np.linalg.norm(W32 - ds.approximation(got))
    re = np.linalg.norm(W32 - ds.approximation(ref))
    assert e < e1
    assert abs(e - re) <= 0.05 * re, (e, re)


def test_dual_svid_recovers_an_exact_branch():
    """W = c (h o s_u)(g o s_v)^T with fp16-exact h, g (mean 1) and c: one rank-1 branch
    represents it exactly, and the GPU's stored signs and scales reproduce W."""
    out_f, in_f = 96, 160
    h = np.where(np.arange(out_f) % 2 == 0, 0.5, 1.5)
    g = np.where(np.arange(in_f) % 4 == 0, 1.75, 0.75)
    rng = np.random.default_rng(3)
    su = np.where(rng.random(out_f) < 0.5, -1.0, 1.0)
    sv = np.where(rng.random(in_f) < 0.5, -1.0, 1.0)
    W = 0.375 * np.outer(h * su, g * sv)
    (b,) = lb.dual_svid(torch.tensor(W, dtype=torch.float32, device="cuda"), 1, 1)
    got = gpu_branch(b, out_f, in_f, 1)
    np.testing.assert_array_equal(ds.reconstruct(*got), W)


def test_dual_svid_rejects_bad_ranks():
    W = torch.zeros((64, 32), dtype=torch.float32, device="cuda")
    for r in (0, 33):
        with pytest.raises(lb.LbError):
            lb.dual_svid(W, r, 1)
