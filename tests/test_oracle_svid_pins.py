"""Pins of the Dual-SVID initialisation oracle (CPU only).

"How it works", item 3 of "Samsung LittleBit: A 13B LLM Under 1 GB, and What the
Paper Really Shows": a truncated SVD of the weight mapped onto signs and scales, and
a residual branch fitted to what the first branch missed (``oracle/dual_svid.py``).
Pins: a weight that is exactly one branch is recovered exactly; the rank-1 magnitude
fit of an exact rank-1 matrix is exact; the approximation improves with the rank and
with the residual branch.
"""
import numpy as np
import pytest

from oracle import dual_svid as ds

rng = np.random.default_rng(4242)


def test_rank1_fit_of_an_outer_product_is_exact():
    a = rng.uniform(0.5, 2.0, 37)
    b = rng.uniform(0.1, 3.0, 11)
    x, y = ds.rank1_magnitudes(np.outer(a, b))
    np.testing.assert_allclose(np.outer(x, y), np.outer(a, b), rtol=1e-12)
    assert np.all(x >= 0) and np.all(y >= 0)
    x, y = ds.rank1_magnitudes(np.zeros((5, 3)))
    assert not np.any(x) and not np.any(y)


def test_one_exact_branch_is_recovered_and_the_residual_branch_is_zero():
    """W = c * (h o s_u)(g o s_v)^T with fp16-exact h, g (mean 1) and c: rank 1, so the
    first branch reproduces W exactly and the second fits a zero residual."""
    out_f, in_f = 24, 40
    h = np.where(np.arange(out_f) % 2 == 0, 0.5, 1.5)
    g = np.where(np.arange(in_f) % 4 == 0, 1.75, 0.75)
    su = np.where(rng.random(out_f) < 0.5, -1.0, 1.0)
    sv = np.where(rng.random(in_f) < 0.5, -1.0, 1.0)
    c = 0.375
    W = c * np.outer(h * su, g * sv)
    (b1, b2) = ds.dual_svid(W, 1, 2)
    np.testing.assert_array_equal(ds.reconstruct(*b1), W)
    np.testing.assert_array_equal(b1[2], h)
    np.testing.assert_array_equal(b1[3], g)
    np.testing.assert_array_equal(b1[4], [c])
    assert not np.any(b2[2]) and not np.any(b2[3]) and not np.any(b2[4])
    assert np.all(np.abs(b1[0]) == 1) and np.all(np.abs(b1[1]) == 1)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_error_falls_with_rank_and_with_the_residual_branch(seed):
    g = np.random.default_rng(seed)
    W = g.standard_normal((96, 80)) * 0.02
    errs = []
    for r in (2, 4, 8, 16, 32, 64):
        b1, b2 = ds.dual_svid(W, r, 2)
        e1 = np.linalg.norm(W - ds.reconstruct(*b1))
        e2 = np.linalg.norm(W - ds.approximation([b1, b2]))
        assert e2 < e1 < np.linalg.norm(W)
        assert b1[2].shape == (96,) and b1[3].shape == (80,) and b1[4].shape == (r,)
        assert np.all(b1[2] > 0) and np.all(b1[3] > 0) and np.all(b1[4] >= 0)
        errs.append(e2)
    assert all(b < a for a, b in zip(errs, errs[1:])), errs
