"""Pins of the oracle's bit-serial variant (CPU only).

"The XOR claim" ("Samsung LittleBit: A 13B LLM Under 1 GB, and What the Paper
Really Shows"): with both operands signs, a multiply is an XOR and a popcount.
The variant quantises each activation vector to odd-integer codes whose bit-planes
are signs (``oracle.forward_xor``).  Its pins: the code identity itself, the
quantiser's invariants, and agreement with the float oracle (pinned in
test_oracle_pins.py) inside the error bound the quantisation allows.
"""
import numpy as np
import pytest

import oracle
from oracle import Branch, forward, forward_xor, pack, xor_quantise

rng = np.random.default_rng(777)


@pytest.mark.parametrize("B", [1, 2, 3, 4, 5, 8])
def test_odd_codes_are_sums_of_signed_powers_of_two(B):
    """Every odd q in [-(2^B - 1), 2^B - 1] is sum_p 2^p sigma_p with
    sigma_p = 2 bit_p((q + 2^B - 1) / 2) - 1 in {-1, +1}, and no other integer is."""
    top = 2 ** B - 1
    seen = set()
    for v in range(2 ** B):
        sigma = [2 * ((v >> p) & 1) - 1 for p in range(B)]
        q = sum((1 << p) * s for p, s in enumerate(sigma))
        assert q == 2 * v - top and q % 2 == 1 and -top <= q <= top
        seen.add(q)
    assert seen == set(range(-top, top + 1, 2))


@pytest.mark.parametrize("B", [4, 8, 16])
def test_quantiser_invariants(B):
    top = 2 ** B - 1
    for scale in (1e-6, 0.3, 1.0, 7.5, 3e4):
        v = (scale * rng.standard_normal(777)).astype(np.float32)
        D, q = xor_quantise(v, B)
        A = float(np.abs(v).max())
        assert D == 2.0 ** round(np.log2(D))                       # a power of two
        assert A <= top * D and A > top * D / 2                     # the smallest such
        assert np.all(q % 2 == 1) and np.all(np.abs(q) <= top)      # odd codes in range
        assert np.all(np.abs(D * q - v.astype(np.float64)) <= D)    # error at most D


def test_quantiser_special_cases():
    D, q = xor_quantise(np.zeros(5, np.float32), 16)
    assert D == 2.0 ** -100 and np.all(q == 1)
    # exactly representable: odd integers whose largest is 2^B - 1 come back unchanged
    B = 8
    v = np.array([255, -255, 1, -1, 37, -129], np.float32)
    D, q = xor_quantise(v, B)
    assert D == 1.0 and np.array_equal(q, v.astype(np.int64))


def rand_branches(in_f, out_f, r, nb=2):
    out = []
    for _ in range(nb):
        U = rng.standard_normal((out_f, r)).astype(np.float32)
        V = rng.standard_normal((in_f, r)).astype(np.float32)
        sc = lambda n: np.abs(1 + 0.1 * rng.standard_normal(n)).astype(np.float16).astype(np.float64)
        out.append(Branch.from_latents(U, V, sc(out_f), sc(in_f), sc(r)))
    return out


def signs(words, n, k):
    bits = np.unpackbits(words.view(np.uint8), axis=1, bitorder="little")[:, :k]
    return np.where(bits[:n] == 1, -1.0, 1.0)


def xor_error_bound(x, brs, in_f, out_f, r, B):
    """Worst-case |y_xor - y_float| per output from the quantiser's error <= D per code,
    plus fp32 rounding of the scaled integer sums (2^-23 relative, twice)."""
    bound = np.zeros((x.shape[0], out_f))
    for m in range(x.shape[0]):
        for b in brs:
            u = (b.g.astype(np.float32) * x[m].astype(np.float32)).astype(np.float64)
            D1, _ = xor_quantise(u, B)
            SV = signs(b.Vp, r, in_f)
            t = SV @ u                                   # exact-arithmetic t_k
            tp = b.l * t
            D2, _ = xor_quantise(tp.astype(np.float32), B)
            dt = np.abs(b.l) * in_f * D1 + 2 ** -22 * (np.abs(tp) + np.abs(b.l) * in_f * D1)
            bound[m] += np.abs(b.h) * (r * D2 + dt.sum())
    return bound


@pytest.mark.parametrize("shape,B", [((64, 48, 32), 16), ((300, 129, 70), 16),
                                     ((512, 256, 32), 12), ((96, 64, 64), 10)])
def test_agrees_with_float_oracle_within_quantisation_bound(shape, B):
    in_f, out_f, r = shape
    brs = rand_branches(in_f, out_f, r)
    x = rng.standard_normal((2, in_f)).astype(np.float16).astype(np.float64)
    y = forward_xor(x, brs, in_f, out_f, r, bits=B)
    y_ref = forward(x, brs, in_f, out_f, r)
    bound = xor_error_bound(x, brs, in_f, out_f, r, B)
    assert np.all(np.abs(y - y_ref) <= bound), np.max(np.abs(y - y_ref) - bound)
    if B == 16:
        # the worst-case bound is far below the outputs, so a dropped term or a wrong
        # sign shows; and the actual error is inside the layer's 2e-3 output bound
        assert bound.max() < 0.02 * np.abs(y_ref).max()
        assert np.abs(y - y_ref).max() <= 2e-3 * np.abs(y_ref).max()


def test_exact_first_contraction_on_odd_integer_inputs():
    """g = 1 and x odd integers with max 2^B - 1: the first quantisation is exact, so the
    only error left is the second one (at most r * D2 per branch, times h)."""
    in_f, out_f, r, B = 65, 40, 16, 12
    brs = rand_branches(in_f, out_f, r, nb=1)
    brs[0].g = np.ones(in_f)
    x = (2 * rng.integers(-2 ** (B - 1), 2 ** (B - 1), size=(1, in_f)) + 1).astype(np.float64)
    x[0, 3] = 2 ** B - 1
    y = forward_xor(x, brs, in_f, out_f, r, bits=B)
    y_ref = forward(x, brs, in_f, out_f, r)
    SV = signs(brs[0].Vp, r, in_f)
    tp = (brs[0].l * (SV @ x[0])).astype(np.float32)
    D2, _ = xor_quantise(tp, B)
    np.testing.assert_array_less(np.abs(y - y_ref)[0], np.abs(brs[0].h) * (r * D2 + 1e-9) + 1e-12)
