"""Pins of the oracle to things other than itself (CPU only).

The oracle (``oracle/``) evaluates the layer of "Samsung LittleBit: A 13B LLM
Under 1 GB, and What the Paper Really Shows", section "How it works", items 1-3.
Each test below checks it against something it does not share code with: a
hand-worked example, a closed form, an algebraic invariant, a dense numpy
reconstruction, or brute force over all index triples.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest

import oracle
from oracle import Branch, forward, pack
from oracle import stack as ostack

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng = np.random.default_rng(12345)


def signs_of(latent):
    """+1 / -1 straight from the latents (sign(v) = -1 iff v < 0)."""
    return np.where(np.asarray(latent, dtype=np.float64) < 0, -1.0, 1.0)


def rand_branch(in_f, out_f, r, zero_frac=0.0):
    U = rng.standard_normal((out_f, r)).astype(np.float32)
    V = rng.standard_normal((in_f, r)).astype(np.float32)
    if zero_frac:
        U[rng.random(U.shape) < zero_frac] = 0.0
        V[rng.random(V.shape) < zero_frac] = -0.0
    h = np.abs(1 + 0.1 * rng.standard_normal(out_f)).astype(np.float16).astype(np.float64)
    g = np.abs(1 + 0.1 * rng.standard_normal(in_f)).astype(np.float16).astype(np.float64)
    l = np.abs(1 + 0.1 * rng.standard_normal(r)).astype(np.float16).astype(np.float64)
    return U, V, h, g, l


def dense_w(U, V, h, g, l):
    """W' = diag(h) sign(U) diag(l) sign(V)^T diag(g), built explicitly."""
    return (h[:, None] * signs_of(U)) @ (l[:, None] * signs_of(V).T * g[None, :])


# ---------------------------------------------------------------- packing
def test_pack_matches_format_definition_with_special_values():
    lat = rng.standard_normal((37, 70)).astype(np.float32)
    specials = np.array([0.0, -0.0, np.inf, -np.inf, np.nan, -np.nan, 1e-45, -1e-45,
                         np.finfo(np.float32).tiny, -np.finfo(np.float32).tiny], np.float32)
    lat.flat[: specials.size * 7: 7] = specials
    for axis in (0, 1):
        words = pack(lat, axis=axis)
        neg = (lat < 0) if axis == 1 else (lat < 0).T           # rows to pack along
        k = neg.shape[1]
        padded = np.zeros((neg.shape[0], ((k + 31) // 32) * 32), dtype=np.uint8)
        padded[:, :k] = neg
        expect = np.packbits(padded, axis=1, bitorder="little").view("<u4")
        np.testing.assert_array_equal(words, expect)
        assert int(np.unpackbits(words.view(np.uint8)).sum()) == int(neg.sum())


def test_pack_padding_words_are_zero():
    lat = -np.ones((5, 40), np.float32)
    w = pack(lat, axis=1, ld_words=4)
    assert w.shape == (5, 4)
    assert np.all(w[:, 0] == 0xFFFFFFFF) and np.all(w[:, 1] == 0xFF) and np.all(w[:, 2:] == 0)


# ---------------------------------------------------------------- hand-worked example
def test_hand_worked_example():
    ex = json.load(open(os.path.join(GOLDEN, "hand_example.json")))
    brs = []
    for b in ex["branches"]:
        V = np.array(b["V_latent"], np.float32)
        U = np.array(b["U_latent"], np.float32)
        Vp, Up = pack(V, axis=0), pack(U, axis=1)
        assert Vp[:, 0].tolist() == b["Vp_words"]
        assert Up[:, 0].tolist() == b["Up_words"]
        br = Branch(Vp, Up, b["h"], b["g"], b["l"])
        z = forward(np.array(ex["x"]), [br], ex["in"], ex["out"], ex["r"])[0]
        assert z.tolist() == b["z"]
        brs.append(br)
    y = forward(np.array(ex["x"]), brs, ex["in"], ex["out"], ex["r"])[0]
    assert y.tolist() == ex["y"]


# ---------------------------------------------------------------- closed forms
def test_rank_one_unit_scales_closed_form():
    in_f, out_f = 97, 45
    u = rng.standard_normal((out_f, 1)).astype(np.float32)
    v = rng.standard_normal((in_f, 1)).astype(np.float32)
    x = rng.standard_normal(in_f)
    br = Branch.from_latents(u, v, np.ones(out_f), np.ones(in_f), np.ones(1))
    y = forward(x, [br], in_f, out_f, 1)[0]
    s, vv = signs_of(u[:, 0]), signs_of(v[:, 0])
    np.testing.assert_allclose(y, s * float(np.dot(vv, x)), rtol=1e-13, atol=1e-12)


def sylvester(n):
    H = np.array([[1.0]])
    while H.shape[0] < n:
        H = np.block([[H, H], [H, -H]])
    return H


@pytest.mark.parametrize("n", [32, 64, 128])
def test_hadamard_factors_give_scaled_identity(n):
    H = sylvester(n).astype(np.float32)
    h = np.abs(1 + 0.1 * rng.standard_normal(n))
    g = np.abs(1 + 0.1 * rng.standard_normal(n))
    x = rng.standard_normal(n)
    br = Branch.from_latents(H, H, h, g, np.ones(n))
    y = forward(x, [br], n, n, n)[0]
    # sign(H) sign(H)^T = H H^T = n I, so W' = n diag(h) diag(g)
    np.testing.assert_allclose(y, n * h * g * x, rtol=1e-13, atol=1e-12)


# ---------------------------------------------------------------- dense reconstruction
@pytest.mark.parametrize("shape", [(64, 48, 8), (130, 70, 33), (256, 512, 64)])
def test_matches_dense_reconstruction(shape):
    in_f, out_f, r = shape
    parts = [rand_branch(in_f, out_f, r, zero_frac=0.02) for _ in range(2)]
    x = rng.standard_normal((3, in_f))
    W = sum(dense_w(*p) for p in parts)
    brs = [Branch.from_latents(U, V, h, g, l) for U, V, h, g, l in parts]
    y = forward(x, brs, in_f, out_f, r)
    np.testing.assert_allclose(y, x @ W.T, rtol=1e-11, atol=1e-9 * np.abs(x @ W.T).max())


def test_selected_rows_equal_full_rows():
    in_f, out_f, r = 300, 200, 40
    brs = [Branch.from_latents(*rand_branch(in_f, out_f, r)) for _ in range(2)]
    x = rng.standard_normal((2, in_f))
    full = forward(x, brs, in_f, out_f, r)
    rows = [0, 7, 199, 100, 7]
    np.testing.assert_array_equal(forward(x, brs, in_f, out_f, r, rows=rows), full[:, rows])


# ---------------------------------------------------------------- brute force
@pytest.mark.parametrize("shape", [(1, 1, 1), (3, 5, 2), (8, 7, 8), (5, 8, 3)])
def test_brute_force_tiny(shape):
    in_f, out_f, r = shape
    parts = [rand_branch(in_f, out_f, r, zero_frac=0.1) for _ in range(2)]
    x = rng.standard_normal(in_f)
    y_bf = [0.0] * out_f
    for U, V, h, g, l in parts:
        for i, j, k in itertools.product(range(out_f), range(in_f), range(r)):
            su = -1.0 if U[i, k] < 0 else 1.0
            sv = -1.0 if V[j, k] < 0 else 1.0
            y_bf[i] += h[i] * su * l[k] * sv * g[j] * x[j]
    brs = [Branch.from_latents(*p) for p in parts]
    y = forward(x, brs, in_f, out_f, r)[0]
    np.testing.assert_allclose(y, y_bf, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- invariants
def test_linear_in_residual_scales_and_input():
    in_f, out_f, r = 96, 80, 24
    p0, p1 = rand_branch(in_f, out_f, r), rand_branch(in_f, out_f, r)
    x = rng.standard_normal(in_f)
    b0 = Branch.from_latents(*p0)

    def y_with(h1=None, g1=None, l1=None, xx=x):
        U, V, h, g, l = p1
        b1 = Branch.from_latents(U, V, h if h1 is None else h1, g if g1 is None else g1,
                                 l if l1 is None else l1)
        return forward(xx, [b0, b1], in_f, out_f, r)[0]

    base = y_with(h1=np.zeros(out_f))
    np.testing.assert_allclose(base, forward(x, [b0], in_f, out_f, r)[0], rtol=1e-13)
    for a in (0.5, 3.0, -2.0):
        for kw, vec in (("h1", p1[2]), ("g1", p1[3]), ("l1", p1[4])):
            zero = y_with(**{kw: np.zeros_like(vec)})
            one = y_with(**{kw: vec})
            scaled = y_with(**{kw: a * vec})
            np.testing.assert_allclose(scaled - zero, a * (one - zero), rtol=1e-10, atol=1e-9)
    x2 = rng.standard_normal(in_f)
    np.testing.assert_allclose(y_with(xx=2 * x - 3 * x2), 2 * y_with(xx=x) - 3 * y_with(xx=x2),
                               rtol=1e-10, atol=1e-9)


def test_negating_both_latents_complements_bits_and_keeps_output():
    in_f, out_f, r = 100, 60, 20
    U, V, h, g, l = rand_branch(in_f, out_f, r)
    x = rng.standard_normal(in_f)
    b = Branch.from_latents(U, V, h, g, l)
    bn = Branch.from_latents(-U, -V, h, g, l)
    mask_v = np.uint32((1 << (in_f % 32)) - 1)
    full = np.uint32(0xFFFFFFFF)
    np.testing.assert_array_equal(bn.Vp[:, :-1], b.Vp[:, :-1] ^ full)
    np.testing.assert_array_equal(bn.Vp[:, -1], b.Vp[:, -1] ^ mask_v)
    np.testing.assert_array_equal(forward(x, [bn], in_f, out_f, r), forward(x, [b], in_f, out_f, r))


# ---------------------------------------------------------------- decoder glue
def dense_linear(rs_rng, in_f, out_f, r):
    parts = [rand_branch(in_f, out_f, r) for _ in range(2)]
    W = sum(dense_w(*p) for p in parts)
    lin = ostack.Linear([Branch.from_latents(*p) for p in parts], in_f, out_f, r)
    return lin, W


def test_glue_closed_forms():
    v = np.array([3.0, 4.0])
    np.testing.assert_allclose(ostack.rmsnorm(v), v / math.sqrt(12.5 + 1e-5))
    np.testing.assert_allclose(ostack.silu(np.array([0.0, 1.0, -1.0])),
                               [0.0, 1 / (1 + math.exp(-1)), -1 / (1 + math.exp(1))])
    vv = np.arange(2 * 3, dtype=float)      # 2 kv heads of dim 3, 4 query heads
    np.testing.assert_array_equal(ostack.gqa_broadcast(vv, 4, 2, 3),
                                  [0, 1, 2, 0, 1, 2, 3, 4, 5, 3, 4, 5])


def test_decoder_layer_matches_dense_composition():
    hidden, inter, nh, nkv, hd = 64, 96, 4, 2, 16
    kv = nkv * hd
    shapes = dict(q=(hidden, hidden), k=(hidden, kv), v=(hidden, kv), o=(hidden, hidden),
                  gate=(hidden, inter), up=(hidden, inter), down=(inter, hidden))
    layers, dense = [], []
    for _ in range(2):
        L, D = {}, {}
        for name, (i, o) in shapes.items():
            L[name], D[name] = dense_linear(rng, i, o, 16)
        layers.append(L)
        dense.append(D)
    x = rng.standard_normal(hidden)
    got = ostack.decoder_stack(x, layers, nh, nkv, hd)
    h = x.copy()
    for D in dense:
        a = h / np.sqrt(np.mean(h ** 2) + 1e-5)
        v = D["v"] @ a
        attn = np.concatenate([v[(q // (nh // nkv)) * hd:(q // (nh // nkv) + 1) * hd]
                               for q in range(nh)])
        h = h + D["o"] @ attn
        a = h / np.sqrt(np.mean(h ** 2) + 1e-5)
        gt, up = D["gate"] @ a, D["up"] @ a
        h = h + D["down"] @ (gt / (1 + np.exp(-gt)) * up)
    np.testing.assert_allclose(got, h, rtol=1e-10, atol=1e-10 * np.abs(h).max())


def test_mlp_block_matches_dense_composition():
    hidden, inter = 48, 80
    gate, Wg = dense_linear(rng, hidden, inter, 16)
    up, Wu = dense_linear(rng, hidden, inter, 16)
    down, Wd = dense_linear(rng, inter, hidden, 16)
    x = rng.standard_normal(hidden)
    gt, u = Wg @ x, Wu @ x
    ref = Wd @ (gt / (1 + np.exp(-gt)) * u)
    np.testing.assert_allclose(ostack.mlp_block(x, gate, up, down), ref, rtol=1e-10,
                               atol=1e-10 * np.abs(ref).max())


def test_threads_reported():
    assert oracle.threads() >= 1
