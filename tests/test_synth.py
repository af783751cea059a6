"""The seeded input generators shared by both sides of the parity tests (CPU)."""
import numpy as np
import torch

from binary_rank_linear_lb_b200 import LB_LAYOUT_ROWS, LB_LAYOUT_SLICES, synth, unslice_words
from binary_rank_linear_lb_b200.model import build_branch


def test_sign_words_shape_tail_and_balance():
    w = synth.sign_words(300, 1001, seed=5)
    assert w.shape == (300, 32) and w.dtype == torch.int32
    a = w.numpy().view(np.uint32)
    assert not (a[:, -1] >> (1001 % 32)).any()            # bits past k are zero
    bits = np.unpackbits(a[:, :-1].view(np.uint8))
    assert abs(bits.mean() - 0.5) < 0.01                     # fair coins
    assert torch.equal(w, synth.sign_words(300, 1001, seed=5))
    assert not torch.equal(w, synth.sign_words(300, 1001, seed=6))


def test_bits_mode_branches_hold_the_shared_words():
    # both layouts of a signs="bits" branch carry exactly synth.sign_words of its seeds
    in_f, out_f, r = 700, 530, 96
    s = lambda k: synth.tensor_seed(2, 1, 4, 1, k)
    v = synth.sign_words(r, in_f, s(synth.KIND_V))
    u = synth.sign_words(out_f, r, s(synth.KIND_U))
    b = build_branch(in_f, out_f, r, 2, 1, 4, 1, device="cpu", signs="bits",
                     layout=LB_LAYOUT_SLICES)
    assert torch.equal(unslice_words(b.Vp, r, in_f), v)
    assert torch.equal(unslice_words(b.Up, out_f, r), u)
    b = build_branch(in_f, out_f, r, 2, 1, 4, 1, device="cpu", signs="bits",
                     layout=LB_LAYOUT_ROWS)
    assert torch.equal(b.Vp[:, :v.shape[1]], v) and not b.Vp[:, v.shape[1]:].any()
    assert torch.equal(b.Up[:, :u.shape[1]], u) and not b.Up[:, u.shape[1]:].any()
