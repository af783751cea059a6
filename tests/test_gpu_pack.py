"""lb_pack_signs / lb_pack_signs_sliced against the oracle's packer: bit-exact (GPU)."""
import numpy as np
import pytest
import torch

import oracle
import binary_rank_linear_lb_b200 as lb
from binary_rank_linear_lb_b200 import synth

pytestmark = pytest.mark.gpu


def gpu_pack(lat_host: np.ndarray, axis: int, ld_words=None) -> np.ndarray:
    t = torch.from_numpy(lat_host).cuda()
    w = lb.pack_signs(t, axis, ld_words)
    torch.cuda.synchronize()
    return w.cpu().numpy().view(np.uint32)


@pytest.mark.parametrize("shape", [(1, 1), (31, 33), (64, 32), (100, 257), (512, 32),
                                   (1000, 70), (33, 2000)])
@pytest.mark.parametrize("axis", [0, 1])
def test_pack_bit_exact_random_and_special(shape, axis):
    rng = np.random.default_rng(shape[0] * 7 + shape[1] + axis)
    lat = rng.standard_normal(shape).astype(np.float32)
    specials = np.array([0.0, -0.0, np.inf, -np.inf, np.nan, 1e-45, -1e-45, -1e-38],
                        np.float32)
    idx = rng.integers(0, lat.size, size=min(lat.size, 64))
    lat.flat[idx] = specials[np.arange(idx.size) % specials.size]
    np.testing.assert_array_equal(gpu_pack(lat, axis), oracle.pack(lat, axis))


@pytest.mark.parametrize("axis", [0, 1])
def test_pack_with_padding_words(axis):
    rng = np.random.default_rng(5)
    lat = rng.standard_normal((70, 45)).astype(np.float32)
    k = 45 if axis == 1 else 70
    ldw = (k + 31) // 32 + 3
    np.testing.assert_array_equal(gpu_pack(lat, axis, ldw), oracle.pack(lat, axis, ldw))


def test_pack_strided_latent():
    rng = np.random.default_rng(9)
    big = torch.from_numpy(rng.standard_normal((40, 100)).astype(np.float32)).cuda()
    view = big[:, 10:77]                     # row stride 100, 67 columns
    w = lb.pack_signs(view, 1)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(w.cpu().numpy().view(np.uint32),
                                  oracle.pack(view.cpu().numpy(), 1))


@pytest.mark.parametrize("which", ["V", "U"])
def test_pack_full_size_70b_gate(which):
    """The largest factor of the 70B stack (gate, 1.0 bits per weight): 8192 x 3136 / 28672 x 3136."""
    in_f, out_f, r = 8192, 28672, 3136
    seed = synth.tensor_seed(0, 0, 4, 0, synth.KIND_V if which == "V" else synth.KIND_U)
    rows = in_f if which == "V" else out_f
    lat = synth.latent(rows, r, seed, "cuda")
    axis = 0 if which == "V" else 1
    w = lb.pack_signs(lat, axis)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(w.cpu().numpy().view(np.uint32), oracle.pack(lat.cpu().numpy(), axis))


def spec_slices(words: np.ndarray, k: int) -> np.ndarray:
    """The sliced layout as include/lb.h defines it, from row-major words [n][ceil(k/32)]."""
    n, nw = words.shape[0], (k + 31) // 32
    ns = (nw + 15) // 16
    out = []
    for s in range(ns):
        width = min(16, nw - 16 * s)
        pitch = 16 if s < ns - 1 else (width + 3) // 4 * 4
        block = np.zeros((n, pitch), np.uint32)
        block[:, :width] = words[:, 16 * s:16 * s + width]
        out.append(block.reshape(-1))
    return np.concatenate(out)


@pytest.mark.parametrize("shape", [(1, 1), (31, 33), (64, 512), (100, 513), (700, 1100),
                                   (2000, 33), (1536, 96)])
@pytest.mark.parametrize("axis", [0, 1])
def test_pack_sliced_bit_exact(shape, axis):
    rng = np.random.default_rng(shape[0] * 3 + shape[1] + 11 * axis)
    lat = rng.standard_normal(shape).astype(np.float32)
    lat.flat[rng.integers(0, lat.size, size=min(lat.size, 16))] = -0.0
    t = torch.from_numpy(lat).cuda()
    got = lb.pack_signs(t, axis, layout=lb.LB_LAYOUT_SLICES)
    torch.cuda.synchronize()
    k = shape[1] if axis == 1 else shape[0]
    n = shape[0] if axis == 1 else shape[1]
    ref = oracle.pack(lat, axis)
    assert got.numel() == lb.packed_words(n, k, lb.LB_LAYOUT_SLICES)
    np.testing.assert_array_equal(got.cpu().numpy().view(np.uint32), spec_slices(ref, k))
    # and the binding's converters agree with the layout
    back = lb.unslice_words(got, n, k).cpu().numpy().view(np.uint32)
    np.testing.assert_array_equal(back, ref)
    np.testing.assert_array_equal(
        lb.slice_words(torch.from_numpy(ref.view(np.int32)), k).numpy().view(np.uint32),
        spec_slices(ref, k))
