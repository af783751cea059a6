"""Seeded synthetic inputs: latent factors, FP16 scales and activations.

This module only draws random numbers; it holds none of the layer's arithmetic
and is shared by the CUDA path (tests, bench) and the oracle side of the tests.
Every tensor has its own seed derived from (base seed, layer, projection,
branch, kind), so any single tensor can be regenerated on its own.

Distributions: latents N(0, 1) fp32; scales |N(1, 0.1)| rounded to fp16;
activations N(0, 1) in the requested dtype; sign words uniform random bits
(the signs of i.i.d. N(0, 1) latents are i.i.d. fair coins, so packed words
drawn directly have the distribution of packed latents).
"""
from __future__ import annotations

import torch

KIND_U, KIND_V, KIND_H, KIND_G, KIND_L, KIND_X = range(6)


def tensor_seed(base: int, layer: int, proj: int, branch: int, kind: int) -> int:
    return base * 1_000_003 + (layer * 7 + proj) * 16 + branch * 8 + kind


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def latent(rows: int, cols: int, seed: int, device="cpu") -> torch.Tensor:
    """N(0, 1) fp32 latent factor, rows x cols."""
    return torch.randn((rows, cols), generator=_gen(seed, device), device=device,
                       dtype=torch.float32)


def scale(n: int, seed: int, device="cpu") -> torch.Tensor:
    """|N(1, 0.1)| rounded to fp16."""
    z = torch.randn((n,), generator=_gen(seed, device), device=device, dtype=torch.float32)
    return (1.0 + 0.1 * z).abs().to(torch.float16)


def activation(shape, seed: int, dtype=torch.bfloat16, device="cpu") -> torch.Tensor:
    """N(0, 1) activations in `dtype`."""
    if isinstance(shape, int):
        shape = (shape,)
    z = torch.randn(tuple(shape), generator=_gen(seed, device), device=device, dtype=torch.float32)
    return z.to(dtype)


def sign_words(n_rows: int, k: int, seed: int, device="cpu") -> torch.Tensor:
    """Uniform random packed signs: int32 words [n_rows][ceil(k/32)], bit j of
    word w of a row standing for element 32*w + j; the bits past k are zero."""
    nw = (k + 31) // 32
    w = torch.randint(-2 ** 31, 2 ** 31, (n_rows, nw), generator=_gen(seed, device),
                      device=device, dtype=torch.int64).to(torch.int32)
    if k % 32:
        w[:, nw - 1] &= (1 << (k % 32)) - 1
    return w


def branch_tensors(in_f: int, out_f: int, r: int, base: int, layer: int, proj: int, branch: int,
                   device="cpu"):
    """(U latent out x r, V latent in x r, h out, g in, l r) of one branch."""
    s = lambda k: tensor_seed(base, layer, proj, branch, k)
    return (latent(out_f, r, s(KIND_U), device), latent(in_f, r, s(KIND_V), device),
            scale(out_f, s(KIND_H), device), scale(in_f, s(KIND_G), device),
            scale(r, s(KIND_L), device))
