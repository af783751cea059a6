"""Device-resident factorised linears and decoder stacks built from seeded inputs.

Each branch is generated from its own seeds (``synth``) and binarised on the GPU
with ``lb_pack_signs_sliced`` (the default sliced layout, whose 512-sign slices
are contiguous blocks of rows) or ``lb_pack_signs`` (row-major, with a 64-byte
pitch: ``ld_words`` a multiple of 16, zero padding); the fp32 latents are
dropped right after packing.

``signs="bits"`` instead draws the packed words directly from a uniform bit
source (``synth.sign_words``).  The signs of i.i.d. N(0, 1) latents are i.i.d.
fair coins, so the packed matrices have the same distribution; this shortens
the set-up of the largest stacks (whose latents would be hundreds of GB of
fp32).  The oracle side of a test draws the same words from the same seeds.
"""
from __future__ import annotations

from typing import List, Optional

import torch

from . import LB_LAYOUT_ROWS, LB_LAYOUT_SLICES, Branch, Stack, pack_signs, slice_words, synth
from .configs import Model, proj_shape


def padded_words(k: int, pad: bool = True) -> int:
    """Words per packed row of k signs: ceil(k/32), rounded up to a multiple of 16 if pad.

    A 64-byte pitch puts every 512-column slice of every row in one aligned
    64-byte piece of memory, the DRAM access unit; the kernels never read the
    padding, so the bytes streamed stay the packed signs themselves.
    """
    w = (k + 31) // 32
    return (w + 15) // 16 * 16 if pad else w


def build_branch(in_f: int, out_f: int, r: int, base: int, layer: int, proj: int, branch: int,
                 device="cuda", signs: str = "latent", pad: bool = True,
                 layout: int = LB_LAYOUT_SLICES) -> Branch:
    """One branch from its seeds.  layout: LB_LAYOUT_SLICES (the batch-1 fast
    layout, the default) or LB_LAYOUT_ROWS (row-major, pitch padded_words(k, pad))."""
    s = lambda k: synth.tensor_seed(base, layer, proj, branch, k)
    h = synth.scale(out_f, s(synth.KIND_H), device)
    g = synth.scale(in_f, s(synth.KIND_G), device)
    l = synth.scale(r, s(synth.KIND_L), device)
    if signs == "latent":
        V = synth.latent(in_f, r, s(synth.KIND_V), device)
        Vp = pack_signs(V, axis=0, ld_words=padded_words(in_f, pad), layout=layout)
        del V
        U = synth.latent(out_f, r, s(synth.KIND_U), device)
        Up = pack_signs(U, axis=1, ld_words=padded_words(r, pad), layout=layout)
        del U
    elif signs == "bits":
        def words(n_rows, k, seed):
            w = synth.sign_words(n_rows, k, seed, device)
            if layout != LB_LAYOUT_ROWS:
                return slice_words(w, k)
            ldw = padded_words(k, pad)
            out = torch.zeros((n_rows, ldw), dtype=torch.int32, device=device)
            out[:, :w.shape[1]] = w
            return out
        Vp = words(r, in_f, s(synth.KIND_V))
        Up = words(out_f, r, s(synth.KIND_U))
    else:
        raise ValueError(signs)
    return Branch(Vp, Up, h, g, l, layout)


def build_linear(in_f: int, out_f: int, r: int, base: int = 0, layer: int = 0, proj: int = 0,
                 n_branches: int = 2, device="cuda", signs: str = "latent",
                 pad: bool = True, layout: int = LB_LAYOUT_SLICES) -> List[Branch]:
    return [build_branch(in_f, out_f, r, base, layer, proj, b, device, signs, pad, layout)
            for b in range(n_branches)]


def build_stack(model: Model, bpw: float, base: int = 0, n_layers: Optional[int] = None,
                n_branches: int = 2, device="cuda", signs: str = "latent",
                ranks: Optional[List[int]] = None, layout: int = LB_LAYOUT_SLICES) -> Stack:
    nl = n_layers or model.n_layers
    rk = ranks or model.ranks(bpw)
    linears, all_ranks = [], []
    for li in range(nl):
        L = []
        for p in range(7):
            i, o = proj_shape(p, model.hidden, model.inter, model.kv_dim)
            L.append(build_linear(i, o, rk[p], base, li, p, n_branches, device, signs,
                                  layout=layout))
        linears.append(L)
        all_ranks.append(list(rk))
    return Stack(linears, all_ranks, model.hidden, model.inter, model.n_heads, model.n_kv_heads,
                 model.head_dim, device=device)


def build_mlp_block(model: Model, bpw: float, base: int = 0, n_branches: int = 2,
                    device="cuda", signs: str = "latent",
                    ranks: Optional[List[int]] = None, layout: int = LB_LAYOUT_SLICES) -> Stack:
    rk = ranks or model.ranks(bpw)
    L: list = [None] * 7
    for p in (4, 5, 6):
        i, o = proj_shape(p, model.hidden, model.inter, model.kv_dim)
        L[p] = build_linear(i, o, rk[p], base, 0, p, n_branches, device, signs, layout=layout)
    return Stack([L], [list(rk)], model.hidden, model.inter, mlp_only=True, device=device)
