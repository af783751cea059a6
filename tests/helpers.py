"""Shared helpers for the GPU parity tests: the same seeded inputs on both sides.

Inputs come from ``binary_rank_linear_lb_b200.synth`` only.  The CUDA side packs
them with ``lb_pack_signs``; the oracle side packs host copies with its own packer.
"""
import numpy as np
import torch

import oracle
from binary_rank_linear_lb_b200 import synth

TOL = 2e-3   # max|y - y_ref| <= TOL * max|y_ref|


def oracle_branch(in_f, out_f, r, base, layer, proj, b, device="cuda"):
    U, V, h, g, l = synth.branch_tensors(in_f, out_f, r, base, layer, proj, b, device)
    host = lambda t: t.float().cpu().numpy()
    return oracle.Branch.from_latents(host(U), host(V), host(h).astype(np.float64),
                                      host(g).astype(np.float64), host(l).astype(np.float64))


def oracle_branch_bits(in_f, out_f, r, base, layer, proj, b, device="cuda"):
    """A branch whose packed signs are drawn directly as words (model's signs="bits")."""
    s = lambda k: synth.tensor_seed(base, layer, proj, b, k)
    words = lambda n, k, kind: synth.sign_words(n, k, s(kind), device).cpu().numpy().view(np.uint32)
    sc = lambda n, kind: synth.scale(n, s(kind), device).float().cpu().numpy().astype(np.float64)
    return oracle.Branch(words(r, in_f, synth.KIND_V), words(out_f, r, synth.KIND_U),
                         sc(out_f, synth.KIND_H), sc(in_f, synth.KIND_G), sc(r, synth.KIND_L))


def oracle_linear(in_f, out_f, r, base, layer, proj, nb=2, device="cuda"):
    return [oracle_branch(in_f, out_f, r, base, layer, proj, b, device) for b in range(nb)]


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def rel_err(y, y_ref) -> float:
    y = np.asarray(y, dtype=np.float64)
    y_ref = np.asarray(y_ref, dtype=np.float64)
    scale = np.abs(y_ref).max()
    return float(np.abs(y - y_ref).max() / scale) if scale > 0 else float(np.abs(y).max())


def assert_close(y, y_ref, tol=TOL, what=""):
    e = rel_err(y, y_ref)
    assert e <= tol, f"{what}: max|y-y_ref| / max|y_ref| = {e:.3e} > {tol}"
    return e
