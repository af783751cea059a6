"""Dual-SVID initialisation of the factorised layer, in numpy fp64.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

"Samsung LittleBit: A 13B LLM Under 1 GB, and What the Paper Really Shows",
section "How it works", item 3: the layer is initialised from a truncated SVD
of the real weight, whose signs and magnitudes are mapped onto the binary
factors and the scales; a second, residual branch is then fitted to what the
first one missed.  The page gives only this outline; the steps below are the
plainest reading of it (each one a line of the definition):

  for each branch b, on the residual R (R = W for the first branch):
    R ~ U S V^T                        rank-r truncated SVD
    U' = U S^(1/2),  V' = V S^(1/2)    the singular values split evenly
    sign(U'), sign(V')                 the binary factors (sign(0) = +1)
    |U'| ~ h l_u^T,  |V'| ~ g l_v^T    best rank-1 fits of the magnitudes
                                       (their leading singular pairs, taken >= 0)
    h, g scaled to mean 1, l = l_u * l_v; h, g, l rounded to fp16
    W_b = diag(h) sign(U') diag(l) sign(V')^T diag(g)
    R  <- R - W_b
A library SVD (``numpy.linalg.svd``) is a step of the definition.  A zero
magnitude matrix (a residual of zero) fits to zero scales.
"""
from __future__ import annotations

from typing import List, Tuple

import numpy as np


def signs(a: np.ndarray) -> np.ndarray:
    """+1 / -1 with sign(0) = +1 (the packing convention: bit set iff v < 0)."""
    return np.where(a < 0, -1.0, 1.0)


def rank1_magnitudes(A: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """Nonnegative (a, b) with a b^T the best rank-1 approximation of A >= 0."""
    if not np.any(A):
        return np.zeros(A.shape[0]), np.zeros(A.shape[1])
    u, s, vt = np.linalg.svd(A, full_matrices=False)
    a, b = np.abs(u[:, 0]) * np.sqrt(s[0]), np.abs(vt[0]) * np.sqrt(s[0])
    return a, b


def fp16(v: np.ndarray) -> np.ndarray:
    return np.asarray(v, dtype=np.float64).astype(np.float16).astype(np.float64)


def branch_from(R: np.ndarray, r: int):
    """One branch fitted to R: (sign(U') out x r, sign(V') in x r, h, g, l) in fp64
    (h, g, l hold fp16 values)."""
    U, s, Vt = np.linalg.svd(R, full_matrices=False)
    Up = U[:, :r] * np.sqrt(s[:r])
    Vp = Vt[:r].T * np.sqrt(s[:r])
    h, lu = rank1_magnitudes(np.abs(Up))
    g, lv = rank1_magnitudes(np.abs(Vp))
    ch, cg = h.mean(), g.mean()
    if ch > 0:
        h, lu = h / ch, lu * ch
    if cg > 0:
        g, lv = g / cg, lv * cg
    return signs(Up), signs(Vp), fp16(h), fp16(g), fp16(lu * lv)


def reconstruct(SU, SV, h, g, l) -> np.ndarray:
    """diag(h) SU diag(l) SV^T diag(g)."""
    return (h[:, None] * SU * l[None, :]) @ (SV * g[:, None]).T


def dual_svid(W: np.ndarray, r: int, n_branches: int = 2) -> List[tuple]:
    """Branches of the layer initialised from W (out x in); each (SU, SV, h, g, l)."""
    R = np.asarray(W, dtype=np.float64).copy()
    out = []
    for _ in range(n_branches):
        br = branch_from(R, r)
        R = R - reconstruct(*br)
        out.append(br)
    return out


def approximation(branches) -> np.ndarray:
    """The weight the initialised layer represents: the sum of its branches."""
    return sum(reconstruct(*b) for b in branches)
