"""Oracle for the LittleBit factorised binary linear layer.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  It shares no code with
the CUDA library in ``binary_rank_linear_lb_b200`` and never imports it.

The arithmetic lives in ``lb_oracle.c`` (plain C, fp64) and in ``stack.py``
(numpy fp64 glue for decoder stacks).  This module only builds and loads the C
library and converts arrays.  Parity of every function here is pinned by the
``-m "not gpu"`` tests in ``tests/test_oracle_pins.py``.

``dual_svid.py`` holds the Dual-SVID initialisation (numpy fp64, library SVD),
pinned by ``tests/test_oracle_svid_pins.py``.

Sources (web pages on LittleBit; cited by page title and section):
  * "Samsung LittleBit: A 13B LLM Under 1 GB, and What the Paper Really Shows",
    section "How it works": 1 (binary factors U, V), 2 (FP16 scales along rows,
    columns and the latent dimension), 3 (residual branch).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "lb_oracle.c")
_LIB_PATH = os.path.join(_HERE, "_lb_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle with gcc (OpenMP, -O2, no fast-math, no fused multiply-add)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-ffp-contract=off",
             "-Wall", "-Wextra",
             "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        i64, vp = ctypes.c_int64, ctypes.c_void_p
        lib.lbo_pack.argtypes = [vp, i64, i64, i64, ctypes.c_int, vp, i64]
        lib.lbo_pack.restype = ctypes.c_int
        lib.lbo_forward.argtypes = [vp, i64, i64, i64, i64, ctypes.c_int,
                                    vp, i64, vp, i64, vp, vp, vp, vp, i64, vp]
        lib.lbo_forward.restype = ctypes.c_int
        lib.lbo_forward_xor.argtypes = [vp, i64, i64, i64, i64, ctypes.c_int, ctypes.c_int,
                                        vp, i64, vp, i64, vp, vp, vp, vp]
        lib.lbo_forward_xor.restype = ctypes.c_int
        lib.lbo_xor_quantise.argtypes = [vp, i64, ctypes.c_int, vp]
        lib.lbo_xor_quantise.restype = ctypes.c_float
        lib.lbo_threads.restype = ctypes.c_int
        lib.lbo_set_threads.argtypes = [ctypes.c_int]
        _lib = lib
    return _lib


def threads() -> int:
    """Number of OpenMP threads the oracle runs with."""
    return int(_load().lbo_threads())


def set_threads(n: int) -> None:
    _load().lbo_set_threads(int(n))


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def pack(latent: np.ndarray, axis: int, ld_words: Optional[int] = None) -> np.ndarray:
    """Pack the signs of an fp32 latent matrix: bit = (latent < 0), LSB first.

    axis=1 packs every row along its columns (U: out x r -> [out][ceil(r/32)]);
    axis=0 packs every column along the rows (V: in x r -> [r][ceil(in/32)]).
    """
    lat = np.ascontiguousarray(latent, dtype=np.float32)
    if lat.ndim != 2:
        raise ValueError("latent must be 2-D")
    rows, cols = lat.shape
    k = cols if axis == 1 else rows
    n_out = rows if axis == 1 else cols
    ldw = (k + 31) // 32 if ld_words is None else int(ld_words)
    out = np.empty((n_out, ldw), dtype=np.uint32)
    rc = _load().lbo_pack(_ptr(lat), rows, cols, cols, int(axis), _ptr(out), ldw)
    if rc != 0:
        raise ValueError("lbo_pack rejected its arguments")
    return out


class Branch:
    """One branch of the layer: packed signs and fp64 copies of its scales."""

    def __init__(self, Vp, Up, h, g, l):
        self.Vp = np.ascontiguousarray(Vp, dtype=np.uint32)   # [r][ldv]
        self.Up = np.ascontiguousarray(Up, dtype=np.uint32)   # [out][ldu]
        self.h = np.ascontiguousarray(h, dtype=np.float64)    # out
        self.g = np.ascontiguousarray(g, dtype=np.float64)    # in
        self.l = np.ascontiguousarray(l, dtype=np.float64)    # r

    @classmethod
    def from_latents(cls, U_lat, V_lat, h, g, l):
        """Binarise latent factors with the oracle's own packer."""
        return cls(pack(V_lat, axis=0), pack(U_lat, axis=1), h, g, l)


def forward(x: np.ndarray, branches: Sequence[Branch], in_f: int, out_f: int, r: int,
            rows: Optional[Sequence[int]] = None) -> np.ndarray:
    """y = sum_b h_b * (sign(U_b) @ (l_b * (sign(V_b)^T @ (g_b * x)))) in fp64.

    x is (M, in) or (in,); returns (M, out) or (M, len(rows)).
    """
    lib = _load()
    xx = np.ascontiguousarray(np.atleast_2d(x), dtype=np.float64)
    M = xx.shape[0]
    if xx.shape[1] != in_f:
        raise ValueError("x has the wrong width")
    nb = len(branches)
    for b in branches:
        if b.Vp.shape[0] != r or b.Up.shape[0] != out_f:
            raise ValueError("packed factor shapes do not match (in, out, r)")
        if b.h.shape[0] != out_f or b.g.shape[0] != in_f or b.l.shape[0] != r:
            raise ValueError("scale lengths do not match (in, out, r)")
    ldv = branches[0].Vp.shape[1]
    ldu = branches[0].Up.shape[1]
    arr = lambda vals: (ctypes.c_void_p * nb)(*vals)
    Vp = arr([_ptr(b.Vp) for b in branches])
    Up = arr([_ptr(b.Up) for b in branches])
    h = arr([_ptr(b.h) for b in branches])
    g = arr([_ptr(b.g) for b in branches])
    l = arr([_ptr(b.l) for b in branches])
    if rows is None:
        ny, rows_p, n_rows, keep = out_f, None, 0, None
    else:
        keep = np.ascontiguousarray(rows, dtype=np.int64)
        ny, rows_p, n_rows = keep.shape[0], _ptr(keep), keep.shape[0]
    y = np.empty((M, ny), dtype=np.float64)
    rc = lib.lbo_forward(_ptr(xx), M, in_f, out_f, r, nb,
                         ctypes.cast(Vp, ctypes.c_void_p), ldv,
                         ctypes.cast(Up, ctypes.c_void_p), ldu,
                         ctypes.cast(h, ctypes.c_void_p), ctypes.cast(g, ctypes.c_void_p),
                         ctypes.cast(l, ctypes.c_void_p), rows_p, n_rows, _ptr(y))
    del keep
    if rc != 0:
        raise ValueError("lbo_forward rejected its arguments")
    return y


def _check_branches(branches, in_f, out_f, r):
    for b in branches:
        if b.Vp.shape[0] != r or b.Up.shape[0] != out_f:
            raise ValueError("packed factor shapes do not match (in, out, r)")
        if b.h.shape[0] != out_f or b.g.shape[0] != in_f or b.l.shape[0] != r:
            raise ValueError("scale lengths do not match (in, out, r)")


def forward_xor(x: np.ndarray, branches: Sequence[Branch], in_f: int, out_f: int, r: int,
                bits: int = 16) -> np.ndarray:
    """The bit-serial (XOR / popcount) variant of the layer, per its definition in
    lb_oracle.c: each vector quantised to ``bits``-bit odd-integer codes (fp32
    decisions), exact integer contractions, y in fp64.  x is (M, in) or (in,)."""
    lib = _load()
    xx = np.ascontiguousarray(np.atleast_2d(x), dtype=np.float64)
    M = xx.shape[0]
    if xx.shape[1] != in_f:
        raise ValueError("x has the wrong width")
    _check_branches(branches, in_f, out_f, r)
    nb = len(branches)
    arr = lambda vals: ctypes.cast((ctypes.c_void_p * nb)(*vals), ctypes.c_void_p)
    y = np.empty((M, out_f), dtype=np.float64)
    rc = lib.lbo_forward_xor(_ptr(xx), M, in_f, out_f, r, nb, int(bits),
                             arr([_ptr(b.Vp) for b in branches]), branches[0].Vp.shape[1],
                             arr([_ptr(b.Up) for b in branches]), branches[0].Up.shape[1],
                             arr([_ptr(b.h) for b in branches]), arr([_ptr(b.g) for b in branches]),
                             arr([_ptr(b.l) for b in branches]), _ptr(y))
    if rc != 0:
        raise ValueError("lbo_forward_xor rejected its arguments")
    return y


def xor_quantise(v: np.ndarray, bits: int = 16):
    """(D, codes) of the bit-serial variant's quantiser for the fp32 vector v."""
    vv = np.ascontiguousarray(v, dtype=np.float32).reshape(-1)
    codes = np.empty(vv.shape[0], dtype=np.int64)
    D = _load().lbo_xor_quantise(_ptr(vv), vv.shape[0], int(bits), _ptr(codes))
    return float(D), codes
