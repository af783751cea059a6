"""Python binding of liblb.so — the B200 LittleBit factorised binary linear layer.

Argument marshalling only: every step of the forward runs in the CUDA kernels
behind the C ABI declared in ``include/lb.h``.  PyTorch supplies device memory
and streams.  There is no CPU fallback: if ``liblb.so`` has not been built, the
first call raises.

Names follow the layer's formula

    y = sum_b h_b * (sign(U_b) @ (l_b * (sign(V_b)^T @ (g_b * x))))

("Samsung LittleBit: A 13B LLM Under 1 GB ...", section "How it works").
"""
from __future__ import annotations

import ctypes
import os
from typing import List, Optional, Sequence

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "liblb.so")

LB_OK, LB_ERR_INVALID_ARG, LB_ERR_ALIGNMENT, LB_ERR_UNSUPPORTED, LB_ERR_CUDA, \
    LB_ERR_TIMEOUT, LB_ERR_WORKSPACE = range(7)
LB_F16, LB_BF16, LB_F32 = 0, 1, 2
LB_Q, LB_K, LB_V, LB_O, LB_GATE, LB_UP, LB_DOWN = range(7)
PROJ_NAMES = ("q", "k", "v", "o", "gate", "up", "down")
LB_STACK_MLP_ONLY = 1

_DTYPES = {torch.float16: LB_F16, torch.bfloat16: LB_BF16, torch.float32: LB_F32}


class LbError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what} failed: {status_string(status)}")


LB_LAYOUT_ROWS, LB_LAYOUT_SLICES = 0, 1
LAYOUTS = {"rows": LB_LAYOUT_ROWS, "slices": LB_LAYOUT_SLICES}


class lb_branch(ctypes.Structure):
    _fields_ = [("Vp", ctypes.c_void_p), ("Up", ctypes.c_void_p), ("h", ctypes.c_void_p),
                ("g", ctypes.c_void_p), ("l", ctypes.c_void_p), ("ld_v", ctypes.c_int64),
                ("ld_u", ctypes.c_int64), ("layout", ctypes.c_int32),
                ("reserved", ctypes.c_int32)]


class lb_stack_desc(ctypes.Structure):
    _fields_ = [("n_layers", ctypes.c_int), ("hidden", ctypes.c_int), ("inter", ctypes.c_int),
                ("n_heads", ctypes.c_int), ("n_kv_heads", ctypes.c_int),
                ("head_dim", ctypes.c_int), ("n_branches", ctypes.c_int),
                ("flags", ctypes.c_int), ("lin", ctypes.c_void_p), ("ranks", ctypes.c_void_p)]


EXPORTS = ("lb_status_string", "lb_version", "lb_pack_signs", "lb_linear_forward",
           "lb_linear_workspace_size", "lb_linear_path", "lb_stack_workspace_size",
           "lb_stack_prepare", "lb_stack_forward", "lb_stack_forward_host",
           "lb_workspace_status", "lb_stack_output", "lb_linear_forward_noalloc",
           "lb_noalloc_scratch_bytes", "lb_pack_signs_sliced", "lb_packed_words",
           "lb_stack_plan_host", "lb_linear_forward_xor", "lb_linear_xor_workspace_size",
           "lb_dual_svid", "lb_dual_svid_workspace_size")

_lib = None


def lib() -> ctypes.CDLL:
    """Load liblb.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m binary_rank_linear_lb_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i64, sz, st = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t, ctypes.c_int
        L.lb_status_string.argtypes = [st]
        L.lb_status_string.restype = ctypes.c_char_p
        L.lb_version.restype = ctypes.c_int
        L.lb_pack_signs.argtypes = [vp, i64, i64, i64, ctypes.c_int, vp, i64, vp]
        L.lb_pack_signs.restype = st
        L.lb_pack_signs_sliced.argtypes = [vp, i64, i64, i64, ctypes.c_int, vp, vp]
        L.lb_pack_signs_sliced.restype = st
        L.lb_packed_words.argtypes = [i64, i64, ctypes.c_int, i64]
        L.lb_packed_words.restype = sz
        L.lb_linear_forward.argtypes = [vp, st, i64, i64, i64, i64, vp, ctypes.c_int, vp, vp,
                                        sz, vp]
        L.lb_linear_forward.restype = st
        L.lb_linear_workspace_size.argtypes = [i64, i64, i64, i64, ctypes.c_int]
        L.lb_linear_workspace_size.restype = sz
        L.lb_linear_path.argtypes = [i64, i64, i64, i64]
        L.lb_linear_path.restype = ctypes.c_int
        L.lb_stack_workspace_size.argtypes = [vp]
        L.lb_stack_workspace_size.restype = sz
        L.lb_stack_prepare.argtypes = [vp, vp, sz, vp]
        L.lb_stack_prepare.restype = st
        L.lb_stack_plan_host.argtypes = [vp, ctypes.c_int, vp, sz, vp, vp]
        L.lb_stack_plan_host.restype = st
        L.lb_stack_forward.argtypes = [vp, vp, sz, vp, vp, vp]
        L.lb_stack_forward.restype = st
        L.lb_stack_forward_host.argtypes = [vp, vp, sz, vp, vp, vp]
        L.lb_stack_forward_host.restype = st
        L.lb_workspace_status.argtypes = [vp, vp]
        L.lb_workspace_status.restype = st
        L.lb_stack_output.argtypes = [vp, vp, ctypes.c_int, ctypes.c_int]
        L.lb_stack_output.restype = vp
        L.lb_linear_forward_noalloc.argtypes = [vp, st, i64, i64, i64, i64, vp, ctypes.c_int, vp,
                                                vp]
        L.lb_linear_forward_noalloc.restype = st
        L.lb_noalloc_scratch_bytes.restype = sz
        L.lb_linear_forward_xor.argtypes = [vp, st, i64, i64, i64, i64, vp, ctypes.c_int,
                                            ctypes.c_int, vp, vp, sz, vp]
        L.lb_linear_forward_xor.restype = st
        L.lb_linear_xor_workspace_size.argtypes = [i64, i64, i64, i64, ctypes.c_int, ctypes.c_int]
        L.lb_linear_xor_workspace_size.restype = sz
        L.lb_dual_svid.argtypes = [vp, i64, i64, i64, ctypes.c_int, ctypes.c_int, vp, vp, vp, vp,
                                   vp, vp, sz, vp]
        L.lb_dual_svid.restype = st
        L.lb_dual_svid_workspace_size.argtypes = [i64, i64, i64, ctypes.c_int]
        L.lb_dual_svid_workspace_size.restype = sz
        _lib = L
    return _lib


def status_string(s: int) -> str:
    return lib().lb_status_string(int(s)).decode()


def _check(status: int, what: str) -> None:
    if status != LB_OK:
        raise LbError(status, what)


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


# ------------------------------------------------------------------ packing
def packed_words(n: int, k: int, layout: int = LB_LAYOUT_ROWS, ld_words: int = 0) -> int:
    """Words a packed matrix of n rows of k signs occupies (lb_packed_words)."""
    return int(lib().lb_packed_words(n, k, int(layout), int(ld_words)))


def pack_signs(latent: torch.Tensor, axis: int, ld_words: Optional[int] = None,
               out: Optional[torch.Tensor] = None, stream=None,
               layout: int = LB_LAYOUT_ROWS) -> torch.Tensor:
    """Packed sign words (int32 storage of uint32 words) of an fp32 latent.

    axis=1: n = rows packed rows of k = cols signs (U: out x r); axis=0: n = cols
    packed rows of k = rows signs (V: in x r).  LB_LAYOUT_ROWS gives [n][ld_words]
    (default ceil(k/32)); LB_LAYOUT_SLICES gives the sliced layout as a flat tensor
    of packed_words(n, k, LB_LAYOUT_SLICES) words.
    """
    rows, cols = latent.shape
    k = cols if axis == 1 else rows
    n = rows if axis == 1 else cols
    ld = latent.stride(0) if latent.dim() == 2 else cols
    if latent.stride(-1) != 1:
        raise ValueError("latent must have unit stride along its columns")
    if layout == LB_LAYOUT_SLICES:
        if out is None:
            out = torch.empty(packed_words(n, k, LB_LAYOUT_SLICES), dtype=torch.int32,
                              device=latent.device)
        _check(lib().lb_pack_signs_sliced(_ptr(latent), rows, cols, ld, int(axis), _ptr(out),
                                          _stream(stream)), "lb_pack_signs_sliced")
        return out
    ldw = (k + 31) // 32 if ld_words is None else int(ld_words)
    if out is None:
        out = torch.empty((n, ldw), dtype=torch.int32, device=latent.device)
    _check(lib().lb_pack_signs(_ptr(latent), rows, cols, ld, int(axis), _ptr(out), ldw,
                               _stream(stream)), "lb_pack_signs")
    return out


def _slice_pitch(nw: int, s: int) -> int:
    last = (nw - 1) // 16
    return 16 if s < last else (nw - 16 * last + 3) // 4 * 4


def slice_words(words: torch.Tensor, k: int) -> torch.Tensor:
    """Row-major packed words [n][>= ceil(k/32)] regrouped into LB_LAYOUT_SLICES (flat)."""
    n, nw = words.shape[0], (k + 31) // 32
    blocks = []
    for s in range((nw + 15) // 16):
        w = words[:, 16 * s:min(16 * s + 16, nw)]
        pitch = _slice_pitch(nw, s)
        if w.shape[1] < pitch:
            w = torch.cat([w, torch.zeros((n, pitch - w.shape[1]), dtype=w.dtype,
                                          device=w.device)], dim=1)
        blocks.append(w.reshape(-1))
    return torch.cat(blocks).contiguous()


def unslice_words(flat: torch.Tensor, n: int, k: int) -> torch.Tensor:
    """Inverse of slice_words: [n][ceil(k/32)] row-major words of a sliced matrix."""
    nw = (k + 31) // 32
    cols, off = [], 0
    for s in range((nw + 15) // 16):
        pitch = _slice_pitch(nw, s)
        block = flat[off:off + n * pitch].reshape(n, pitch)
        cols.append(block[:, :min(16, nw - 16 * s)])
        off += n * pitch
    return torch.cat(cols, dim=1)


# ------------------------------------------------------------------ one linear
class Branch:
    """Device tensors of one branch: packed signs (in `layout`) and FP16 scales."""

    def __init__(self, Vp: torch.Tensor, Up: torch.Tensor, h: torch.Tensor, g: torch.Tensor,
                 l: torch.Tensor, layout: int = LB_LAYOUT_ROWS):
        self.Vp, self.Up, self.h, self.g, self.l = Vp, Up, h, g, l
        self.layout = layout

    def c_struct(self) -> lb_branch:
        rows = self.layout == LB_LAYOUT_ROWS
        return lb_branch(_ptr(self.Vp), _ptr(self.Up), _ptr(self.h), _ptr(self.g), _ptr(self.l),
                         self.Vp.shape[1] if rows else 0, self.Up.shape[1] if rows else 0,
                         self.layout, 0)

    @property
    def nbytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in (self.Vp, self.Up, self.h, self.g, self.l))


def linear_workspace_size(M: int, in_f: int, out_f: int, r: int, n_branches: int) -> int:
    return int(lib().lb_linear_workspace_size(M, in_f, out_f, r, n_branches))


def linear_path(M: int, in_f: int, out_f: int, r: int) -> int:
    return int(lib().lb_linear_path(M, in_f, out_f, r))


def linear_forward(x: torch.Tensor, branches: Sequence[Branch], in_f: int, out_f: int, r: int,
                   y: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                   stream=None) -> torch.Tensor:
    """y (M x out, fp32) = the factorised layer applied to x (M x in)."""
    x2 = x if x.dim() == 2 else x.reshape(1, -1)
    M = x2.shape[0]
    if y is None:
        y = torch.empty((M, out_f), dtype=torch.float32, device=x.device)
    nb = len(branches)
    if workspace is None:
        workspace = torch.empty(linear_workspace_size(M, in_f, out_f, r, nb), dtype=torch.uint8,
                                device=x.device)
    arr = (lb_branch * nb)(*[b.c_struct() for b in branches])
    dt = _DTYPES.get(x2.dtype)
    if dt is None:
        raise ValueError(f"unsupported x dtype {x2.dtype}")
    _check(lib().lb_linear_forward(_ptr(x2), dt, M, in_f, out_f, r, ctypes.addressof(arr), nb,
                                   _ptr(y), _ptr(workspace), workspace.numel(), _stream(stream)),
           "lb_linear_forward")
    return y


def linear_forward_noalloc(x: torch.Tensor, branches: Sequence[Branch], in_f: int, out_f: int,
                           r: int, y: torch.Tensor, stream=None) -> torch.Tensor:
    """lb_linear_forward_noalloc: like linear_forward, with the library's own fixed scratch.

    For callers that cannot allocate device memory; `y` (M x out, fp32) must be given.
    """
    x2 = x if x.dim() == 2 else x.reshape(1, -1)
    nb = len(branches)
    arr = (lb_branch * nb)(*[b.c_struct() for b in branches])
    dt = _DTYPES.get(x2.dtype)
    if dt is None:
        raise ValueError(f"unsupported x dtype {x2.dtype}")
    _check(lib().lb_linear_forward_noalloc(_ptr(x2), dt, x2.shape[0], in_f, out_f, r,
                                           ctypes.addressof(arr), nb, _ptr(y), _stream(stream)),
           "lb_linear_forward_noalloc")
    return y


def linear_forward_xor(x: torch.Tensor, branches: Sequence[Branch], in_f: int, out_f: int,
                       r: int, bits: int = 16, y: Optional[torch.Tensor] = None,
                       workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """lb_linear_forward_xor: the bit-serial (XOR / popcount) variant, activations
    quantised to ``bits``-bit sign-plane codes; y (M x out, fp32)."""
    x2 = x if x.dim() == 2 else x.reshape(1, -1)
    M = x2.shape[0]
    if y is None:
        y = torch.empty((M, out_f), dtype=torch.float32, device=x.device)
    nb = len(branches)
    if workspace is None:
        n = int(lib().lb_linear_xor_workspace_size(M, in_f, out_f, r, nb, bits))
        if n == 0:
            raise LbError(LB_ERR_INVALID_ARG, "lb_linear_xor_workspace_size")
        workspace = torch.empty(n, dtype=torch.uint8, device=x.device)
    arr = (lb_branch * nb)(*[b.c_struct() for b in branches])
    dt = _DTYPES.get(x2.dtype)
    if dt is None:
        raise ValueError(f"unsupported x dtype {x2.dtype}")
    _check(lib().lb_linear_forward_xor(_ptr(x2), dt, M, in_f, out_f, r, ctypes.addressof(arr), nb,
                                       int(bits), _ptr(y), _ptr(workspace), workspace.numel(),
                                       _stream(stream)), "lb_linear_forward_xor")
    return y


def dual_svid(W: torch.Tensor, r: int, n_branches: int = 2, layout: int = LB_LAYOUT_SLICES,
              stream=None) -> List[Branch]:
    """lb_dual_svid: the branches of a factorised layer initialised from the dense
    fp32 weight W (out x in) by Dual-SVID, packed in ``layout``."""
    out_f, in_f = W.shape
    W = W.contiguous()
    dev = W.device
    brs = []
    for _ in range(n_branches):
        if layout == LB_LAYOUT_SLICES:
            Vp = torch.empty(packed_words(r, in_f, layout), dtype=torch.int32, device=dev)
            Up = torch.empty(packed_words(out_f, r, layout), dtype=torch.int32, device=dev)
        else:
            Vp = torch.empty((r, (in_f + 31) // 32), dtype=torch.int32, device=dev)
            Up = torch.empty((out_f, (r + 31) // 32), dtype=torch.int32, device=dev)
        brs.append(Branch(Vp, Up, torch.empty(out_f, dtype=torch.float16, device=dev),
                          torch.empty(in_f, dtype=torch.float16, device=dev),
                          torch.empty(r, dtype=torch.float16, device=dev), layout))
    n = int(lib().lb_dual_svid_workspace_size(out_f, in_f, r, n_branches))
    if n == 0:
        raise LbError(LB_ERR_INVALID_ARG, "lb_dual_svid_workspace_size")
    ws = torch.empty(n + 256, dtype=torch.uint8, device=dev)
    off = (-ws.data_ptr()) % 256
    arr = lambda ts: (ctypes.c_void_p * n_branches)(*[t.data_ptr() for t in ts])
    _check(lib().lb_dual_svid(_ptr(W), out_f, in_f, r, n_branches, int(layout),
                              arr([b.Vp for b in brs]), arr([b.Up for b in brs]),
                              arr([b.h for b in brs]), arr([b.g for b in brs]),
                              arr([b.l for b in brs]), ws.data_ptr() + off, n, _stream(stream)),
           "lb_dual_svid")
    return brs


def workspace_status(workspace: torch.Tensor, stream=None) -> int:
    return int(lib().lb_workspace_status(_ptr(workspace), _stream(stream)))


# ------------------------------------------------------------------ stacks
class Stack:
    """A prepared decoder stack (or MLP block) over device-resident branches.

    ``linears[layer][proj]`` is a list of Branch (proj in q,k,v,o,gate,up,down order;
    entries may be None for unused projections of an MLP-only block) and
    ``ranks[layer][proj]`` the latent rank of each.
    """

    def __init__(self, linears, ranks, hidden: int, inter: int, n_heads: int = 0,
                 n_kv_heads: int = 0, head_dim: int = 0, mlp_only: bool = False,
                 device=None, stream=None):
        self.n_layers = len(linears)
        self.nb = next(len(p) for L in linears for p in L if p)
        self.hidden, self.inter = hidden, inter
        self._keep = linears
        nb = self.nb
        n = self.n_layers * 7 * nb
        self._lin = (lb_branch * n)()
        self._ranks = (ctypes.c_int64 * (self.n_layers * 7))()
        for li, L in enumerate(linears):
            for p in range(7):
                self._ranks[li * 7 + p] = int(ranks[li][p]) if ranks[li][p] else 0
                if L[p]:
                    for b in range(nb):
                        self._lin[(li * 7 + p) * nb + b] = L[p][b].c_struct()
        self.desc = lb_stack_desc(self.n_layers, hidden, inter, n_heads, n_kv_heads, head_dim, nb,
                                  LB_STACK_MLP_ONLY if mlp_only else 0,
                                  ctypes.addressof(self._lin), ctypes.addressof(self._ranks))
        size = int(lib().lb_stack_workspace_size(ctypes.byref(self.desc)))
        if size == 0:
            raise LbError(LB_ERR_INVALID_ARG, "lb_stack_workspace_size")
        dev = device if device is not None else torch.device("cuda")
        self.workspace = torch.empty(size, dtype=torch.uint8, device=dev)
        self.prepare(stream)

    def prepare(self, stream=None) -> None:
        """(Re)write the plan into the workspace: lb_stack_prepare (also clears a timeout)."""
        _check(lib().lb_stack_prepare(ctypes.byref(self.desc), _ptr(self.workspace),
                                      self.workspace.numel(), _stream(stream)), "lb_stack_prepare")

    def forward(self, x: torch.Tensor, y: Optional[torch.Tensor] = None,
                stream=None) -> torch.Tensor:
        if y is None:
            y = torch.empty(self.hidden, dtype=torch.float32, device=x.device)
        _check(lib().lb_stack_forward(ctypes.byref(self.desc), _ptr(self.workspace),
                                      self.workspace.numel(), _ptr(x), _ptr(y), _stream(stream)),
               "lb_stack_forward")
        return y

    def forward_host(self, x_host: torch.Tensor, y_host: torch.Tensor, stream=None) -> torch.Tensor:
        _check(lib().lb_stack_forward_host(ctypes.byref(self.desc), _ptr(self.workspace),
                                           self.workspace.numel(), _ptr(x_host), _ptr(y_host),
                                           _stream(stream)), "lb_stack_forward_host")
        return y_host

    def output(self, layer: int, proj: int) -> Optional[torch.Tensor]:
        """fp32 output of linear `proj` of `layer` from the last forward (q,k,v,gate,up)."""
        p = lib().lb_stack_output(ctypes.byref(self.desc), _ptr(self.workspace), layer, proj)
        if not p:
            return None
        base = self.workspace.data_ptr()
        off = p - base
        from .configs import proj_shape
        _, out_f = proj_shape(proj, self.hidden, self.inter, self.desc.n_kv_heads * self.desc.head_dim)
        return self.workspace[off:off + 4 * out_f].view(torch.float32)

    def status(self, stream=None) -> int:
        return workspace_status(self.workspace, stream)
