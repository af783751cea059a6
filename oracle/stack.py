"""Decoder-stack oracle: numpy fp64 glue around the C layer oracle.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

The pages describe the factorised layer only; they say nothing about the rest of
a decoder.  The stack exists to drive the layer the way a Llama-2-shaped decoder
does at batch 1, so the glue takes the plainest reading that keeps activations
bounded through many layers:

  per layer (hidden state h, fp64 here):
    a    = rmsnorm(h)                     weightless, eps = 1e-5
    q, k, v = L_q(a), L_k(a), L_v(a)
    attn = v broadcast over the query heads of its group (attention over a
           context of one position: the softmax over a single key is 1)
    h    = h + L_o(attn)
    a    = rmsnorm(h)
    d    = silu(L_gate(a)) * L_up(a)
    h    = h + L_down(d)

  MLP block without attention, norm or residual (the 7B-shaped MLP workload):
    y = L_down(silu(L_gate(x)) * L_up(x))

Every L_* is ``oracle.forward`` (the layer definition in ``lb_oracle.c``).
"""
from __future__ import annotations

from typing import Dict, List, Sequence

import numpy as np

from . import Branch, forward

RMS_EPS = 1e-5


class Linear:
    """A factorised linear: its branches and its (in, out, r)."""

    def __init__(self, branches: Sequence[Branch], in_f: int, out_f: int, r: int):
        self.branches = list(branches)
        self.in_f, self.out_f, self.r = int(in_f), int(out_f), int(r)

    def __call__(self, a: np.ndarray) -> np.ndarray:
        return forward(a, self.branches, self.in_f, self.out_f, self.r)[0]


def rmsnorm(v: np.ndarray, eps: float = RMS_EPS) -> np.ndarray:
    return v / np.sqrt(np.mean(v * v) + eps)


def silu(v: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):     # exp(-v) -> inf for very negative v gives -0.0
        return v / (1.0 + np.exp(-v))


def gqa_broadcast(v: np.ndarray, n_heads: int, n_kv_heads: int, head_dim: int) -> np.ndarray:
    """Query head q reads key/value head q // (n_heads / n_kv_heads)."""
    group = n_heads // n_kv_heads
    vh = v.reshape(n_kv_heads, head_dim)
    return np.repeat(vh, group, axis=0).reshape(n_heads * head_dim)


def decoder_stack(x: np.ndarray, layers: List[Dict[str, Linear]], n_heads: int,
                  n_kv_heads: int, head_dim: int, keep: bool = False):
    """Run the decoder glue for one token; returns h (and per-linear outputs if keep)."""
    h = np.asarray(x, dtype=np.float64).reshape(-1).copy()
    outs = []
    for L in layers:
        a = rmsnorm(h)
        q, k, v = L["q"](a), L["k"](a), L["v"](a)
        o = L["o"](gqa_broadcast(v, n_heads, n_kv_heads, head_dim))
        h = h + o
        a = rmsnorm(h)
        gate, up = L["gate"](a), L["up"](a)
        down = L["down"](silu(gate) * up)
        h = h + down
        if keep:
            outs.append(dict(q=q, k=k, v=v, o=o, gate=gate, up=up, down=down, h=h.copy()))
    return (h, outs) if keep else h


def mlp_block(x: np.ndarray, gate: Linear, up: Linear, down: Linear) -> np.ndarray:
    """y = down(silu(gate(x)) * up(x)); no norm and no residual."""
    xx = np.asarray(x, dtype=np.float64).reshape(-1)
    return down(silu(gate(xx)) * up(xx))
