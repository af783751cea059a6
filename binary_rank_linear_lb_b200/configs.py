"""Workload shapes: Llama-2-shaped linears and stacks, the rank rule and byte counts.

These are the shapes the layer is measured on (single linear, 7B MLP block,
13B and 70B decoder stacks, 7B gate projection swept over the token batch).
Nothing here computes the layer itself.
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from fractions import Fraction
from typing import Dict, List, Tuple

PROJ_NAMES = ("q", "k", "v", "o", "gate", "up", "down")


def rank_for(bpw: float, in_f: int, out_f: int) -> int:
    """Latent rank per branch for a bits-per-weight target.

    Two branches of binary factors store 2*r*(in+out) sign bits for in*out
    weights, so r = bpw*in*out / (2*(in+out)), rounded down to a multiple of 64.
    """
    exact = Fraction(str(bpw)) * in_f * out_f / (2 * (in_f + out_f)) / 64
    return int(math.floor(exact)) * 64


def proj_shape(p: int, hidden: int, inter: int, kv_dim: int) -> Tuple[int, int]:
    """(in, out) of projection p in q, k, v, o, gate, up, down order."""
    return [(hidden, hidden), (hidden, kv_dim), (hidden, kv_dim), (hidden, hidden),
            (hidden, inter), (hidden, inter), (inter, hidden)][p]


def linear_bytes(in_f: int, out_f: int, r: int, n_branches: int = 2) -> int:
    """Algorithmic bytes of one linear: packed signs of U and V plus FP16 h, g, l."""
    signs = n_branches * r * (in_f + out_f) // 8
    scales = n_branches * 2 * (in_f + out_f + r)
    return signs + scales


def linear_flops(M: int, in_f: int, out_f: int, r: int, n_branches: int = 2) -> int:
    """Multiply-add flops of the two contractions of every branch (2 per MAC)."""
    return 2 * M * r * (in_f + out_f) * n_branches


@dataclass(frozen=True)
class Model:
    name: str
    hidden: int
    inter: int
    n_layers: int
    n_heads: int
    n_kv_heads: int
    head_dim: int = 128

    @property
    def kv_dim(self) -> int:
        return self.n_kv_heads * self.head_dim

    def shapes(self) -> List[Tuple[int, int]]:
        return [proj_shape(p, self.hidden, self.inter, self.kv_dim) for p in range(7)]

    def ranks(self, bpw: float) -> List[int]:
        return [rank_for(bpw, i, o) for i, o in self.shapes()]

    def bytes_per_token(self, bpw: float, n_layers: int = 0) -> int:
        nl = n_layers or self.n_layers
        return nl * sum(linear_bytes(i, o, r) for (i, o), r in zip(self.shapes(), self.ranks(bpw)))


LLAMA2_7B = Model("llama2-7b", 4096, 11008, 32, 32, 32)
LLAMA2_13B = Model("llama2-13b", 5120, 13824, 40, 40, 40)
LLAMA2_70B = Model("llama2-70b", 8192, 28672, 80, 64, 8)
MODELS: Dict[str, Model] = {m.name: m for m in (LLAMA2_7B, LLAMA2_13B, LLAMA2_70B)}

# The small single-linear case the oracle finishes instantly.
SINGLE = dict(in_f=512, out_f=256, r=32, M=1)
MLP7B_BPW = (1.0, 0.55, 0.3, 0.1)
STACK13B_BPW = (0.55, 0.1)
STACK70B_BPW = (1.0, 0.55)
PREFILL_BPW = (1.0, 0.1)
PREFILL_M = (1, 8, 64, 512, 4096)


def stored_model_bytes(model: Model, bpw: float, vocab: int = 32000) -> int:
    """Whole-model bytes in this format: factorised blocks plus FP16 embedding and head."""
    return model.bytes_per_token(bpw) + 2 * 2 * vocab * model.hidden
