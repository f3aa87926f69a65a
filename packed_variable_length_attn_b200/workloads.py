"""Seeded synthetic packed-varlen inputs shared by the tests, the benchmark and
the CPU oracle's callers.

This module draws random numbers and lays them out; it contains none of the
attention arithmetic. Everything is generated on the CPU with a
``torch.Generator`` so that the same seed gives the same bits on every
machine. Draw order for every workload: sequence lengths first, then Q, K, V
(fp32 standard normal, rounded to nearest-even bf16), then the per-pair bias
grid, then the per-key bias.

The five named workloads stand in for the pages' datasets (GenRec prompts on
Qwen2.5-0.5B, GiGL graph batches, a short GQA training row), which are not
available here; they keep the shapes, head splits, length mixes and bias
layouts those pages describe.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional, Sequence

import torch

SEED_BASE = 20261202


@dataclass
class Workload:
    name: str
    lengths_q: list
    lengths_k: list
    cu_q: torch.Tensor            # int32 [B+1]
    cu_k: torch.Tensor            # int32 [B+1]
    q: torch.Tensor               # [Tq, Hq, D]
    k: torch.Tensor               # [Tk, Hkv, D]
    v: torch.Tensor               # [Tk, Hkv, D]
    n_heads: int
    n_kv_heads: int
    head_dim: int
    causal: bool
    softmax_scale: float
    bias_key: Optional[torch.Tensor] = None    # fp32 [Tk, Hq]
    bias_pair: Optional[torch.Tensor] = None   # fp32 storage of the per-pair grid
    bias_strides: tuple = (0, 0, 0, 0)         # (sb, sh, sr, sc) in elements
    meta: dict = field(default_factory=dict)

    @property
    def batch(self) -> int:
        return len(self.lengths_q)

    @property
    def total_q(self) -> int:
        return int(self.cu_q[-1])

    @property
    def total_k(self) -> int:
        return int(self.cu_k[-1])

    @property
    def max_seqlen_q(self) -> int:
        return max(self.lengths_q) if self.lengths_q else 0

    @property
    def max_seqlen_k(self) -> int:
        return max(self.lengths_k) if self.lengths_k else 0


def _cumsum(lengths: Sequence[int]) -> torch.Tensor:
    cu = [0]
    for L in lengths:
        cu.append(cu[-1] + int(L))
    return torch.tensor(cu, dtype=torch.int32)


def _normal(shape, g, dtype, std=1.0):
    x = torch.randn(*shape, generator=g, dtype=torch.float32)
    if std != 1.0:
        x = x * std
    return x.to(dtype)


def make_custom(lengths_q, lengths_k=None, n_heads=2, n_kv_heads=None, head_dim=64,
                causal=True, seed=0, dtype=torch.bfloat16, bias_key=False, bias_pair=None,
                bias_key_std=1.0, softmax_scale=None, name="custom",
                g: Optional[torch.Generator] = None) -> Workload:
    """A packed batch with the given per-sequence lengths.

    ``bias_pair``: None, or a 4-tuple ``(B, H_grid, R, C)`` for a contiguous
    fp32 grid read with strides (R*C*H_grid, R*C if H_grid > 1 else 0, C, 1).
    """
    lengths_q = [int(x) for x in lengths_q]
    lengths_k = lengths_q if lengths_k is None else [int(x) for x in lengths_k]
    n_kv_heads = n_heads if n_kv_heads is None else n_kv_heads
    if g is None:
        g = torch.Generator("cpu").manual_seed(int(seed))
    cu_q, cu_k = _cumsum(lengths_q), _cumsum(lengths_k)
    Tq, Tk = int(cu_q[-1]), int(cu_k[-1])
    q = _normal((Tq, n_heads, head_dim), g, dtype)
    k = _normal((Tk, n_kv_heads, head_dim), g, dtype)
    v = _normal((Tk, n_kv_heads, head_dim), g, dtype)
    bp, strides = None, (0, 0, 0, 0)
    if bias_pair is not None:
        Bg, Hg, R, C = bias_pair
        bp = _normal((Bg, Hg, R, C), g, torch.float32)
        strides = (Hg * R * C, R * C if Hg > 1 else 0, C, 1)
    bk = _normal((Tk, n_heads), g, torch.float32, std=bias_key_std) if bias_key else None
    scale = 1.0 / math.sqrt(head_dim) if softmax_scale is None else float(softmax_scale)
    return Workload(name, lengths_q, lengths_k, cu_q, cu_k, q, k, v, n_heads, n_kv_heads,
                    head_dim, bool(causal), scale, bk, bp, strides)


WORKLOADS = {
    1: "tiny_packed_causal",
    2: "genrec_packed_causal_gqa",
    3: "graph_packed_pair_bias",
    4: "short_query_gqa_unequal_lengths",
    5: "long_causal_gqa",
}


def make(config: int, seed: Optional[int] = None) -> Workload:
    """One of the five named workloads; seed defaults to SEED_BASE + config."""
    seed = SEED_BASE + config if seed is None else seed
    g = torch.Generator("cpu").manual_seed(int(seed))
    name = WORKLOADS[config]
    if config == 1:
        # 4 sequences {5,17,32,64} (118 tokens), 2 = 2 heads, D 64, causal.
        w = make_custom([5, 17, 32, 64], n_heads=2, n_kv_heads=2, head_dim=64, causal=True,
                        name=name, g=g)
    elif config == 2:
        # 20 GenRec prompts, lengths U[128, 2048], 14/2 heads (Qwen2.5-0.5B), D 64, causal.
        lengths = torch.randint(128, 2048 + 1, (20,), generator=g).tolist()
        w = make_custom(lengths, n_heads=14, n_kv_heads=2, head_dim=64, causal=True,
                        name=name, g=g)
    elif config == 3:
        # 512 graph sequences, lengths U[1, 256], 8 heads, D 64, non-causal; a one-head
        # fp32 pair grid [512,1,256,256] ~N(0,1) and a per-key bias [Tk,8] ~N(0,0.5).
        lengths = torch.randint(1, 256 + 1, (512,), generator=g).tolist()
        w = make_custom(lengths, n_heads=8, n_kv_heads=8, head_dim=64, causal=False,
                        bias_pair=(512, 1, 256, 256), bias_key=True, bias_key_std=0.5,
                        name=name, g=g)
    elif config == 4:
        # 64 rows of 112 queries against 262 keys, 32/8 heads, D 128, bottom-right causal.
        w = make_custom([112] * 64, [262] * 64, n_heads=32, n_kv_heads=8, head_dim=128,
                        causal=True, name=name, g=g)
    elif config == 5:
        # 16 long sequences, lengths U[2048, 8192], 32/8 heads, D 128, causal.
        lengths = torch.randint(2048, 8192 + 1, (16,), generator=g).tolist()
        w = make_custom(lengths, n_heads=32, n_kv_heads=8, head_dim=128, causal=True,
                        name=name, g=g)
    else:
        raise KeyError(f"unknown workload {config}")
    w.meta["seed"] = int(seed)
    w.meta["config"] = int(config)
    return w
