"""Work measures for packed variable-length attention.

A (query, key) pair is *useful* when the mask lets the query see the key: all
Lq*Lk pairs of a sequence without a causal mask, and with the bottom-right
causal mask the pairs with c <= r + (Lk - Lq). Only useful pairs are counted:
a packed stream pays for its real sequences alone, where a dense mask over the
whole stream would pay for (sum L)^2 pairs and left padding for B * max(L)^2
(page "pack the GenRec training forward through FlashAttention-2", Choosing
the kernel, the 8 x 128 example).

Useful FLOPs = 4 * D * Hq * pairs: one multiply-add per head dimension for
the score and one for the value product.
"""
from __future__ import annotations

from typing import Sequence


def causal_pairs(lq: int, lk: int) -> int:
    """Sum over rows r < lq of clamp(r + lk - lq + 1, 0, lk), in closed form."""
    if lq <= 0 or lk <= 0:
        return 0
    off = lk - lq
    total = 0
    # rows with r + off + 1 >= lk see every key
    r_full = max(0, min(lq, lk - off - 1))  # first row index that sees all lk keys
    total += (lq - r_full) * lk
    # rows r in [r0, r_full) with 1 <= r + off + 1 < lk see r + off + 1 keys
    r0 = max(0, -off)
    if r_full > r0:
        a = r0 + off + 1
        b = r_full - 1 + off + 1
        total += (a + b) * (r_full - r0) // 2
    return total


def useful_pairs(lengths_q: Sequence[int], lengths_k: Sequence[int], causal: bool) -> int:
    total = 0
    for lq, lk in zip(lengths_q, lengths_k):
        total += causal_pairs(int(lq), int(lk)) if causal else int(lq) * int(lk)
    return total


def useful_flops(lengths_q, lengths_k, causal, n_heads, head_dim) -> int:
    return 4 * int(head_dim) * int(n_heads) * useful_pairs(lengths_q, lengths_k, causal)


def algorithmic_bytes(w) -> int:
    """Bytes one forward must move at least: Q, K, V read once (bf16), O
    written once (bf16), LSE written (fp32 [Hq, Tq]), the per-key bias read
    once (fp32 [Tk, Hq]) and, of the per-pair grid, only the in-sequence
    entries (Lq_i x Lk_i per sequence, per head unless the grid broadcasts
    heads), read once."""
    e = 2  # bf16
    tq, tk = w.total_q, w.total_k
    b = tq * w.n_heads * w.head_dim * e * 2             # Q read, O written
    b += 2 * tk * w.n_kv_heads * w.head_dim * e         # K, V
    b += tq * w.n_heads * 4                              # LSE
    if w.bias_key is not None:
        b += tk * w.n_heads * 4
    if w.bias_pair is not None:
        heads = 1 if w.bias_strides[1] == 0 else w.n_heads
        b += 4 * heads * sum(int(lq) * int(lk) for lq, lk in zip(w.lengths_q, w.lengths_k))
    return b
