"""CPU oracle for the packed-layout helpers (TEST INFRASTRUCTURE).

Same status as the rest of this package: only the test suite, the benchmark's
CPU legs and ``__graft_entry__.smoke()`` may use it; the product never does.
Plain numpy, written from the definitions below, no blocking or fusion.

Definitions (pages cited by title and section):

``mask_to_seqlens`` — the varlen unpadding step of the FlashAttention-style
pipeline ("Flash Dynamic Mask Attention (FDMA) Into Transformers-Style
Attention", Key Implementation Points, Variable Length Flow): a padded batch
[B, S] with a boolean validity mask becomes one packed stream. The packed
order is row-major over (b, s): batch row b's valid positions, in increasing
s, follow those of rows < b. Returns cu_seqlens [B+1] (cu[b+1] - cu[b] = the
number of valid positions of row b), the flat padded position b*S + s of
every packed row, and the largest per-row count.

``gather_rows`` — packed[t] = padded[indices[t]] (unpad).

``scatter_rows`` — padded[indices[t]] = packed[t], every other padded row 0
(pad).

``fold_pair_row`` — the first-token fold ("[GiGL] pull request 858",
Approach): when a sequence's only query is its first token, row ``row`` of
that sequence's per-pair bias is a per-key bias:
out[cu_k[i] + c, h] = in[cu_k[i] + c, h] + bias_pair[i*sb + hg*sh + row*sr + c*sc]
for c < Lk_i, with hg = h (grid over query heads) or h // G (grid over K/V
heads, ``head_div = G``); in = 0 when no per-key bias is given. Key rows
outside every sequence stay 0 (or the input's value).

``expand_kv_head_grid`` — a per-K/V-head pair grid [B, Hkv, R, C] ("Flash
Dynamic Mask Attention (FDMA) Into Transformers-Style Attention", Key
Implementation Points, Attn Bias Path: attention_bias shaped (batch,
n_kv_heads, q_len, k_len)) read for query head h at K/V head h // G is the
per-query-head grid whose head h is the K/V grid's head h // G.
"""
from __future__ import annotations

import numpy as np


def mask_to_seqlens(mask):
    m = np.asarray(mask).astype(bool)
    B, S = m.shape
    cu = np.zeros(B + 1, dtype=np.int32)
    idx = []
    for b in range(B):
        n = 0
        for s in range(S):
            if m[b, s]:
                idx.append(b * S + s)
                n += 1
        cu[b + 1] = cu[b] + n
    lens = np.diff(cu)
    return cu, np.array(idx, dtype=np.int32), int(lens.max()) if B else 0


def gather_rows(padded_rows, indices):
    x = np.asarray(padded_rows)
    return x[np.asarray(indices, dtype=np.int64)]


def scatter_rows(packed_rows, indices, n_rows):
    x = np.asarray(packed_rows)
    out = np.zeros((int(n_rows),) + x.shape[1:], dtype=x.dtype)
    out[np.asarray(indices, dtype=np.int64)] = x
    return out


def fold_pair_row(bias_pair, strides, row, cu_k, n_heads, total_k, head_div=1, bias_key=None):
    g = np.asarray(bias_pair, dtype=np.float64).reshape(-1)
    sb, sh, sr, sc = (int(x) for x in strides)
    cu = np.asarray(cu_k, dtype=np.int64)
    out = (np.zeros((total_k, n_heads), dtype=np.float64) if bias_key is None
           else np.array(bias_key, dtype=np.float64).reshape(total_k, n_heads).copy())
    for i in range(len(cu) - 1):
        for h in range(n_heads):
            hg = h // head_div
            for c in range(int(cu[i + 1] - cu[i])):
                out[cu[i] + c, h] += g[i * sb + hg * sh + row * sr + c * sc]
    return out


def expand_kv_head_grid(grid, group):
    x = np.asarray(grid)
    return np.repeat(x, int(group), axis=1)
