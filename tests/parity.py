"""Helpers for GPU-vs-oracle parity tests."""
import numpy as np
import torch

import oracle
from packed_variable_length_attn_b200 import varlen_attn_fwd

# Tolerances for bf16 inputs (O: max-abs and relative L2 over the compared
# rows), fp32 inputs (relative L2). LSE tolerances are this library's own
# (the pages give none): the scores are exact fp32 sums of exact bf16
# products, so LSE error comes only from the fp32 exp/log approximations and
# the running sum, far below 1e-3.
BF16_MAX_ABS = 2e-2
BF16_REL_L2 = 1e-2
BF16_LSE_ABS = 1e-3
F32_REL_L2 = 1e-4
F32_LSE_ABS = 1e-5


def to_device(w, device="cuda"):
    d = {
        "q": w.q.to(device), "k": w.k.to(device), "v": w.v.to(device),
        "cu_q": w.cu_q.to(device), "cu_k": w.cu_k.to(device),
        "bias_key": None if w.bias_key is None else w.bias_key.to(device),
        "bias_pair": None if w.bias_pair is None else w.bias_pair.to(device),
    }
    return d


def run_gpu(w, dev=None, **kw):
    dev = dev or to_device(w)
    strides = w.bias_strides if w.bias_pair is not None else None
    out, lse = varlen_attn_fwd(dev["q"], dev["k"], dev["v"], dev["cu_q"], dev["cu_k"],
                               w.max_seqlen_q, w.max_seqlen_k, softmax_scale=w.softmax_scale,
                               causal=w.causal, bias_per_key=dev["bias_key"],
                               bias_pair=dev["bias_pair"], bias_pair_strides=strides, **kw)
    torch.cuda.synchronize()
    return out, lse


def run_oracle(w):
    return oracle.fwd(w.q, w.k, w.v, w.cu_q, w.cu_k, w.n_heads, w.n_kv_heads, w.softmax_scale,
                      w.causal, bias_key=w.bias_key, bias_pair=w.bias_pair,
                      bias_strides=w.bias_strides)


def compare(out, lse, ref_out, ref_lse, fp32=False):
    """Element-wise comparison; returns a dict of error figures, asserts the bar."""
    o = out.float().cpu().numpy().astype(np.float64)
    l = lse.float().cpu().numpy().astype(np.float64)
    ref_out = np.asarray(ref_out, dtype=np.float64)
    ref_lse = np.asarray(ref_lse, dtype=np.float64)
    assert o.shape == ref_out.shape and l.shape == ref_lse.shape
    assert np.isfinite(o).all(), "non-finite output"
    diff = o - ref_out
    max_abs = float(np.abs(diff).max()) if diff.size else 0.0
    denom = float(np.linalg.norm(ref_out))
    rel_l2 = float(np.linalg.norm(diff) / denom) if denom > 0 else float(np.linalg.norm(diff))
    inf_ref = np.isinf(ref_lse)
    assert np.array_equal(np.isinf(l), inf_ref), "LSE -inf pattern differs"
    assert (l[inf_ref] < 0).all()
    lse_abs = float(np.abs(l[~inf_ref] - ref_lse[~inf_ref]).max()) if (~inf_ref).any() else 0.0
    res = {"max_abs": max_abs, "rel_l2": rel_l2, "lse_abs": lse_abs}
    if fp32:
        assert rel_l2 <= F32_REL_L2, res
        assert lse_abs <= F32_LSE_ABS, res
    else:
        assert max_abs <= BF16_MAX_ABS, res
        assert rel_l2 <= BF16_REL_L2, res
        assert lse_abs <= BF16_LSE_ABS, res
    return res


def sample_rows(w, n, seed):
    """(seq, head, local row) samples: random rows plus every sequence's first
    and last row and the rows at 128-row block edges."""
    g = np.random.default_rng(seed)
    seqs = [i for i in range(w.batch) if w.lengths_q[i] > 0]
    out = set()
    for i in seqs:
        L = w.lengths_q[i]
        for r in {0, L - 1, min(127, L - 1), min(128, L - 1)}:
            out.add((i, int(g.integers(w.n_heads)), r))
    while len(out) < n + len(seqs):
        i = seqs[int(g.integers(len(seqs)))]
        out.add((i, int(g.integers(w.n_heads)), int(g.integers(w.lengths_q[i]))))
    s = sorted(out)
    return [x[0] for x in s], [x[1] for x in s], [x[2] for x in s]


def stratified_rows(w, rows_per_block=4, seed=0):
    """(seq, head, local row) samples covering every (sequence, 128-row
    q-block): its first and last row plus rows_per_block - 2 random rows,
    each on one head drawn at random from every K/V group."""
    g = np.random.default_rng(seed)
    G = w.n_heads // w.n_kv_heads
    out = set()
    for i in range(w.batch):
        L = w.lengths_q[i]
        for b0 in range(0, L, 128):
            b1 = min(b0 + 128, L) - 1
            rows = {b0, b1}
            while len(rows) < min(rows_per_block, b1 - b0 + 1):
                rows.add(int(g.integers(b0, b1 + 1)))
            for r in rows:
                for kvh in range(w.n_kv_heads):
                    out.add((i, kvh * G + int(g.integers(G)), r))
    s = sorted(out)
    return [x[0] for x in s], [x[1] for x in s], [x[2] for x in s]


def compare_rows(w, out, lse, seq, head, row):
    ro, rl = oracle.rows(w.q, w.k, w.v, w.cu_q, w.cu_k, w.n_heads, w.n_kv_heads,
                         w.softmax_scale, w.causal, seq, head, row, bias_key=w.bias_key,
                         bias_pair=w.bias_pair, bias_strides=w.bias_strides)
    t = torch.tensor([int(w.cu_q[s]) + r for s, r in zip(seq, row)])
    h = torch.tensor(head)
    go = out.cpu()[t, h]
    gl = lse.cpu()[h, t]
    return compare(go, gl, ro, rl)


def compare_sampled(w, out, lse, n=256, seed=0):
    return compare_rows(w, out, lse, *sample_rows(w, n, seed))


def compare_stratified(w, out, lse, rows_per_block=4, seed=0):
    return compare_rows(w, out, lse, *stratified_rows(w, rows_per_block, seed))
