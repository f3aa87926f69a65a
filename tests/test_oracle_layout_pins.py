"""Pins for the layout-helper oracle (oracle/layout.py): hand-worked examples
(tests/golden/layout_examples.json), round-trip and ordering invariants, and
the first-token fold tied to the attention oracle itself (a per-pair bias
seen by a single query row is a per-key bias)."""
import json
import os

import numpy as np
import pytest

import oracle
from oracle import layout
from packed_variable_length_attn_b200 import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "layout_examples.json")


def _golden():
    with open(GOLDEN) as f:
        return json.load(f)


@pytest.mark.parametrize("ex", _golden()["unpad"], ids=lambda e: e["name"])
def test_unpad_hand_examples(ex):
    cu, idx, mx = layout.mask_to_seqlens(np.array(ex["mask"]))
    assert cu.tolist() == ex["cu_seqlens"]
    assert idx.tolist() == ex["indices"]
    assert mx == ex["max_seqlen"]


@pytest.mark.parametrize("ex", _golden()["fold"], ids=lambda e: e["name"])
def test_fold_hand_example(ex):
    B, H, R, C = ex["grid_shape"]
    i, h, r, c = np.meshgrid(np.arange(B), np.arange(H), np.arange(R), np.arange(C), indexing="ij")
    grid = (100 * i + 10 * h + 3 * r + c).astype(np.float64)
    cu_k = np.concatenate([[0], np.cumsum(ex["lengths_k"])])
    out = layout.fold_pair_row(grid, ex["strides"], ex["row"], cu_k, ex["n_heads"],
                               int(cu_k[-1]))
    np.testing.assert_array_equal(out, np.array(ex["out"], dtype=np.float64))


def test_unpad_invariants_random():
    rng = np.random.default_rng(7)
    mask = rng.random((9, 33)) < 0.4
    mask[3] = False
    cu, idx, mx = layout.mask_to_seqlens(mask)
    assert cu[0] == 0 and cu[-1] == mask.sum()
    assert np.all(np.diff(cu) == mask.sum(axis=1))
    assert np.all(np.diff(idx) > 0)                       # row-major order
    assert np.all(mask.reshape(-1)[idx])                  # only valid positions
    assert mx == mask.sum(axis=1).max()
    x = rng.standard_normal((9 * 33, 5))
    packed = layout.gather_rows(x, idx)
    back = layout.scatter_rows(packed, idx, 9 * 33)
    np.testing.assert_array_equal(back, x * mask.reshape(-1, 1))   # pad(unpad(x)) = x * mask
    np.testing.assert_array_equal(layout.gather_rows(back, idx), packed)  # unpad(pad(p)) = p


def test_fold_matches_attention_with_single_query_row():
    """With Lq_i = 1 and causal off, the per-pair grid's row 0 seen by the
    attention oracle equals the folded per-key bias seen by the same oracle."""
    rng = np.random.default_rng(3)
    lk = [5, 1, 9, 4]
    w = workloads.make_custom([1] * 4, lk, n_heads=4, n_kv_heads=2, head_dim=8, causal=False,
                              seed=11, bias_pair=(4, 4, 3, 9), bias_key=True)
    grid = w.bias_pair.double().numpy()
    folded = layout.fold_pair_row(grid, w.bias_strides, 0, w.cu_k, 4, w.total_k,
                                  bias_key=w.bias_key.double().numpy())
    o1, l1 = oracle.fwd(w.q, w.k, w.v, w.cu_q, w.cu_k, 4, 2, w.softmax_scale, False,
                        bias_key=w.bias_key.double().numpy(), bias_pair=grid,
                        bias_strides=w.bias_strides)
    o2, l2 = oracle.fwd(w.q, w.k, w.v, w.cu_q, w.cu_k, 4, 2, w.softmax_scale, False,
                        bias_key=folded)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-12)


def test_kv_head_grid_expansion():
    g = np.arange(2 * 3 * 2 * 2, dtype=np.float64).reshape(2, 3, 2, 2)
    e = layout.expand_kv_head_grid(g, 4)
    assert e.shape == (2, 12, 2, 2)
    for h in range(12):
        np.testing.assert_array_equal(e[:, h], g[:, h // 4])
    np.testing.assert_array_equal(layout.expand_kv_head_grid(g, 1), g)
