"""Pins for the CPU oracle: checks against things other than the oracle itself.

Each test fixes the oracle to something the pages or the mathematics
determine independently: hand-derived closed forms (tests/golden), the
pages' printed pair counts, brute-force padded attention with an explicit
mask, PyTorch's SDPA math path, and invariants (row isolation, GQA as
repeated heads, bias shift, q_len = 1 causal = non-causal).
"""
import json
import math
import os

import numpy as np
import pytest
from hypothesis import HealthCheck, given, settings, strategies as st
import torch

import oracle
from packed_variable_length_attn_b200 import metrics, workloads
from tests.bruteforce import padded_attention

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _run_oracle(w, **kw):
    return oracle.fwd(w.q, w.k, w.v, w.cu_q, w.cu_k, w.n_heads, w.n_kv_heads, w.softmax_scale,
                      w.causal, bias_key=w.bias_key, bias_pair=w.bias_pair,
                      bias_strides=w.bias_strides, **kw)


def _assert_close_inf(a, b, atol):
    a, b = np.asarray(a, dtype=np.float64), np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape
    inf_a, inf_b = np.isinf(a), np.isinf(b)
    assert np.array_equal(inf_a, inf_b)
    assert np.array_equal(a[inf_a], b[inf_b])
    np.testing.assert_allclose(a[~inf_a], b[~inf_b], rtol=0, atol=atol)


# --------------------------------------------------------------------------- golden

def _golden_examples():
    with open(os.path.join(GOLDEN, "closed_form_examples.json")) as f:
        return json.load(f)["examples"]


@pytest.mark.parametrize("ex", _golden_examples(), ids=lambda e: e["name"])
def test_hand_derived_examples(ex):
    q = np.array(ex["q"], dtype=np.float64)
    k = np.array(ex["k"], dtype=np.float64)
    v = np.array(ex["v"], dtype=np.float64)
    cu_q = np.concatenate([[0], np.cumsum(ex["lengths_q"])]).astype(np.int32)
    cu_k = np.concatenate([[0], np.cumsum(ex["lengths_k"])]).astype(np.int32)
    bk = np.array(ex["bias_key"], dtype=np.float64) if "bias_key" in ex else None
    bp = np.array(ex["bias_pair"], dtype=np.float64) if "bias_pair" in ex else None
    out, lse = oracle.fwd(q, k, v, cu_q, cu_k, ex["n_heads"], ex["n_kv_heads"], ex["scale"],
                          ex["causal"], bias_key=bk, bias_pair=bp,
                          bias_strides=ex.get("bias_strides"))
    want_lse = np.array([[float(x) for x in row] for row in ex["lse"]])
    np.testing.assert_allclose(out, np.array(ex["out"]), rtol=0, atol=1e-13)
    _assert_close_inf(lse, want_lse, 1e-13)


def test_page_pair_counts_dense_vs_padded():
    """8 rows of 128: a dense mask over the packed stream visits 1,048,576
    pairs, the padded batch 131,072 (printed on the GenRec packing page).
    Count the pairs the oracle gives non-zero probability, and the counter."""
    with open(os.path.join(GOLDEN, "page_pair_counts.json")) as f:
        g = json.load(f)
    rows, L = g["rows"], g["row_length"]
    # one 1024-token sequence with no mask = the dense (1,1,T,T) layout
    dense = workloads.make_custom([rows * L], n_heads=1, head_dim=4, causal=False, seed=1,
                                  dtype=torch.float32)
    p = oracle.probs(dense.q, dense.k, dense.v, dense.cu_q, dense.cu_k, 1, 1,
                     dense.softmax_scale, False, 0, 0)
    assert int((p > 0).sum()) == g["dense_mask_over_packed_stream_pairs"]
    padded = workloads.make_custom([L] * rows, n_heads=1, head_dim=4, causal=False, seed=2,
                                   dtype=torch.float32)
    n = 0
    for i in range(rows):
        p = oracle.probs(padded.q, padded.k, padded.v, padded.cu_q, padded.cu_k, 1, 1,
                         padded.softmax_scale, False, i, 0)
        n += int((p > 0).sum())
    assert n == g["padded_batch_pairs"]
    assert metrics.useful_pairs([rows * L], [rows * L], False) == g["dense_mask_over_packed_stream_pairs"]
    assert metrics.useful_pairs([L] * rows, [L] * rows, False) == g["padded_batch_pairs"]


def test_useful_pairs_counter():
    # tiny packed causal workload: sum L(L+1)/2 over {5,17,32,64}
    assert metrics.useful_pairs([5, 17, 32, 64], [5, 17, 32, 64], True) == 2776
    assert metrics.useful_flops([5, 17, 32, 64], [5, 17, 32, 64], True, 2, 64) == 1421312
    # short-query GQA: 112 queries x 262 keys, bottom-right: row r sees r + 151 keys
    assert metrics.causal_pairs(112, 262) == sum(r + 151 for r in range(112)) == 23128
    for lq in range(0, 12):
        for lk in range(0, 12):
            brute = sum(1 for r in range(lq) for c in range(lk) if c <= r + lk - lq)
            assert metrics.causal_pairs(lq, lk) == brute


# --------------------------------------------------------------------------- brute force

CASES = [
    dict(lq=[5, 17, 32], lk=None, Hq=2, Hkv=2, D=16, causal=True),
    dict(lq=[17, 5, 31], lk=None, Hq=4, Hkv=2, D=8, causal=False),
    dict(lq=[3, 0, 9, 1], lk=[7, 4, 2, 1], Hq=6, Hkv=2, D=8, causal=True),   # Lq != Lk, empty seq
    dict(lq=[4, 6], lk=[9, 3], Hq=3, Hkv=1, D=4, causal=False),
    dict(lq=[1, 1, 1], lk=[5, 1, 8], Hq=2, Hkv=1, D=8, causal=True),         # decode rows
]


@pytest.mark.parametrize("case", CASES)
@pytest.mark.parametrize("bias", ["none", "key", "pair", "both"])
def test_oracle_matches_bruteforce(case, bias):
    lk = case["lk"] or case["lq"]
    B = len(case["lq"])
    mq, mk = max(case["lq"]), max(lk)
    w = workloads.make_custom(case["lq"], lk, n_heads=case["Hq"], n_kv_heads=case["Hkv"],
                              head_dim=case["D"], causal=case["causal"], seed=7,
                              bias_key=bias in ("key", "both"),
                              bias_pair=(B, case["Hq"], mq + 1, mk + 2) if bias in ("pair", "both") else None)
    out, lse = _run_oracle(w)
    bo, bl = padded_attention(w.q, w.k, w.v, w.cu_q, w.cu_k, w.n_heads, w.n_kv_heads,
                              w.softmax_scale, w.causal, w.bias_key, w.bias_pair, w.bias_strides)
    np.testing.assert_allclose(out, bo, rtol=0, atol=1e-12)
    _assert_close_inf(lse, bl, 1e-12)


def test_oracle_matches_sdpa_math():
    """PyTorch SDPA (CPU math path, fp64, float mask) per sequence, the
    comparison the short-GQA and GiGL pages use."""
    w = workloads.make_custom([9, 14, 3], [12, 14, 7], n_heads=4, n_kv_heads=2, head_dim=16,
                              causal=True, seed=11, bias_key=True)
    out, lse = _run_oracle(w)
    G = w.n_heads // w.n_kv_heads
    for i in range(w.batch):
        q = w.q[w.cu_q[i]:w.cu_q[i + 1]].double().transpose(0, 1)
        k = w.k[w.cu_k[i]:w.cu_k[i + 1]].double().transpose(0, 1).repeat_interleave(G, 0)
        v = w.v[w.cu_k[i]:w.cu_k[i + 1]].double().transpose(0, 1).repeat_interleave(G, 0)
        lq, lk = q.shape[1], k.shape[1]
        r = torch.arange(lq)[:, None]
        c = torch.arange(lk)[None, :]
        vis = c <= r + (lk - lq)
        mask = torch.where(vis, 0.0, float("-inf")).double()
        mask = mask[None] + w.bias_key[w.cu_k[i]:w.cu_k[i + 1]].double().T[:, None, :]
        ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=mask,
                                                               scale=w.softmax_scale)
        got = torch.from_numpy(out[w.cu_q[i]:w.cu_q[i + 1]]).transpose(0, 1)
        rows_ok = vis.any(dim=1)
        torch.testing.assert_close(got[:, rows_ok], ref[:, rows_ok], rtol=0, atol=1e-12)


# --------------------------------------------------------------------------- closed forms

def test_zero_queries_give_uniform_weights():
    """q = 0 and no bias: every visible key has weight 1/n, so LSE = ln n and
    O is the mean of the visible V rows (a prefix mean under the causal mask)."""
    w = workloads.make_custom([6, 11], [9, 11], n_heads=2, n_kv_heads=1, head_dim=8,
                              causal=True, seed=3, dtype=torch.float32)
    w.q.zero_()
    out, lse = _run_oracle(w)
    for i in range(w.batch):
        lq, lk = w.lengths_q[i], w.lengths_k[i]
        for h in range(2):
            for r in range(lq):
                n = min(max(r + lk - lq + 1, 0), lk)
                row = w.cu_q[i] + r
                vv = w.v[w.cu_k[i]:w.cu_k[i] + n, 0].double().numpy()
                if n == 0:
                    assert lse[h, row] == -math.inf and not out[row, h].any()
                else:
                    assert abs(lse[h, row] - math.log(n)) < 1e-13
                    np.testing.assert_allclose(out[row, h], vv.mean(axis=0), atol=1e-13)


def test_constant_values_and_single_key():
    w = workloads.make_custom([5, 1], [7, 1], n_heads=2, n_kv_heads=2, head_dim=4,
                              causal=False, seed=4, dtype=torch.float32)
    w.v[:] = torch.tensor([0.25, -1.5, 3.0, 7.0])
    out, lse = _run_oracle(w)
    np.testing.assert_allclose(out, np.broadcast_to([0.25, -1.5, 3.0, 7.0], out.shape), atol=1e-13)
    # the second sequence has one key: O = v, LSE = its score
    q = w.q[5].double()
    k = w.k[7].double()
    for h in range(2):
        s = w.softmax_scale * float((q[h] * k[h]).sum())
        assert abs(lse[h, 5] - s) < 1e-12


def test_probabilities_rows_sum_to_one():
    w = workloads.make_custom([13, 4], [20, 9], n_heads=2, n_kv_heads=1, head_dim=8,
                              causal=True, seed=5, bias_key=True)
    out, _ = _run_oracle(w)
    for i in range(w.batch):
        for h in range(2):
            p = oracle.probs(w.q, w.k, w.v, w.cu_q, w.cu_k, 2, 1, w.softmax_scale, True, i, h,
                             bias_key=w.bias_key)
            lq, lk = p.shape
            vis = np.arange(lk)[None, :] <= np.arange(lq)[:, None] + lk - lq
            assert not p[~vis].any()
            np.testing.assert_allclose(p.sum(axis=1), 1.0, atol=1e-14)
            # O = P V on the sequence's own rows
            vv = w.v[w.cu_k[i]:w.cu_k[i + 1], 0].double().numpy()
            np.testing.assert_allclose(out[w.cu_q[i]:w.cu_q[i + 1], h], p @ vv, atol=1e-13)


# --------------------------------------------------------------------------- invariants

def test_bias_shift_invariance():
    w = workloads.make_custom([7, 12], None, n_heads=2, n_kv_heads=2, head_dim=8, causal=True,
                              seed=6, bias_key=True)
    w.bias_key = w.bias_key.double()  # shift in fp64 so the shift itself does not round
    out0, lse0 = _run_oracle(w)
    w.bias_key = w.bias_key + 2.5
    out1, lse1 = _run_oracle(w)
    np.testing.assert_allclose(out1, out0, atol=1e-13)
    np.testing.assert_allclose(lse1, lse0 + 2.5, atol=1e-12)


def test_decode_row_causal_equals_noncausal():
    """q_len = 1 under the bottom-right mask sees every key."""
    w = workloads.make_custom([1, 1, 1], [9, 1, 30], n_heads=4, n_kv_heads=2, head_dim=16,
                              causal=True, seed=8)
    oc, lc = _run_oracle(w)
    w.causal = False
    on, ln_ = _run_oracle(w)
    np.testing.assert_array_equal(oc, on)
    np.testing.assert_array_equal(lc, ln_)


def test_gqa_equals_repeated_heads():
    w = workloads.make_custom([10, 6], [10, 15], n_heads=6, n_kv_heads=2, head_dim=8,
                              causal=True, seed=9)
    out, lse = _run_oracle(w)
    k_rep = w.k.repeat_interleave(3, dim=1)
    v_rep = w.v.repeat_interleave(3, dim=1)
    o2, l2 = oracle.fwd(w.q, k_rep, v_rep, w.cu_q, w.cu_k, 6, 6, w.softmax_scale, True)
    np.testing.assert_array_equal(out, o2)
    np.testing.assert_array_equal(lse, l2)


def test_pair_grid_with_zero_row_stride_equals_per_key_bias():
    w = workloads.make_custom([8, 5], [8, 11], n_heads=2, n_kv_heads=2, head_dim=8,
                              causal=False, seed=10, bias_key=True)
    ok, lk_ = _run_oracle(w)
    # per-key bias as a grid: seq i, head h, row r, col c -> bias_key[cu_k[i]+c, h]
    # stored [Tk, H] so sb = cu_k-based offsets are impossible; build [B, H, 1, maxLk]
    B, H, mk = w.batch, 2, max(w.lengths_k)
    grid = torch.zeros(B, H, 1, mk, dtype=torch.float32)
    for i in range(B):
        grid[i, :, 0, :w.lengths_k[i]] = w.bias_key[w.cu_k[i]:w.cu_k[i + 1]].T
    op, lp = oracle.fwd(w.q, w.k, w.v, w.cu_q, w.cu_k, 2, 2, w.softmax_scale, False,
                        bias_pair=grid, bias_strides=(H * mk, mk, 0, 1))
    np.testing.assert_allclose(op, ok, atol=1e-13)
    np.testing.assert_allclose(lp, lk_, atol=1e-13)


def test_head_broadcast_and_permuted_grid_views():
    w = workloads.make_custom([6, 9], [7, 9], n_heads=3, n_kv_heads=3, head_dim=8,
                              causal=True, seed=12, bias_pair=(2, 1, 10, 12))
    o1, l1 = _run_oracle(w)  # sh = 0 broadcast
    # materialised per head
    full = w.bias_pair.expand(2, 3, 10, 12).contiguous()
    o2, l2 = oracle.fwd(w.q, w.k, w.v, w.cu_q, w.cu_k, 3, 3, w.softmax_scale, True,
                        bias_pair=full, bias_strides=(3 * 120, 120, 12, 1))
    np.testing.assert_allclose(o2, o1, atol=1e-13)
    np.testing.assert_allclose(l2, l1, atol=1e-13)
    # a permuted (column-major) view: store the transpose, read with swapped strides
    tr = full.transpose(2, 3).contiguous()          # [2, 3, 12, 10]
    o3, l3 = oracle.fwd(w.q, w.k, w.v, w.cu_q, w.cu_k, 3, 3, w.softmax_scale, True,
                        bias_pair=tr, bias_strides=(3 * 120, 120, 1, 10))
    np.testing.assert_allclose(o3, o1, atol=1e-13)
    np.testing.assert_allclose(l3, l1, atol=1e-13)


def test_row_isolation_bit_identical():
    """Rewrite sequence 0's inputs: sequence 1's outputs stay bit-identical."""
    w = workloads.make_custom([9, 14, 5], [11, 14, 8], n_heads=4, n_kv_heads=2, head_dim=16,
                              causal=True, seed=13, bias_key=True)
    o1, l1 = _run_oracle(w)
    g = torch.Generator().manual_seed(99)
    w.q[:9] = torch.randn(9, 4, 16, generator=g).to(w.q.dtype)
    w.k[:11] = torch.randn(11, 2, 16, generator=g).to(w.k.dtype)
    w.v[:11] = torch.randn(11, 2, 16, generator=g).to(w.v.dtype)
    w.bias_key[:11] = torch.randn(11, 4, generator=g)
    o2, l2 = _run_oracle(w)
    np.testing.assert_array_equal(o2[9:], o1[9:])
    np.testing.assert_array_equal(l2[:, 9:], l1[:, 9:])
    assert not np.array_equal(o2[:9], o1[:9])


def test_oracle_rows_equals_full_and_threads_do_not_matter():
    w = workloads.make(1)
    o1, l1 = _run_oracle(w, threads=1)
    o4, l4 = _run_oracle(w, threads=4)
    np.testing.assert_array_equal(o1, o4)
    np.testing.assert_array_equal(l1, l4)
    seq = [0, 1, 3, 3]
    head = [1, 0, 1, 0]
    row = [4, 16, 0, 63]
    orow, lrow = oracle.rows(w.q, w.k, w.v, w.cu_q, w.cu_k, 2, 2, w.softmax_scale, True,
                             seq, head, row)
    for n in range(4):
        t = int(w.cu_q[seq[n]]) + row[n]
        np.testing.assert_array_equal(orow[n], o1[t, head[n]])
        assert lrow[n] == l1[head[n], t]


def test_oracle_rejects_malformed_arguments():
    w = workloads.make(1)
    with pytest.raises(ValueError):
        oracle.fwd(w.q, w.k, w.v, w.cu_q, w.cu_k, 3, 2, w.softmax_scale, True)  # 3 % 2 != 0
    bad = w.cu_q.clone()
    bad[2] = 1  # decreasing boundaries
    with pytest.raises(ValueError):
        oracle.fwd(w.q, w.k, w.v, bad, w.cu_k, 2, 2, w.softmax_scale, True)


# --------------------------------------------------------------------------- randomized brute force


@settings(max_examples=40, deadline=None, suppress_health_check=[HealthCheck.too_slow])
@given(data=st.data())
def test_oracle_matches_bruteforce_random_shapes(data):
    """Random packs (empty members, Lq != Lk, GQA groups, both biases) against
    the padded brute force: any index or mask slip in either shows here."""
    B = data.draw(st.integers(1, 4))
    lq = data.draw(st.lists(st.integers(0, 12), min_size=B, max_size=B))
    lk = data.draw(st.lists(st.integers(0, 12), min_size=B, max_size=B))
    hkv = data.draw(st.sampled_from([1, 2]))
    g = data.draw(st.sampled_from([1, 2, 3]))
    D = data.draw(st.sampled_from([4, 8]))
    causal = data.draw(st.booleans())
    bias = data.draw(st.sampled_from(["none", "key", "pair", "both"]))
    seed = data.draw(st.integers(0, 10_000))
    if sum(lq) == 0:
        lq[0] = 1
    mq, mk = max(max(lq), 1), max(max(lk), 1)
    w = workloads.make_custom(lq, lk, n_heads=hkv * g, n_kv_heads=hkv, head_dim=D,
                              causal=causal, seed=seed, bias_key=bias in ("key", "both"),
                              bias_pair=(B, hkv * g, mq, mk) if bias in ("pair", "both") else None)
    out, lse = _run_oracle(w)
    bo, bl = padded_attention(w.q, w.k, w.v, w.cu_q, w.cu_k, w.n_heads, w.n_kv_heads,
                              w.softmax_scale, w.causal, w.bias_key, w.bias_pair, w.bias_strides)
    np.testing.assert_allclose(out, bo, rtol=0, atol=1e-12)
    _assert_close_inf(lse, bl, 1e-12)
