"""The seeded workload generator: shapes and length mixes of the five named
workloads, and determinism across calls."""
import torch

from packed_variable_length_attn_b200 import metrics, workloads


def test_tiny_workload_shape():
    w = workloads.make(1)
    assert w.lengths_q == [5, 17, 32, 64] and w.total_q == 118
    assert w.q.shape == (118, 2, 64) and w.q.dtype == torch.bfloat16
    assert w.causal and abs(w.softmax_scale - 0.125) < 1e-12
    assert metrics.useful_flops(w.lengths_q, w.lengths_k, True, 2, 64) == 1421312


def test_named_workload_shapes_and_ranges():
    w = workloads.make(2)
    assert w.batch == 20 and all(128 <= L <= 2048 for L in w.lengths_q)
    assert (w.n_heads, w.n_kv_heads, w.head_dim) == (14, 2, 64)
    w = workloads.make(3)
    assert w.batch == 512 and all(1 <= L <= 256 for L in w.lengths_q) and not w.causal
    assert tuple(w.bias_pair.shape) == (512, 1, 256, 256)
    assert w.bias_strides == (65536, 0, 256, 1)
    assert tuple(w.bias_key.shape) == (w.total_k, 8)
    assert 0.45 < float(w.bias_key.std()) < 0.55
    w = workloads.make(4)
    assert w.lengths_q == [112] * 64 and w.lengths_k == [262] * 64
    assert (w.n_heads, w.n_kv_heads, w.head_dim) == (32, 8, 128)
    assert metrics.useful_pairs(w.lengths_q, w.lengths_k, True) == 64 * 23128


def test_long_workload_lengths_only():
    g = torch.Generator("cpu").manual_seed(workloads.SEED_BASE + 5)
    lengths = torch.randint(2048, 8192 + 1, (16,), generator=g).tolist()
    assert all(2048 <= L <= 8192 for L in lengths)


def test_determinism():
    a = workloads.make(2)
    b = workloads.make(2)
    assert a.lengths_q == b.lengths_q
    assert torch.equal(a.q.view(torch.int16), b.q.view(torch.int16))


def test_algorithmic_bytes_closed_forms():
    """Bytes one forward must move, checked against closed forms."""
    from packed_variable_length_attn_b200 import metrics, workloads
    w4 = workloads.make(4)  # 64 rows of 112 queries, 262 keys, 32/8 heads, D 128
    want = 64 * 112 * 32 * 128 * 2 * 2 + 2 * 64 * 262 * 8 * 128 * 2 + 64 * 112 * 32 * 4
    assert metrics.algorithmic_bytes(w4) == want
    w3 = workloads.make(3)  # one-head pair grid (heads broadcast) + per-key bias
    base = (w3.total_q * 8 * 64 * 2 * 2 + 2 * w3.total_k * 8 * 64 * 2 + w3.total_q * 8 * 4
            + w3.total_k * 8 * 4)
    grid = 4 * sum(L * L for L in w3.lengths_q)
    assert metrics.algorithmic_bytes(w3) == base + grid
