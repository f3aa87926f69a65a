"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Full element-by-element comparisons on inputs the oracle finishes in
seconds (several 128-row tiles and ragged tails) and on the tiny, GenRec,
graph-batch and short-query workloads at their full sizes; a stratified
sample of the long causal GQA workload (every sequence and q-block, every
K/V group) at its full size in the launch configuration the benchmark times;
edge cases; and the bit-exact invariants (row isolation, packed-vs-solo,
sequence order, run-to-run determinism) on every named workload.
"""
import zlib

import numpy as np
import pytest
import torch

import oracle
from packed_variable_length_attn_b200 import (VarlenAttnError, get_device_error,
                                              varlen_attn_fwd, workloads)
from tests.parity import compare, compare_stratified, run_gpu, run_oracle, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    yield
    assert get_device_error() == 0


def test_tiny_packed_causal_full():
    w = workloads.make(1)
    out, lse = run_gpu(w)
    compare(out, lse, *run_oracle(w))


SMALL = [
    # lengths_q, lengths_k, Hq, Hkv, D, causal
    ([300, 129, 1, 0, 257], None, 2, 2, 64, True),
    ([300, 129, 1, 0, 257], None, 4, 2, 128, False),
    ([128, 256, 255, 17], None, 6, 2, 64, True),
    ([112, 112, 112], [262, 262, 262], 8, 2, 128, True),     # bottom-right, Lq < Lk
    ([200, 70, 5], [90, 20, 300], 4, 4, 64, True),          # Lq > Lk rows that see nothing
    ([1, 1, 1, 1], [513, 1, 128, 129], 7, 1, 64, True),      # decode rows, G = 7
    ([385, 3], [385, 700], 3, 1, 128, False),               # odd G
    ([640], None, 2, 1, 128, True),
    ([640, 300, 5, 129], None, 7, 1, 64, True),               # odd G: pairs across q-blocks
    ([200, 333, 1], [500, 333, 40], 5, 1, 128, True),        # odd G, Lq != Lk
]


@pytest.mark.parametrize("case", SMALL, ids=lambda c: f"{c[2]}x{c[3]}_D{c[4]}_{'c' if c[5] else 'nc'}_{len(c[0])}seq")
def test_small_full_parity(case):
    lq, lk, hq, hkv, d, causal = case
    w = workloads.make_custom(lq, lk, n_heads=hq, n_kv_heads=hkv, head_dim=d, causal=causal,
                              seed=zlib.crc32(str(case).encode()) % 1000)
    out, lse = run_gpu(w)
    compare(out, lse, *run_oracle(w))


@pytest.mark.parametrize("bias", ["key", "pair", "both"])
@pytest.mark.parametrize("d", [64, 128])
def test_bias_full_parity(bias, d):
    lq = [77, 256, 1, 130]
    lk = [77, 256, 1, 130]
    B = len(lq)
    w = workloads.make_custom(lq, lk, n_heads=4, n_kv_heads=2, head_dim=d, causal=False, seed=5,
                              bias_key=bias in ("key", "both"),
                              bias_pair=(B, 1, 256, 256) if bias in ("pair", "both") else None)
    out, lse = run_gpu(w)
    compare(out, lse, *run_oracle(w))


def test_pair_bias_per_head_and_permuted_view():
    """Per-head grid (sh != 0) and a permuted (column-major) view, the case
    the GiGL page tests; row length not a multiple of 8."""
    lq = [37, 150, 9]
    w = workloads.make_custom(lq, None, n_heads=3, n_kv_heads=3, head_dim=64, causal=True,
                              seed=21, bias_pair=(3, 3, 150, 150))
    out1, lse1 = run_gpu(w)
    compare(out1, lse1, *run_oracle(w))
    # same grid stored transposed, read through a permuted view
    grid_t = w.bias_pair.transpose(2, 3).contiguous()
    view = grid_t.transpose(2, 3)
    w2 = workloads.make_custom(lq, None, n_heads=3, n_kv_heads=3, head_dim=64, causal=True,
                               seed=21, bias_pair=(3, 3, 150, 150))
    w2.bias_pair = view
    w2.bias_strides = tuple(view.stride())
    dev = to_device(w2)
    dev["bias_pair"] = grid_t.cuda().transpose(2, 3)
    out2, lse2 = run_gpu(w2, dev=dev)
    compare(out2, lse2, *run_oracle(w))


@pytest.mark.parametrize("config", [2, 3, 4])
def test_named_workloads_full_parity(config):
    """Every output element of the GenRec, graph-batch and short-query
    workloads at their full sizes, in the benchmark's launch configuration."""
    w = workloads.make(config)
    out, lse = run_gpu(w)
    res = compare(out, lse, *run_oracle(w))
    print(config, res)


def test_long_workload_stratified_parity():
    """The long causal GQA workload (the benchmark's) at full size: every
    (sequence, 128-row q-block) is checked on its first and last row and two
    random rows, each on one head drawn from every K/V group."""
    w = workloads.make(5)
    out, lse = run_gpu(w)
    res = compare_stratified(w, out, lse, rows_per_block=4, seed=5)
    print(res)


@pytest.mark.parametrize("batch,causal,hq,hkv", [(16385, True, 2, 1), (40000, False, 2, 2),
                                                  (40000, True, 4, 2)])
def test_packs_beyond_one_shared_memory_sort(batch, causal, hq, hkv):
    """More sequences than the schedule sorts in one shared-memory pass: its
    runs are merged in global memory. Every row must still be computed
    exactly once (outputs start as NaN)."""
    g = np.random.default_rng(batch + hq)
    lq = [int(x) for x in g.integers(0, 41, batch)]
    lq[batch // 2] = 300  # one longer sequence (several q-blocks)
    w = workloads.make_custom(lq, None, n_heads=hq, n_kv_heads=hkv, head_dim=64, causal=causal,
                              seed=batch)
    dev = to_device(w)
    out = torch.full_like(dev["q"], float("nan"))
    lse = torch.full((w.n_heads, w.total_q), float("nan"), device="cuda")
    run_gpu(w, dev=dev, out=out, lse=lse)
    compare(out, lse, *run_oracle(w))


def test_fp32_path_parity():
    w = workloads.make_custom([300, 1, 129, 64], [300, 7, 129, 200], n_heads=4, n_kv_heads=2,
                              head_dim=128, causal=True, seed=31, dtype=torch.float32,
                              bias_key=True, bias_pair=(4, 1, 300, 300))
    out, lse = run_gpu(w)
    assert out.dtype == torch.float32
    compare(out, lse, *run_oracle(w), fp32=True)
    w64 = workloads.make_custom([65, 200], None, n_heads=2, n_kv_heads=1, head_dim=64,
                                causal=False, seed=32, dtype=torch.float32)
    out, lse = run_gpu(w64)
    compare(out, lse, *run_oracle(w64), fp32=True)


# ------------------------------------------------------------------ invariants

def _bits(t):
    return t.contiguous().view(torch.int16 if t.dtype == torch.bfloat16 else torch.int32).cpu()


@pytest.mark.parametrize("config", [1, 2, 3, 4, 5])
def test_row_isolation_bit_exact(config):
    """Rewrite sequence 0's Q/K/V (and biases): every other sequence's output
    and LSE stay bit-identical."""
    w = workloads.make(config)
    dev = to_device(w)
    out1, lse1 = run_gpu(w, dev=dev)
    g = torch.Generator().manual_seed(1234)
    lq0, lk0 = w.lengths_q[0], w.lengths_k[0]
    dev["q"][:lq0] = torch.randn(lq0, w.n_heads, w.head_dim, generator=g).to(w.q.dtype).cuda()
    dev["k"][:lk0] = torch.randn(lk0, w.n_kv_heads, w.head_dim, generator=g).to(w.k.dtype).cuda()
    dev["v"][:lk0] = torch.randn(lk0, w.n_kv_heads, w.head_dim, generator=g).to(w.v.dtype).cuda()
    if dev["bias_key"] is not None:
        dev["bias_key"][:lk0] = torch.randn(lk0, w.n_heads, generator=g).cuda()
    if dev["bias_pair"] is not None:
        dev["bias_pair"][0] = torch.randn(dev["bias_pair"][0].shape, generator=g).cuda()
    out2, lse2 = run_gpu(w, dev=dev)
    assert torch.equal(_bits(out2[lq0:]), _bits(out1[lq0:]))
    assert torch.equal(_bits(lse2[:, lq0:]), _bits(lse1[:, lq0:]))
    assert not torch.equal(_bits(out2[:lq0]), _bits(out1[:lq0]))


@pytest.mark.parametrize("config", [1, 2, 3, 4, 5])
def test_packed_vs_solo_bit_exact(config):
    """Each sequence run alone (batch of one) gives bit-identical O and LSE
    to its slice of the packed run."""
    w = workloads.make(config)
    dev = to_device(w)
    out, lse = run_gpu(w, dev=dev)
    picks = sorted(set([0, w.batch - 1, w.batch // 2, int(np.argmax(w.lengths_q))]))
    for i in picks:
        qa, qb = int(w.cu_q[i]), int(w.cu_q[i + 1])
        ka, kb = int(w.cu_k[i]), int(w.cu_k[i + 1])
        cu1 = torch.tensor([0, qb - qa], dtype=torch.int32, device="cuda")
        ck1 = torch.tensor([0, kb - ka], dtype=torch.int32, device="cuda")
        bk = None if dev["bias_key"] is None else dev["bias_key"][ka:kb].contiguous()
        bp = None if dev["bias_pair"] is None else dev["bias_pair"][i:i + 1]
        o1, l1 = varlen_attn_fwd(dev["q"][qa:qb].contiguous(), dev["k"][ka:kb].contiguous(),
                                 dev["v"][ka:kb].contiguous(), cu1, ck1, qb - qa, kb - ka,
                                 softmax_scale=w.softmax_scale, causal=w.causal,
                                 bias_per_key=bk, bias_pair=bp,
                                 bias_pair_strides=w.bias_strides if bp is not None else None)
        torch.cuda.synchronize()
        assert torch.equal(_bits(o1), _bits(out[qa:qb])), i
        assert torch.equal(_bits(l1), _bits(lse[:, qa:qb])), i


@pytest.mark.parametrize("config", [2, 4, 5])
def test_sequence_order_permutation_bit_exact(config):
    """The pack in reverse order gives every sequence bit-identical O and LSE."""
    w = workloads.make(config)
    out, lse = run_gpu(w)
    perm = list(reversed(range(w.batch)))
    lq = [w.lengths_q[i] for i in perm]
    lk = [w.lengths_k[i] for i in perm]
    q = torch.cat([w.q[w.cu_q[i]:w.cu_q[i + 1]] for i in perm])
    k = torch.cat([w.k[w.cu_k[i]:w.cu_k[i + 1]] for i in perm])
    v = torch.cat([w.v[w.cu_k[i]:w.cu_k[i + 1]] for i in perm])
    w2 = workloads.make_custom(lq, lk, n_heads=w.n_heads, n_kv_heads=w.n_kv_heads,
                               head_dim=w.head_dim, causal=w.causal, seed=0)
    w2.q, w2.k, w2.v = q, k, v
    out2, lse2 = run_gpu(w2)
    for j, i in enumerate(perm):
        a, b = int(w.cu_q[i]), int(w.cu_q[i + 1])
        a2, b2 = int(w2.cu_q[j]), int(w2.cu_q[j + 1])
        assert torch.equal(_bits(out2[a2:b2]), _bits(out[a:b])), i
        assert torch.equal(_bits(lse2[:, a2:b2]), _bits(lse[:, a:b])), i


def test_run_to_run_deterministic():
    w = workloads.make(3)
    dev = to_device(w)
    o1, l1 = run_gpu(w, dev=dev)
    o2, l2 = run_gpu(w, dev=dev)
    assert torch.equal(_bits(o1), _bits(o2)) and torch.equal(_bits(l1), _bits(l2))


# ------------------------------------------------------------------ edges and guards

def test_canaries_untouched():
    """Outputs sit inside larger buffers filled with a NaN pattern: nothing
    outside [0, total_q) rows is written."""
    w = workloads.make_custom([130, 5, 256], [140, 5, 256], n_heads=4, n_kv_heads=2,
                              head_dim=128, causal=True, seed=41)
    dev = to_device(w)
    pad = 64
    nan_bits = torch.tensor(0x7FC1, dtype=torch.int16)
    ob = torch.full((w.total_q + 2 * pad, w.n_heads, w.head_dim), 0, dtype=torch.int16,
                    device="cuda")
    ob.fill_(int(nan_bits))
    out = ob[pad:pad + w.total_q].view(torch.bfloat16)
    lb = torch.full((w.n_heads * w.total_q + 2 * pad,), float("nan"), device="cuda")
    lse = lb[pad:pad + w.n_heads * w.total_q].view(w.n_heads, w.total_q)
    run_gpu(w, dev=dev, out=out, lse=lse)
    assert (ob[:pad] == int(nan_bits)).all() and (ob[-pad:] == int(nan_bits)).all()
    assert torch.isnan(lb[:pad]).all() and torch.isnan(lb[-pad:]).all()
    compare(out, lse, *run_oracle(w))


def test_trailing_rows_beyond_cu_untouched():
    """total_q larger than cu_q[B]: rows past the last sequence are not written."""
    w = workloads.make_custom([100, 30], None, n_heads=2, n_kv_heads=2, head_dim=64,
                              causal=True, seed=42)
    dev = to_device(w)
    extra = 50
    q = torch.cat([dev["q"], torch.zeros(extra, 2, 64, dtype=torch.bfloat16, device="cuda")])
    k = torch.cat([dev["k"], torch.zeros(extra, 2, 64, dtype=torch.bfloat16, device="cuda")])
    v = torch.cat([dev["v"], torch.zeros(extra, 2, 64, dtype=torch.bfloat16, device="cuda")])
    out = torch.full_like(q, 7.0)
    lse = torch.full((2, q.shape[0]), 7.0, device="cuda")
    varlen_attn_fwd(q, k, v, dev["cu_q"], dev["cu_k"], 100, 100, causal=True, out=out, lse=lse)
    torch.cuda.synchronize()
    assert (out[130:] == 7.0).all() and (lse[:, 130:] == 7.0).all()
    compare(out[:130], lse[:, :130], *run_oracle(w))


def test_all_sequences_without_keys():
    w = workloads.make_custom([3, 4], [0, 0], n_heads=2, n_kv_heads=1, head_dim=64,
                              causal=False, seed=43)
    dev = to_device(w)
    dev["k"] = torch.zeros(1, 1, 64, dtype=torch.bfloat16, device="cuda")
    dev["v"] = torch.zeros(1, 1, 64, dtype=torch.bfloat16, device="cuda")
    out, lse = varlen_attn_fwd(dev["q"], dev["k"], dev["v"], dev["cu_q"], dev["cu_k"], 4, 0)
    torch.cuda.synchronize()
    assert (out.float() == 0).all() and torch.isneginf(lse).all()


def test_invalid_cu_seqlens_reported_and_nothing_written():
    w = workloads.make(1)
    dev = to_device(w)
    bad = dev["cu_q"].clone()
    bad[2] = bad[1] - 1   # decreasing
    out = torch.full_like(dev["q"], 3.0)
    lse = torch.full((w.n_heads, w.total_q), 3.0, device="cuda")
    assert get_device_error() == 0
    varlen_attn_fwd(dev["q"], dev["k"], dev["v"], bad, dev["cu_k"], w.max_seqlen_q,
                    w.max_seqlen_k, causal=True, out=out, lse=lse)
    assert get_device_error() == 9
    assert (out == 3.0).all() and (lse == 3.0).all()
    # a length above max_seqlen is rejected the same way
    varlen_attn_fwd(dev["q"], dev["k"], dev["v"], dev["cu_q"], dev["cu_k"], 10, 10,
                    causal=True, out=out, lse=lse)
    assert get_device_error() == 9
    assert (out == 3.0).all()


def test_host_argument_errors():
    q3 = torch.zeros(10, 3, 64, dtype=torch.bfloat16, device="cuda")
    k2 = torch.zeros(10, 2, 64, dtype=torch.bfloat16, device="cuda")
    cu = torch.tensor([0, 10], dtype=torch.int32, device="cuda")
    with pytest.raises(VarlenAttnError) as e:
        varlen_attn_fwd(q3, k2, k2, cu, cu, 10, 10)
    assert e.value.status == 3
    q96 = torch.zeros(10, 2, 96, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(VarlenAttnError) as e:
        varlen_attn_fwd(q96, q96, q96, cu, cu, 10, 10)
    assert e.value.status == 4
