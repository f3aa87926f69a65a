"""GPU parity of the backward pass (varlen_attn_bwd, through the C ABI)
against the backward oracle (oracle/backward.py, pinned by finite
differences of the forward oracle).

Tolerance: relative L2 error <= 1e-2 for every gradient (the ASpec PR 25
page, "Verification", bounds bf16 Q/K/V gradients at 1% relative L2 against
a dense math backend), and max-abs error <= 2e-2 of the reference's largest
magnitude. The GPU path rounds P and dS to bf16 for the tensor-core products
and takes delta = rowsum(dO * O) from the forward's bf16 output; the oracle
keeps fp64 throughout.
"""
import numpy as np
import pytest
import torch

from oracle.backward import bwd as oracle_bwd
import packed_variable_length_attn_b200 as va
from packed_variable_length_attn_b200 import workloads
from tests.parity import to_device

pytestmark = pytest.mark.gpu

REL_L2 = 1e-2
MAX_ABS_FRAC = 2e-2


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    va.get_device_error()
    yield
    assert va.get_device_error() == 0


def _close(name, got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, name
    assert np.isfinite(got).all(), name
    den = np.linalg.norm(ref)
    err = np.linalg.norm(got - ref)
    rel = err / den if den > 0 else err
    mx = np.abs(got - ref).max() if got.size else 0.0
    scale = np.abs(ref).max() if ref.size else 0.0
    assert rel <= REL_L2, (name, rel)
    assert mx <= MAX_ABS_FRAC * max(scale, 1e-6), (name, mx, scale)


def _run(lq, lk, Hq, Hkv, D, causal, seed, bias=False, kv_head_grid=False):
    Hg = Hkv if kv_head_grid else Hq
    w = workloads.make_custom(lq, lk, n_heads=Hq, n_kv_heads=Hkv, head_dim=D, causal=causal,
                              seed=seed, bias_key=bias,
                              bias_pair=(len(lq), Hg, max(max(lq), 1), max(max(lk), 1))
                              if bias else None)
    dev = to_device(w)
    strides = w.bias_strides if bias else None
    kw = dict(softmax_scale=w.softmax_scale, causal=causal, bias_per_key=dev["bias_key"],
              bias_pair=dev["bias_pair"], bias_pair_strides=strides,
              bias_pair_kv_heads=kv_head_grid)
    out, lse = va.varlen_attn_fwd(dev["q"], dev["k"], dev["v"], dev["cu_q"], dev["cu_k"],
                                  w.max_seqlen_q, w.max_seqlen_k, **kw)
    g = torch.Generator().manual_seed(seed + 1000)
    dout = torch.randn(w.q.shape, generator=g).to(torch.bfloat16)
    dq, dk, dv, dbk, dbp = va.varlen_attn_bwd(
        dev["q"], dev["k"], dev["v"], out, lse, dout.cuda(), dev["cu_q"], dev["cu_k"],
        w.max_seqlen_q, w.max_seqlen_k, need_dbias_per_key=bias, need_dbias_pair=bias, **kw)
    torch.cuda.synchronize()
    bias_pair = w.bias_pair
    bstr = w.bias_strides if bias else None
    if bias and kv_head_grid:
        from oracle import layout
        bias_pair = torch.from_numpy(layout.expand_kv_head_grid(w.bias_pair.numpy(), Hq // Hkv))
        B, H, R, C = bias_pair.shape
        bstr = (H * R * C, R * C, C, 1)
    ref = oracle_bwd(w.q, w.k, w.v, dout, w.cu_q, w.cu_k, Hq, Hkv, w.softmax_scale, causal,
                     bias_key=w.bias_key if bias else None,
                     bias_pair=bias_pair if bias else None, bias_strides=bstr)
    _close("dq", dq.float().cpu().numpy(), ref["dq"])
    _close("dk", dk.float().cpu().numpy(), ref["dk"])
    _close("dv", dv.float().cpu().numpy(), ref["dv"])
    if bias:
        _close("dbias_key", dbk.cpu().numpy(), ref["dbias_key"])
        _close("dbias_pair", dbp.cpu().numpy(), ref["dbias_pair"])
    return dq, dk, dv


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_backward_parity(D, causal):
    # ragged: several 128-blocks, tails, a one-token sequence, Lq != Lk
    _run([7, 130, 1, 257, 64], [9, 130, 40, 300, 64], 4, 2, D, causal, seed=31 + D + causal)


def test_backward_parity_gqa4_long_rows():
    _run([300, 129, 513], [300, 200, 513], 8, 2, 128, True, seed=77)


@pytest.mark.parametrize("causal", [False, True])
def test_backward_with_biases(causal):
    _run([33, 150, 1, 200], [40, 150, 17, 260], 4, 2, 64, causal, seed=91 + causal, bias=True)


def test_backward_broadcast_and_strided_grid():
    # one grid shared by all heads (head stride 0), read through a permuted
    # view (column stride != 1: the per-element load path)
    lq, lk = [60, 131], [70, 131]
    Hq, Hkv, D = 4, 2, 64
    w = workloads.make_custom(lq, lk, n_heads=Hq, n_kv_heads=Hkv, head_dim=D, causal=True,
                              seed=211)
    g = torch.Generator().manual_seed(212)
    base = torch.randn(len(lq), max(lk), max(lq), generator=g)   # [B, C, R]
    grid = base.permute(0, 2, 1)                                  # [B, R, C] view, sc = R
    strides = (grid.stride(0), 0, grid.stride(1), grid.stride(2))
    dev = to_device(w)
    kw = dict(softmax_scale=w.softmax_scale, causal=True, bias_pair=base.cuda().permute(0, 2, 1),
              bias_pair_strides=strides)
    out, lse = va.varlen_attn_fwd(dev["q"], dev["k"], dev["v"], dev["cu_q"], dev["cu_k"],
                                  w.max_seqlen_q, w.max_seqlen_k, **kw)
    dout = torch.randn(w.q.shape, generator=g).to(torch.bfloat16)
    dq, dk, dv, _, dbp = va.varlen_attn_bwd(dev["q"], dev["k"], dev["v"], out, lse, dout.cuda(),
                                            dev["cu_q"], dev["cu_k"], w.max_seqlen_q,
                                            w.max_seqlen_k, need_dbias_pair=True, **kw)
    torch.cuda.synchronize()
    flat = base.contiguous()  # the oracle reads the same entries through the same strides
    ref = oracle_bwd(w.q, w.k, w.v, dout, w.cu_q, w.cu_k, Hq, Hkv, w.softmax_scale, True,
                     bias_pair=flat, bias_strides=strides)
    _close("dq", dq.float().cpu().numpy(), ref["dq"])
    _close("dk", dk.float().cpu().numpy(), ref["dk"])
    _close("dv", dv.float().cpu().numpy(), ref["dv"])
    _close("dbias_pair", dbp.cpu().numpy(), ref["dbias_pair"])
    # the broadcast grid's own gradient is the sum over the heads
    _close("dbias_pair summed over heads", dbp.sum(dim=1).cpu().numpy(),
           ref["dbias_pair"].sum(axis=1))


def test_backward_kv_head_grid():
    _run([50, 140], [60, 140], 4, 2, 64, True, seed=123, bias=True, kv_head_grid=True)


def test_backward_empty_sequences():
    # Lq = 0 with keys (dK = dV = 0 there), Lk = 0 with queries (dQ = 0 there)
    _run([0, 5, 3, 130], [4, 0, 6, 130], 2, 1, 64, True, seed=5)


def test_backward_deterministic():
    a = _run([200, 77], [260, 77], 4, 2, 128, True, seed=17)
    b = _run([200, 77], [260, 77], 4, 2, 128, True, seed=17)
    for x, y in zip(a, b):
        assert torch.equal(x.view(torch.int16), y.view(torch.int16))


def test_backward_packed_equals_solo_bit_exact():
    # each sequence's gradients, run alone, equal its slice of the packed run
    # bit for bit (the other sequences contribute exact zeros)
    lq, lk = [150, 7, 260], [170, 40, 260]
    Hq, Hkv, D = 4, 2, 128
    w = workloads.make_custom(lq, lk, n_heads=Hq, n_kv_heads=Hkv, head_dim=D, causal=True,
                              seed=404)
    g = torch.Generator().manual_seed(405)
    dout = torch.randn(w.q.shape, generator=g).to(torch.bfloat16)
    dev = to_device(w)
    kw = dict(softmax_scale=w.softmax_scale, causal=True)
    out, lse = va.varlen_attn_fwd(dev["q"], dev["k"], dev["v"], dev["cu_q"], dev["cu_k"],
                                  w.max_seqlen_q, w.max_seqlen_k, **kw)
    dq, dk, dv, _, _ = va.varlen_attn_bwd(dev["q"], dev["k"], dev["v"], out, lse, dout.cuda(),
                                          dev["cu_q"], dev["cu_k"], w.max_seqlen_q,
                                          w.max_seqlen_k, **kw)
    cq, ck = w.cu_q.tolist(), w.cu_k.tolist()
    for i in range(len(lq)):
        qs, ks = slice(cq[i], cq[i + 1]), slice(ck[i], ck[i + 1])
        one = lambda n: torch.tensor([0, n], dtype=torch.int32, device="cuda")
        q1, k1, v1 = (dev["q"][qs].contiguous(), dev["k"][ks].contiguous(),
                      dev["v"][ks].contiguous())
        o1, l1 = va.varlen_attn_fwd(q1, k1, v1, one(lq[i]), one(lk[i]), lq[i], lk[i], **kw)
        d1 = va.varlen_attn_bwd(q1, k1, v1, o1, l1, dout[qs].contiguous().cuda(), one(lq[i]),
                                one(lk[i]), lq[i], lk[i], **kw)
        torch.cuda.synchronize()
        assert torch.equal(d1[0].view(torch.int16), dq[qs].view(torch.int16)), i
        assert torch.equal(d1[1].view(torch.int16), dk[ks].view(torch.int16)), i
        assert torch.equal(d1[2].view(torch.int16), dv[ks].view(torch.int16)), i
