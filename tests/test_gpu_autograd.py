"""The differentiable wrapper ``varlen_attn`` (torch.autograd through the C ABI).

Gradients that flow through ``loss.backward()`` must be the library's own
backward results bit for bit (the wrapper only marshals), and the pair-grid
gradient, reduced to the grid the caller passed (a broadcast grid sums the
heads that read it), must match the oracle's backward.
"""
import numpy as np
import pytest
import torch

import packed_variable_length_attn_b200 as va
from oracle.backward import bwd as oracle_bwd
from packed_variable_length_attn_b200 import workloads
from tests.parity import to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    va.get_device_error()
    yield
    assert va.get_device_error() == 0


def _bits(t):
    return t.contiguous().view(torch.int16 if t.dtype == torch.bfloat16 else torch.int32)


def _close(got, ref, rel_l2=1e-2, max_abs_frac=2e-2):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape
    err = np.linalg.norm(got - ref)
    den = np.linalg.norm(ref)
    assert (err / den if den > 0 else err) <= rel_l2
    assert np.abs(got - ref).max() <= max_abs_frac * max(np.abs(ref).max(), 1e-6)


@pytest.mark.parametrize("causal", [False, True])
def test_autograd_matches_direct_backward_bitwise(causal):
    w = workloads.make_custom([300, 1, 129, 77], n_heads=8, n_kv_heads=2, head_dim=128,
                              causal=causal, seed=61)
    dev = to_device(w)
    q = dev["q"].clone().requires_grad_()
    k = dev["k"].clone().requires_grad_()
    v = dev["v"].clone().requires_grad_()
    out, lse = va.varlen_attn(q, k, v, dev["cu_q"], dev["cu_k"], w.max_seqlen_q, w.max_seqlen_k,
                              softmax_scale=w.softmax_scale, causal=causal)
    dout = torch.randn(out.shape, generator=torch.Generator().manual_seed(62)).to(
        torch.bfloat16).cuda()
    (out.float() * dout.float()).sum().backward()
    o2, l2 = va.varlen_attn_fwd(dev["q"], dev["k"], dev["v"], dev["cu_q"], dev["cu_k"],
                                w.max_seqlen_q, w.max_seqlen_k, softmax_scale=w.softmax_scale,
                                causal=causal)
    dq, dk, dv, _, _ = va.varlen_attn_bwd(dev["q"], dev["k"], dev["v"], o2, l2, dout,
                                          dev["cu_q"], dev["cu_k"], w.max_seqlen_q,
                                          w.max_seqlen_k, softmax_scale=w.softmax_scale,
                                          causal=causal)
    torch.cuda.synchronize()
    assert torch.equal(_bits(out.detach()), _bits(o2))
    for got, ref in ((q.grad, dq), (k.grad, dk), (v.grad, dv)):
        assert torch.equal(_bits(got), _bits(ref))


@pytest.mark.parametrize("grid_heads", ["broadcast", "query_heads"])
def test_autograd_bias_gradients_match_oracle(grid_heads):
    lq = [40, 130, 7]
    Hq, Hkv = 4, 4
    Hg = 1 if grid_heads == "broadcast" else Hq
    w = workloads.make_custom(lq, n_heads=Hq, n_kv_heads=Hkv, head_dim=64, causal=False,
                              seed=63, bias_key=True, bias_pair=(len(lq), Hg, max(lq), max(lq)))
    dev = to_device(w)
    q = dev["q"].clone().requires_grad_()
    k = dev["k"].clone().requires_grad_()
    v = dev["v"].clone().requires_grad_()
    bk = dev["bias_key"].clone().requires_grad_()
    bp = dev["bias_pair"].clone().requires_grad_()
    out, _ = va.varlen_attn(q, k, v, dev["cu_q"], dev["cu_k"], w.max_seqlen_q, w.max_seqlen_k,
                            softmax_scale=w.softmax_scale, bias_per_key=bk, bias_pair=bp)
    dout = torch.randn(out.shape, generator=torch.Generator().manual_seed(64)).to(torch.bfloat16)
    (out.float() * dout.cuda().float()).sum().backward()
    torch.cuda.synchronize()
    ref = oracle_bwd(w.q, w.k, w.v, dout, w.cu_q, w.cu_k, Hq, Hkv, w.softmax_scale, False,
                     bias_key=w.bias_key, bias_pair=w.bias_pair, bias_strides=w.bias_strides)
    _close(q.grad.float().cpu().numpy(), ref["dq"])
    _close(bk.grad.cpu().numpy(), ref["dbias_key"])
    # the oracle's grid gradient is per query head; a broadcast grid sums them
    want = np.asarray(ref["dbias_pair"])
    if grid_heads == "broadcast":
        want = want.sum(axis=1, keepdims=True)
    got = bp.grad.cpu().numpy()
    assert got.shape == tuple(bp.shape)
    _close(got[:, :, :want.shape[2], :want.shape[3]], want)
