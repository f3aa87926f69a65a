"""CUDA-graph capture of the library's calls.

A serving loop that runs many small packs is bound by launch latency; capturing
a call once and replaying it removes the host side of every later step. These
tests capture each entry point on a side stream (after one warm-up call on that
stream, which sizes the library's workspace so that nothing is allocated while
capturing), replay it, and check that the replay is bit-identical to an eager
call: on the captured inputs, and again after new values are copied into the
same input buffers (a replay reads the buffers, not the values seen at capture).
"""
import pytest
import torch

import packed_variable_length_attn_b200 as va
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


def _capture(fn):
    """Warm up `fn` on a side stream, capture it there, return the graph."""
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        fn()
    torch.cuda.synchronize()
    return g


def _refill(tensors, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    for t in tensors:
        t.copy_(torch.randn(t.shape, generator=g, device="cuda").to(t.dtype))


@pytest.mark.parametrize("config,noalloc", [(2, False), (3, False), (4, False), (4, True),
                                            (1, True)])
def test_forward_replay_bit_identical(config, noalloc):
    w = workloads.make(config)
    dev = to_device(w)
    kw = dict(softmax_scale=w.softmax_scale, causal=w.causal, bias_per_key=dev["bias_key"],
              bias_pair=dev["bias_pair"],
              bias_pair_strides=w.bias_strides if w.bias_pair is not None else None)
    out = torch.empty_like(dev["q"])
    lse = torch.empty(w.n_heads, w.total_q, device="cuda")

    def call(o=out, l=lse):
        if noalloc:
            va.varlen_attn_fwd_noalloc(dev["q"], dev["k"], dev["v"], dev["cu_q"], dev["cu_k"],
                                       w.max_seqlen_q, w.max_seqlen_k, o, l, **kw)
        else:
            va.varlen_attn_fwd(dev["q"], dev["k"], dev["v"], dev["cu_q"], dev["cu_k"],
                               w.max_seqlen_q, w.max_seqlen_k, out=o, lse=l, **kw)

    g = _capture(call)
    for seed in (None, 11):
        if seed is not None:
            _refill([dev["q"], dev["k"], dev["v"]], seed)
        out.fill_(float("nan"))
        lse.fill_(float("nan"))
        g.replay()
        ref_o, ref_l = torch.empty_like(out), torch.empty_like(lse)
        call(ref_o, ref_l)  # eager, on the current stream
        torch.cuda.synchronize()
        assert torch.equal(_bits(out), _bits(ref_o))
        assert torch.equal(_bits(lse), _bits(ref_l))
    assert va.get_device_error() == 0


# tensor cores with key ranges (16 x 8 pairs, fewer than the SMs); tensor
# cores, one item per pair; the CUDA-core kernel (explicit key ranges)
@pytest.mark.parametrize("B,Hkv,splits", [(16, 8, 0), (40, 4, 0), (16, 8, 4)])
def test_decode_replay_bit_identical(B, Hkv, splits):
    Hq, D, S = 32, 128, 2048
    gen = torch.Generator().manual_seed(31)
    lens = torch.randint(1, S, (B,), generator=gen, dtype=torch.int32).cuda()
    q = torch.randn(B, Hq, D, generator=gen).to(torch.bfloat16).cuda()
    kc = torch.randn(B, S, Hkv, D, generator=gen).to(torch.bfloat16).cuda()
    vc = torch.randn(B, S, Hkv, D, generator=gen).to(torch.bfloat16).cuda()
    cu = torch.arange(B + 1, dtype=torch.int32).cuda()
    out = torch.empty_like(q)
    lse = torch.empty(Hq, B, device="cuda")

    def call(o=out, l=lse):
        va.varlen_attn_decode(q, cu, 1, kc, vc, lens, num_splits=splits, out=o, lse=l)

    g = _capture(call)
    for seed in (None, 12):
        if seed is not None:
            _refill([q, kc, vc], seed)
        out.fill_(float("nan"))
        g.replay()
        ref_o, ref_l = torch.empty_like(out), torch.empty_like(lse)
        call(ref_o, ref_l)
        torch.cuda.synchronize()
        assert torch.equal(_bits(out), _bits(ref_o))
        assert torch.equal(_bits(lse), _bits(ref_l))


def test_backward_replay_bit_identical():
    w = workloads.make_custom([300, 77, 129, 1, 512], n_heads=8, n_kv_heads=2, head_dim=128,
                              causal=True, seed=41)
    dev = to_device(w)
    o, l = va.varlen_attn_fwd(dev["q"], dev["k"], dev["v"], dev["cu_q"], dev["cu_k"],
                              w.max_seqlen_q, w.max_seqlen_k, softmax_scale=w.softmax_scale,
                              causal=True)
    dout = torch.randn(w.q.shape, generator=torch.Generator().manual_seed(42)).to(
        torch.bfloat16).cuda()
    dq, dk, dv = (torch.empty_like(dev["q"]), torch.empty_like(dev["k"]),
                  torch.empty_like(dev["v"]))

    def call(a=dq, b=dk, c=dv):
        va.varlen_attn_bwd(dev["q"], dev["k"], dev["v"], o, l, dout, dev["cu_q"], dev["cu_k"],
                           w.max_seqlen_q, w.max_seqlen_k, softmax_scale=w.softmax_scale,
                           causal=True, dq=a, dk=b, dv=c)

    g = _capture(call)
    for seed in (None, 13):
        if seed is not None:
            _refill([dout], seed)
        for t in (dq, dk, dv):
            t.fill_(float("nan"))
        g.replay()
        refs = [torch.empty_like(t) for t in (dq, dk, dv)]
        call(*refs)
        torch.cuda.synchronize()
        for got, ref in zip((dq, dk, dv), refs):
            assert torch.equal(_bits(got), _bits(ref))
