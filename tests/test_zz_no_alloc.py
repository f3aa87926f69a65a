"""The no-allocation entry point, varlen_attn_fwd_noalloc.

It serves callers whose device memory is managed elsewhere (a runtime that
reserves the device pool up front, a request loop that must not stall on
cudaMalloc/cudaFree, a plug-in with a fixed budget): the work list lives in a
fixed array inside the library instead of a cudaMalloc'd workspace. It runs
the same kernels on the same work list as varlen_attn_fwd, so its outputs
must be bit-identical to that entry point's. This file is collected last so
that a run stopping at the first failure has already run every other test.
"""
import pytest
import torch

from packed_variable_length_attn_b200 import (VarlenAttnError, get_device_error,
                                              varlen_attn_fwd, varlen_attn_fwd_noalloc,
                                              workloads)
from tests.parity import to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    yield


def _bits(t):
    return t.contiguous().view(torch.int16 if t.dtype == torch.bfloat16 else torch.int32)


def _kw(w, dev):
    strides = w.bias_strides if w.bias_pair is not None else None
    return dict(softmax_scale=w.softmax_scale, causal=w.causal, bias_per_key=dev["bias_key"],
                bias_pair=dev["bias_pair"], bias_pair_strides=strides)


def _noalloc(w, dev, stream=None):
    out = torch.full_like(dev["q"], float("nan"))
    lse = torch.full((w.n_heads, w.total_q), float("nan"), device="cuda")
    varlen_attn_fwd_noalloc(dev["q"], dev["k"], dev["v"], dev["cu_q"], dev["cu_k"],
                            w.max_seqlen_q, w.max_seqlen_k, out, lse, stream=stream,
                            **_kw(w, dev))
    return out, lse


@pytest.mark.parametrize("config", [1, 2, 3, 4, 5])
def test_noalloc_bit_identical_to_allocating_entry_point(config):
    w = workloads.make(config)
    dev = to_device(w)
    ref_o, ref_l = varlen_attn_fwd(dev["q"], dev["k"], dev["v"], dev["cu_q"], dev["cu_k"],
                                   w.max_seqlen_q, w.max_seqlen_k, **_kw(w, dev))
    # two calls in a row share (and overwrite) the fixed scratch
    outs = [_noalloc(w, dev) for _ in range(2)]
    torch.cuda.synchronize()
    for out, lse in outs:
        assert torch.equal(_bits(out), _bits(ref_o))
        assert torch.equal(_bits(lse), _bits(ref_l))
    assert get_device_error() == 0


def test_noalloc_allocates_no_device_memory():
    """On a stream the library has never seen (where varlen_attn_fwd would
    create a workspace), the call leaves the device's free memory unchanged."""
    w = workloads.make(3)
    dev = to_device(w)
    out = torch.empty_like(dev["q"])
    lse = torch.empty((w.n_heads, w.total_q), device="cuda")
    s = torch.cuda.Stream()
    varlen_attn_fwd_noalloc(dev["q"], dev["k"], dev["v"], dev["cu_q"], dev["cu_k"],
                            w.max_seqlen_q, w.max_seqlen_k, out, lse, stream=s, **_kw(w, dev))
    torch.cuda.synchronize()  # kernels loaded, argument buffers settled
    s2 = torch.cuda.Stream()
    with torch.cuda.stream(s2):
        torch.cuda._sleep(10)  # the stream's first launch, outside the measured window
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        varlen_attn_fwd_noalloc(dev["q"], dev["k"], dev["v"], dev["cu_q"], dev["cu_k"],
                                w.max_seqlen_q, w.max_seqlen_k, out, lse, stream=s2,
                                **_kw(w, dev))
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0
    assert get_device_error() == 0


def test_noalloc_rejects_work_lists_beyond_its_scratch():
    q = torch.zeros(16, 2, 64, dtype=torch.bfloat16, device="cuda")
    cu = torch.zeros(20001, dtype=torch.int32, device="cuda")
    cu[1:] = 16
    out = torch.empty_like(q)
    lse = torch.empty(2, 16, device="cuda")
    # 20000 sequences x up to one q-block each: 20000 pairs > 16384
    with pytest.raises(VarlenAttnError) as e:
        varlen_attn_fwd_noalloc(q, q, q, cu, cu, 16, 16, out, lse)
    assert e.value.status == 12
