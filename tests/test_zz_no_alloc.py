"""The no-allocation entry point, varlen_attn_fwd_noalloc.

It serves callers whose device memory is managed elsewhere (a runtime that
reserves the device pool up front, a request loop that must not stall on
cudaMalloc/cudaFree, a plug-in with a fixed budget): the work list lives in a
fixed array inside the library instead of a cudaMalloc'd workspace. This
file is collected last so that a run stopping at the first failure has
already run every other test.
"""
import pytest
import torch

from packed_variable_length_attn_b200 import (VarlenAttnError, get_device_error,
                                              varlen_attn_fwd, varlen_attn_fwd_noalloc,
                                              workloads)
from tests.parity import compare, to_device

pytestmark = pytest.mark.gpu


def _both(w, dev):
    strides = w.bias_strides if w.bias_pair is not None else None
    kw = dict(softmax_scale=w.softmax_scale, causal=w.causal, bias_per_key=dev["bias_key"],
              bias_pair=dev["bias_pair"], bias_pair_strides=strides)
    ref_o, ref_l = varlen_attn_fwd(dev["q"], dev["k"], dev["v"], dev["cu_q"], dev["cu_k"],
                                   w.max_seqlen_q, w.max_seqlen_k, **kw)
    outs = []
    for _ in range(2):  # two calls in a row share (and overwrite) the fixed scratch
        out = torch.full_like(dev["q"], float("nan"))
        lse = torch.full((w.n_heads, w.total_q), float("nan"), device="cuda")
        varlen_attn_fwd_noalloc(dev["q"], dev["k"], dev["v"], dev["cu_q"], dev["cu_k"],
                                w.max_seqlen_q, w.max_seqlen_k, out, lse, **kw)
        outs.append((out, lse))
    torch.cuda.synchronize()
    return (ref_o, ref_l), outs


@pytest.mark.parametrize("config", [2, 3, 5])
def test_noalloc_matches_allocating_entry_point(config):
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required")
    w = workloads.make(config)
    dev = to_device(w)
    (ref_o, ref_l), outs = _both(w, dev)
    for out, lse in outs:
        compare(out, lse, ref_o.float().cpu().numpy(), ref_l.cpu().numpy())
    assert get_device_error() == 0


def test_noalloc_rejects_work_lists_beyond_its_scratch():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required")
    q = torch.zeros(16, 2, 64, dtype=torch.bfloat16, device="cuda")
    cu = torch.zeros(20001, dtype=torch.int32, device="cuda")
    cu[1:] = 16
    out = torch.empty_like(q)
    lse = torch.empty(2, 16, device="cuda")
    # 20000 sequences x up to one q-block each: 20000 pairs > 16384
    with pytest.raises(VarlenAttnError) as e:
        varlen_attn_fwd_noalloc(q, q, q, cu, cu, 16, 16, out, lse)
    assert e.value.status == 12
