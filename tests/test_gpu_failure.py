"""Failure detection on the GPU without a GPU fault.

Every barrier wait of the tensor-core kernels is bounded. Here a wait is
made to run out on purpose: the test hook varlen_attn_set_test_stall makes
the MMA warp of every CTA first wait on a barrier phase that nothing
completes, with the bound shortened to about half a millisecond
(varlen_attn_set_wait_limit). The kernel must report
VARLEN_ATTN_ERR_DEVICE_TIMEOUT (10) in the device error word and return,
having waited (bounded) for its copies in flight and freed its tensor memory. The next call with the default bound on the same context
must then succeed and match the oracle, which shows that the context, the
tensor memory of every SM and the library's workspace are still usable.
Nothing here traps, faults or spins without a bound.
"""
import pytest
import torch

import packed_variable_length_attn_b200 as va
from packed_variable_length_attn_b200 import workloads
from tests.parity import compare, run_gpu, run_oracle, to_device

pytestmark = pytest.mark.gpu

TIMEOUT = 10
SHORT_LIMIT = 1 << 20  # cycles (about 0.5 ms)


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    assert va.get_device_error() == 0
    yield
    va.set_test_stall(False)
    va.set_wait_limit(0)
    assert va.get_device_error() == 0


def _with_stall(fn):
    va.set_wait_limit(SHORT_LIMIT)
    va.set_test_stall(True)
    try:
        fn()
        err = va.get_device_error()
    finally:
        va.set_test_stall(False)
        va.set_wait_limit(0)
    return err


@pytest.mark.parametrize("config", [1, 4])
def test_forward_wait_timeout_reported_then_next_call_correct(config):
    w = workloads.make(config)
    dev = to_device(w)
    assert _with_stall(lambda: run_gpu(w, dev=dev)) == TIMEOUT
    out, lse = run_gpu(w, dev=dev)
    assert va.get_device_error() == 0
    compare(out, lse, *run_oracle(w))


def test_backward_wait_timeout_reported_then_next_call_correct():
    w = workloads.make(1)
    dev = to_device(w)
    out, lse = run_gpu(w, dev=dev)
    g = torch.Generator().manual_seed(3)
    dout = torch.randn(w.q.shape, generator=g).to(torch.bfloat16).cuda()
    kw = dict(softmax_scale=w.softmax_scale, causal=w.causal)

    def bwd():
        r = va.varlen_attn_bwd(dev["q"], dev["k"], dev["v"], out, lse, dout, dev["cu_q"],
                               dev["cu_k"], w.max_seqlen_q, w.max_seqlen_k, **kw)
        torch.cuda.synchronize()
        return r

    ref = bwd()
    assert va.get_device_error() == 0
    assert _with_stall(bwd) == TIMEOUT
    again = bwd()
    assert va.get_device_error() == 0
    for a, b in zip(ref[:3], again[:3]):  # dQ, dK, dV are bitwise reproducible
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))
