"""Large sizes: one very long sequence in a pack, and a very long K/V cache.

The named workloads stop at 8,192 tokens per sequence. Here a 65,536-token
causal sequence (512 q-blocks, 512 K/V tiles per q-block at the end: offsets
and tile counts far beyond the benchmark's) sits between short ones, and a
decode step reads a 131,072-row cache. Outputs start as NaN, so a row that is
never written fails; the long sequence is compared with the oracle on a
stratified sample (first, last and two random rows of every q-block, one head
of every K/V group), the short ones in full through the same sample. The
backward over such a pack is checked bit for bit against the long sequence
run alone, and against the oracle on the short sequences.
"""
import numpy as np
import pytest
import torch

import oracle
import packed_variable_length_attn_b200 as va
from packed_variable_length_attn_b200 import workloads
from tests.parity import compare, compare_stratified, run_gpu, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    va.get_device_error()
    yield
    assert va.get_device_error() == 0


@pytest.mark.parametrize("d,causal", [(128, True), (64, False)])
def test_sixty_four_k_token_sequence(d, causal):
    lq = [5, 65536, 300, 1]
    w = workloads.make_custom(lq, None, n_heads=4, n_kv_heads=2, head_dim=d, causal=causal,
                              seed=65536 + d)
    dev = to_device(w)
    out = torch.full_like(dev["q"], float("nan"))
    lse = torch.full((w.n_heads, w.total_q), float("nan"), device="cuda")
    run_gpu(w, dev=dev, out=out, lse=lse)
    assert torch.isfinite(out).all()
    compare_stratified(w, out, lse, rows_per_block=4, seed=d)


def test_decode_over_a_131k_row_cache():
    B, Hq, Hkv, D, S = 2, 8, 2, 128, 131072
    lens = [131000, 5]
    g = torch.Generator().manual_seed(131072)
    q = torch.randn(B, Hq, D, generator=g).to(torch.bfloat16)
    kc = torch.randn(B, S, Hkv, D, generator=g).to(torch.bfloat16)
    vc = torch.randn(B, S, Hkv, D, generator=g).to(torch.bfloat16)
    cu = torch.arange(B + 1, dtype=torch.int32)
    cs = torch.tensor(lens, dtype=torch.int32)
    scale = 1.0 / np.sqrt(D)
    out, lse = va.varlen_attn_decode(q.cuda(), cu.cuda(), 1, kc.cuda(), vc.cuda(), cs.cuda(),
                                     softmax_scale=scale)
    torch.cuda.synchronize()
    k = torch.cat([kc[i, :lens[i]] for i in range(B)])
    v = torch.cat([vc[i, :lens[i]] for i in range(B)])
    cu_k = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32)
    ref_o, ref_l = oracle.fwd(q, k, v, cu, cu_k, Hq, Hkv, scale, True)
    compare(out, lse, ref_o, ref_l)


def test_backward_with_a_sixty_four_k_token_sequence():
    """Backward over a pack holding a 65,536-token causal sequence: its
    gradients equal (bit for bit) those of the sequence run alone, and the
    short sequences' gradients match the oracle's backward."""
    from oracle.backward import bwd as oracle_bwd
    lq = [300, 65536, 5]
    Hq, Hkv, D = 4, 2, 128
    w = workloads.make_custom(lq, None, n_heads=Hq, n_kv_heads=Hkv, head_dim=D, causal=True,
                              seed=6553)
    dev = to_device(w)
    g = torch.Generator().manual_seed(6554)
    dout = torch.randn(w.q.shape, generator=g).to(torch.bfloat16)

    def grads(q, k, v, do, cu_q, cu_k, mq, mk):
        o, l = va.varlen_attn_fwd(q, k, v, cu_q, cu_k, mq, mk, softmax_scale=w.softmax_scale,
                                  causal=True)
        dq, dk, dv, _, _ = va.varlen_attn_bwd(q, k, v, o, l, do, cu_q, cu_k, mq, mk,
                                              softmax_scale=w.softmax_scale, causal=True)
        torch.cuda.synchronize()
        return dq, dk, dv

    dq, dk, dv = grads(dev["q"], dev["k"], dev["v"], dout.cuda(), dev["cu_q"], dev["cu_k"],
                       w.max_seqlen_q, w.max_seqlen_k)
    for t in (dq, dk, dv):
        assert torch.isfinite(t.float()).all()
    # the long sequence alone
    a, b = int(w.cu_q[1]), int(w.cu_q[2])
    cu1 = torch.tensor([0, b - a], dtype=torch.int32, device="cuda")
    s_dq, s_dk, s_dv = grads(dev["q"][a:b].contiguous(), dev["k"][a:b].contiguous(),
                             dev["v"][a:b].contiguous(), dout[a:b].contiguous().cuda(), cu1, cu1,
                             b - a, b - a)
    for got, ref in ((dq[a:b], s_dq), (dk[a:b], s_dk), (dv[a:b], s_dv)):
        assert torch.equal(got.contiguous().view(torch.int16), ref.view(torch.int16))
    # the short sequences against the oracle (each on its own)
    for i in (0, 2):
        a, b = int(w.cu_q[i]), int(w.cu_q[i + 1])
        cu = torch.tensor([0, b - a], dtype=torch.int32)
        ref = oracle_bwd(w.q[a:b], w.k[a:b], w.v[a:b], dout[a:b], cu, cu, Hq, Hkv,
                         w.softmax_scale, True)
        for name, got in (("dq", dq), ("dk", dk), ("dv", dv)):
            x = got[a:b].float().cpu().numpy().astype(np.float64)
            r = np.asarray(ref[name], dtype=np.float64)
            err = np.linalg.norm(x - r) / max(np.linalg.norm(r), 1e-30)
            assert err <= 1e-2, (i, name, err)
            assert np.abs(x - r).max() <= 2e-2 * max(np.abs(r).max(), 1e-6), (i, name)
