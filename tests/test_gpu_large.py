"""Large sizes: one very long sequence in a pack, and a very long K/V cache.

The named workloads stop at 8,192 tokens per sequence. Here a 65,536-token
causal sequence (512 q-blocks, 512 K/V tiles per q-block at the end: offsets
and tile counts far beyond the benchmark's) sits between short ones, and a
decode step reads a 131,072-row cache. Outputs start as NaN, so a row that is
never written fails; the long sequence is compared with the oracle on a
stratified sample (first, last and two random rows of every q-block, one head
of every K/V group), the short ones in full through the same sample.
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
