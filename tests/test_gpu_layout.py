"""GPU parity of the per-K/V-head pair bias and the packed-layout helpers,
through the C ABI, against the oracle (oracle/ and oracle/layout.py).

Integer and byte work (unpadding metadata, row gather / scatter) must match
bit for bit; the fold is one fp32 add per element and must match the fp32 sum
exactly; attention results use the bf16 tolerances of tests/parity.py.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import layout
import packed_variable_length_attn_b200 as va
from packed_variable_length_attn_b200 import workloads
from tests.parity import compare, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    va.get_device_error()
    yield
    assert va.get_device_error() == 0


# ----------------------------------------------------------------- per-K/V-head pair bias

@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_kv_head_pair_bias_parity(d, causal):
    lq = [7, 130, 1, 257, 64]
    lk = [9, 130, 40, 300, 64]
    Hq, Hkv = 8, 2
    w = workloads.make_custom(lq, lk, n_heads=Hq, n_kv_heads=Hkv, head_dim=d, causal=causal,
                              seed=101 + d, bias_pair=(len(lq), Hkv, max(lq), max(lk)))
    grid = w.bias_pair  # [B, Hkv, R, C]
    dev = to_device(w)
    out, lse = va.varlen_attn_fwd(dev["q"], dev["k"], dev["v"], dev["cu_q"], dev["cu_k"],
                                  w.max_seqlen_q, w.max_seqlen_k, softmax_scale=w.softmax_scale,
                                  causal=causal, bias_pair=dev["bias_pair"],
                                  bias_pair_kv_heads=True)
    torch.cuda.synchronize()
    expanded = layout.expand_kv_head_grid(grid.numpy(), Hq // Hkv)
    B, H, R, C = expanded.shape
    ref_o, ref_l = oracle.fwd(w.q, w.k, w.v, w.cu_q, w.cu_k, Hq, Hkv, w.softmax_scale, causal,
                              bias_pair=expanded, bias_strides=(H * R * C, R * C, C, 1))
    compare(out, lse, ref_o, ref_l)


def test_kv_head_flag_is_identity_without_gqa():
    w = workloads.make_custom([33, 200], n_heads=4, n_kv_heads=4, head_dim=64, causal=True,
                              seed=5, bias_pair=(2, 4, 200, 200))
    dev = to_device(w)
    kw = dict(softmax_scale=w.softmax_scale, causal=True, bias_pair=dev["bias_pair"])
    o1, l1 = va.varlen_attn_fwd(dev["q"], dev["k"], dev["v"], dev["cu_q"], dev["cu_k"], 200, 200,
                                **kw)
    o2, l2 = va.varlen_attn_fwd(dev["q"], dev["k"], dev["v"], dev["cu_q"], dev["cu_k"], 200, 200,
                                bias_pair_kv_heads=True, **kw)
    torch.cuda.synchronize()
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
    assert torch.equal(l1.view(torch.int32), l2.view(torch.int32))


# ----------------------------------------------------------------- unpad / pad

def _masks():
    rng = np.random.default_rng(17)
    yield "holes", rng.random((13, 300)) < 0.35
    prefix = np.zeros((6, 1000), dtype=bool)
    for b, L in enumerate([1000, 1, 0, 513, 257, 999]):
        prefix[b, :L] = True
    yield "prefix", prefix
    yield "all_valid", np.ones((3, 4096), dtype=bool)
    yield "one_row", rng.random((1, 17)) < 0.5


@pytest.mark.parametrize("name,mask", list(_masks()), ids=[n for n, _ in _masks()])
def test_mask_to_seqlens_bit_exact(name, mask):
    cu, idx, mx = va.mask_to_seqlens(torch.from_numpy(mask).cuda())
    torch.cuda.synchronize()
    ref_cu, ref_idx, ref_mx = layout.mask_to_seqlens(mask)
    assert cu.cpu().numpy().tolist() == ref_cu.tolist()
    T = int(ref_cu[-1])
    assert idx[:T].cpu().numpy().tolist() == ref_idx.tolist()
    assert int(mx.item()) == ref_mx


@pytest.mark.parametrize("name,mask", list(_masks())[:2], ids=["holes", "prefix"])
def test_unpad_pad_bit_exact(name, mask):
    B, S = mask.shape
    H, D = 3, 64
    g = torch.Generator().manual_seed(3)
    x = torch.randn(B, S, H, D, generator=g).to(torch.bfloat16)
    packed, idx, cu, mx = va.unpad(x.cuda(), torch.from_numpy(mask).cuda())
    torch.cuda.synchronize()
    ref_cu, ref_idx, _ = layout.mask_to_seqlens(mask)
    ref_packed = layout.gather_rows(x.view(torch.int16).numpy().reshape(B * S, H, D), ref_idx)
    assert np.array_equal(packed.cpu().view(torch.int16).numpy(), ref_packed)
    back = va.pad(packed, idx, cu, B, S)
    torch.cuda.synchronize()
    ref_back = layout.scatter_rows(ref_packed, ref_idx, B * S).reshape(B, S, H, D)
    assert np.array_equal(back.cpu().view(torch.int16).numpy(), ref_back)


def test_gather_rejects_out_of_range_index():
    src = torch.zeros(4, 8, dtype=torch.float32, device="cuda")
    out = torch.full((3, 8), 7.0, device="cuda")
    cu = torch.tensor([0, 3], dtype=torch.int32, device="cuda")
    idx = torch.tensor([0, 9, 1], dtype=torch.int32, device="cuda")   # 9 >= 4 source rows
    va.gather_rows(src, idx, cu, out)
    assert va.get_device_error() == va.ERR_BAD_SEQLENS
    o = out.cpu()
    assert torch.equal(o[1], torch.full((8,), 7.0))   # the bad row is skipped
    assert torch.equal(o[0], torch.zeros(8)) and torch.equal(o[2], torch.zeros(8))


# ----------------------------------------------------------------- first-token fold

@pytest.mark.parametrize("kv_heads", [False, True])
def test_fold_bit_exact_and_equivalent_attention(kv_heads):
    lk = [5, 1, 300, 64, 129]
    Hq, Hkv = 8, 4
    Hg = Hkv if kv_heads else Hq
    w = workloads.make_custom([1] * len(lk), lk, n_heads=Hq, n_kv_heads=Hkv, head_dim=64,
                              causal=False, seed=23 + int(kv_heads),
                              bias_pair=(len(lk), Hg, 1, max(lk)), bias_key=True)
    dev = to_device(w)
    head_div = Hq // Hkv if kv_heads else 1
    folded = va.fold_pair_bias_row(dev["bias_pair"], dev["cu_k"], Hq, w.total_k, row=0,
                                   head_div=head_div, bias_in=dev["bias_key"])
    torch.cuda.synchronize()
    # one fp32 add per element: equal to the fp32 sum of the same two values
    gflat = w.bias_pair.numpy().reshape(-1)
    want = np.zeros((w.total_k, Hq), dtype=np.float32)
    cu = w.cu_k.numpy()
    sb, sh, sr, sc = w.bias_strides
    for i in range(len(lk)):
        for h in range(Hq):
            for c in range(lk[i]):
                want[cu[i] + c, h] = np.float32(w.bias_key[cu[i] + c, h].item()) + \
                    np.float32(gflat[i * sb + (h // head_div) * sh + c * sc])
    assert np.array_equal(folded.cpu().numpy(), want)
    # the fold's oracle agrees with the same definition in fp64
    ref = layout.fold_pair_row(w.bias_pair.numpy(), w.bias_strides, 0, cu, Hq, w.total_k,
                               head_div=head_div, bias_key=w.bias_key.numpy())
    np.testing.assert_allclose(folded.cpu().numpy(), ref, rtol=1e-6, atol=1e-6)
    # attention with the folded per-key bias = attention with the grid (one query row each)
    out_f, lse_f = va.varlen_attn_fwd(dev["q"], dev["k"], dev["v"], dev["cu_q"], dev["cu_k"], 1,
                                      w.max_seqlen_k, softmax_scale=w.softmax_scale,
                                      bias_per_key=folded)
    torch.cuda.synchronize()
    ref_o, ref_l = oracle.fwd(w.q, w.k, w.v, w.cu_q, w.cu_k, Hq, Hkv, w.softmax_scale, False,
                              bias_key=ref)
    compare(out_f, lse_f, ref_o, ref_l)
