"""GPU parity of the K/V-cache decode path (varlen_attn_decode) against the
attention oracle run on the packed K/V the cache holds after the append."""
import numpy as np
import pytest
import torch

import oracle
import packed_variable_length_attn_b200 as va
from tests.parity import compare

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    va.get_device_error()
    yield
    assert va.get_device_error() == 0


def _case(seed, lq, cache_lens, cache_len, hq, hkv, d, new):
    g = torch.Generator().manual_seed(seed)
    B = len(lq)
    cu_q = torch.tensor(np.concatenate([[0], np.cumsum(lq)]), dtype=torch.int32)
    Tq = int(cu_q[-1])
    q = torch.randn(Tq, hq, d, generator=g).to(torch.bfloat16)
    kc = torch.randn(B, cache_len, hkv, d, generator=g).to(torch.bfloat16)
    vc = torch.randn(B, cache_len, hkv, d, generator=g).to(torch.bfloat16)
    cs = torch.tensor(cache_lens, dtype=torch.int32)
    kn = torch.randn(Tq, hkv, d, generator=g).to(torch.bfloat16) if new else None
    vn = torch.randn(Tq, hkv, d, generator=g).to(torch.bfloat16) if new else None
    return cu_q, q, kc, vc, cs, kn, vn


def _expected_cache(kc, cs, cu_q, kn):
    exp = kc.clone()
    if kn is not None:
        for i in range(len(cs)):
            a, b = int(cu_q[i]), int(cu_q[i + 1])
            exp[i, int(cs[i]):int(cs[i]) + (b - a)] = kn[a:b]
    return exp


def _oracle(q, cu_q, kcache, vcache, lk, hq, hkv, scale, causal):
    k = torch.cat([kcache[i, :lk[i]] for i in range(len(lk))])
    v = torch.cat([vcache[i, :lk[i]] for i in range(len(lk))])
    cu_k = torch.tensor(np.concatenate([[0], np.cumsum(lk)]), dtype=torch.int32)
    return oracle.fwd(q, k, v, cu_q, cu_k, hq, hkv, scale, causal)


CASES = [
    # lq, cache lens, cache_len, hq, hkv, d, new rows, splits
    ([1] * 8, [700, 1, 0, 4096, 129, 64, 2000, 3333], 4096, 32, 8, 128, False, 0),
    ([1] * 8, [700, 1, 0, 4096, 129, 64, 2000, 3333], 4096, 32, 8, 128, False, 1),
    ([1] * 5, [10, 300, 511, 0, 77], 512, 16, 4, 64, True, 0),
    ([4, 1, 8, 2], [100, 0, 300, 1000], 1024, 8, 2, 128, True, 3),
    ([1] * 3, [5000, 17, 8000], 8192, 14, 2, 64, True, 7),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"B{len(c[0])}_D{c[5]}_G{c[3] // c[4]}_"
                         f"{'new' if c[6] else 'cached'}_s{c[7]}")
def test_decode_parity(case):
    lq, cache_lens, cache_len, hq, hkv, d, new, splits = case
    cu_q, q, kc, vc, cs, kn, vn = _case(sum(cache_lens) + d, lq, cache_lens, cache_len, hq, hkv,
                                        d, new)
    kcd, vcd = kc.cuda(), vc.cuda()
    scale = 1.0 / np.sqrt(d)
    out, lse = va.varlen_attn_decode(q.cuda(), cu_q.cuda(), max(lq), kcd, vcd, cs.cuda(),
                                     None if kn is None else kn.cuda(),
                                     None if vn is None else vn.cuda(), softmax_scale=scale,
                                     causal=True, num_splits=splits)
    torch.cuda.synchronize()
    exp_k = _expected_cache(kc, cs, cu_q, kn)
    exp_v = _expected_cache(vc, cs, cu_q, vn)
    assert torch.equal(kcd.cpu().view(torch.int16), exp_k.view(torch.int16))
    assert torch.equal(vcd.cpu().view(torch.int16), exp_v.view(torch.int16))
    lk = [cache_lens[i] + (lq[i] if new else 0) for i in range(len(lq))]
    ref_o, ref_l = _oracle(q, cu_q, exp_k, exp_v, lk, hq, hkv, scale, True)
    compare(out, lse, ref_o, ref_l)


@pytest.mark.parametrize("hq,hkv,d,lq", [(32, 8, 128, 1), (14, 2, 64, 1), (8, 2, 128, 8)])
def test_decode_ignores_cache_rows_past_each_length(hq, hkv, d, lq):
    """Cache rows at and past each sequence's length hold NaN: the output is
    finite and equals the result over the valid rows (keys there are masked
    in the scores and never multiplied in P V)."""
    cache_lens = [0, 1, 31, 32, 33, 1000, 4095]
    lqs = [lq] * len(cache_lens)
    cu_q, q, kc, vc, cs, _, _ = _case(77 + d, lqs, cache_lens, 4096 + 8, hq, hkv, d, False)
    kn = torch.zeros(1)  # unused
    kcn, vcn = kc.clone(), vc.clone()
    for i, L in enumerate(cache_lens):
        kcn[i, L:] = float("nan")
        vcn[i, L:] = float("nan")
    scale = 1.0 / np.sqrt(d)
    for splits in (0, 1, 3):
        out, lse = va.varlen_attn_decode(q.cuda(), cu_q.cuda(), lq, kcn.cuda(), vcn.cuda(),
                                         cs.cuda(), softmax_scale=scale, causal=True,
                                         num_splits=splits)
        torch.cuda.synchronize()
        assert torch.isfinite(out.float()).all()
        ref_o, ref_l = _oracle(q, cu_q, kc, vc, cache_lens, hq, hkv, scale, True)
        compare(out, lse, ref_o, ref_l)
    del kn


def test_decode_split_count_changes_only_rounding_and_is_deterministic():
    lq, cache_lens = [1] * 6, [4000, 3000, 1, 2222, 4096, 100]
    cu_q, q, kc, vc, cs, _, _ = _case(9, lq, cache_lens, 4096, 32, 8, 128, False)
    args = (q.cuda(), cu_q.cuda(), 1, kc.cuda(), vc.cuda(), cs.cuda())
    res = {}
    for s in (1, 2, 5, 5):
        o, l = va.varlen_attn_decode(*args, num_splits=s)
        torch.cuda.synchronize()
        if s in res:
            assert torch.equal(o.view(torch.int16), res[s][0].view(torch.int16))
            assert torch.equal(l.view(torch.int32), res[s][1].view(torch.int32))
        res[s] = (o.clone(), l.clone())
    for s in (2, 5):
        assert (res[s][0].float() - res[1][0].float()).abs().max().item() < 2e-2
        assert (res[s][1] - res[1][1]).abs().max().item() < 1e-4


def test_decode_cache_overflow_reported():
    cu_q = torch.tensor([0, 2], dtype=torch.int32, device="cuda")
    q = torch.zeros(2, 4, 64, dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros(1, 8, 1, 64, dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    kn = torch.ones(2, 1, 64, dtype=torch.bfloat16, device="cuda")
    cs = torch.tensor([7], dtype=torch.int32, device="cuda")   # 7 + 2 new rows > 8
    va.varlen_attn_decode(q, cu_q, 2, kc, vc, cs, kn, kn.clone())
    assert va.get_device_error() == va.ERR_BAD_SEQLENS
    assert torch.equal(kc[0, :7].cpu(), torch.zeros(7, 1, 64, dtype=torch.bfloat16))


# Enough (sequence, K/V head) pairs to fill the GPU: the automatic path runs
# on the tensor cores (packed forward kernel, K/V read in place from the cache,
# the G query heads of a group in one tile).
TC_CASES = [
    # B, hkv, G, d, q_len, new rows
    (40, 4, 4, 128, 1, False),
    (40, 4, 4, 128, 4, True),
    (160, 1, 7, 64, 2, False),
    (24, 8, 8, 64, 3, True),
    (75, 2, 1, 128, 1, True),
]


@pytest.mark.parametrize("case", TC_CASES, ids=lambda c: f"B{c[0]}_kv{c[1]}_G{c[2]}_D{c[3]}_q{c[4]}"
                         f"{'_new' if c[5] else ''}")
def test_decode_tensor_core_path_parity(case):
    B, hkv, G, d, ql, new = case
    assert B * hkv >= torch.cuda.get_device_properties(0).multi_processor_count
    hq = hkv * G
    r = np.random.default_rng(B * 7 + d)
    cache_len = 2048
    lq = [ql] * B
    cl = [int(x) for x in r.integers(0, cache_len - (ql if new else 0) + 1, B)]
    cl[0] = 0
    cl[1] = cache_len - (ql if new else 0)
    cu_q, q, kc, vc, cs, kn, vn = _case(B + d, lq, cl, cache_len, hq, hkv, d, new)
    # unwritten cache slots past each length hold NaN
    kcn, vcn = kc.clone(), vc.clone()
    for i, L in enumerate(cl):
        kcn[i, L:] = float("nan")
        vcn[i, L:] = float("nan")
    kcd, vcd = kcn.cuda(), vcn.cuda()
    scale = 1.0 / np.sqrt(d)
    out, lse = va.varlen_attn_decode(q.cuda(), cu_q.cuda(), ql, kcd, vcd, cs.cuda(),
                                     None if kn is None else kn.cuda(),
                                     None if vn is None else vn.cuda(), softmax_scale=scale,
                                     causal=True)
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all()
    exp_k = _expected_cache(kc, cs, cu_q, kn)
    exp_v = _expected_cache(vc, cs, cu_q, vn)
    lk = [cl[i] + (ql if new else 0) for i in range(B)]
    ref_o, ref_l = _oracle(q, cu_q, exp_k, exp_v, lk, hq, hkv, scale, True)
    compare(out, lse, ref_o, ref_l)


# Fewer (sequence, K/V head) pairs than SMs: the automatic path still runs on
# the tensor cores, each sequence's keys cut into fixed ranges of the cache
# (at least 512 keys, a multiple of the 128-key tile), one work item per
# (range, pair), the ranges' outputs merged by LSE. The lengths sit on and
# next to multiples of 512 and at both ends, and several new tokens put the
# causal diagonal across a range boundary (a sequence of 513 keys has a
# one-key last range, so the earlier tokens see only part of the range before).
RANGE_CASES = [
    # B, hkv, G, d, q_len, new rows, cache_len
    (8, 4, 4, 128, 1, False, 4096),
    (8, 4, 4, 128, 4, True, 4096),
    (7, 2, 7, 64, 2, False, 3000),
    (2, 8, 4, 64, 8, True, 8192),
    (6, 1, 1, 128, 16, True, 2048),
    (8, 3, 4, 128, 4, False, 4096),
]


@pytest.mark.parametrize("case", RANGE_CASES, ids=lambda c: f"B{c[0]}_kv{c[1]}_G{c[2]}_D{c[3]}"
                         f"_q{c[4]}{'_new' if c[5] else ''}_S{c[6]}")
def test_decode_key_range_path_parity(case):
    B, hkv, G, d, ql, new, cache_len = case
    assert B * hkv < torch.cuda.get_device_properties(0).multi_processor_count
    hq = hkv * G
    r = np.random.default_rng(B * 11 + d + cache_len)
    extra = ql if new else 0
    targets = [0, 1, 512, 513, 1023, 1029, cache_len, 2 * 512 + 3]
    lk = [max(extra, min(cache_len, t)) for t in targets[:B]]
    if B > len(targets):
        lk += [int(x) for x in r.integers(extra, cache_len + 1, B - len(targets))]
    cl = [L - extra for L in lk]
    cu_q, q, kc, vc, cs, kn, vn = _case(B * 13 + d, [ql] * B, cl, cache_len, hq, hkv, d, new)
    kcn, vcn = kc.clone(), vc.clone()  # unwritten cache slots past each length hold NaN
    for i, L in enumerate(cl):
        kcn[i, L:] = float("nan")
        vcn[i, L:] = float("nan")
    scale = 1.0 / np.sqrt(d)
    outs = []
    for _ in range(2):
        kcd, vcd = kcn.cuda(), vcn.cuda()
        out, lse = va.varlen_attn_decode(q.cuda(), cu_q.cuda(), ql, kcd, vcd, cs.cuda(),
                                         None if kn is None else kn.cuda(),
                                         None if vn is None else vn.cuda(),
                                         softmax_scale=scale, causal=True)
        torch.cuda.synchronize()
        outs.append((out, lse))
    assert torch.isfinite(outs[0][0].float()).all()
    for a, b in zip(outs[0], outs[1]):  # deterministic run to run
        assert torch.equal(a.contiguous().view(torch.int32 if a.dtype == torch.float32
                                               else torch.int16),
                           b.contiguous().view(torch.int32 if b.dtype == torch.float32
                                               else torch.int16))
    exp_k = _expected_cache(kc, cs, cu_q, kn)
    exp_v = _expected_cache(vc, cs, cu_q, vn)
    ref_o, ref_l = _oracle(q, cu_q, exp_k, exp_v, lk, hq, hkv, scale, True)
    compare(outs[0][0], outs[0][1], ref_o, ref_l)
