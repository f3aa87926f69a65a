"""Randomized GPU parity: seeded random packs against the oracle.

Each case draws a batch size, per-sequence query and key lengths (zero-length
members, lengths that are and are not multiples of the 128-row tile, Lq != Lk
in both directions), the GQA group, head_dim, the mask, and the biases
(per-key, per-pair grid shared by the heads, per query head or per K/V head),
then compares every output element of the CUDA path (through the C ABI) with
the oracle at the library's tolerances. The same draws feed the backward (all
gradients) and the K/V-cache decode step; random masks and row shapes feed the
unpad / pad helpers (bit for bit) and random strided grids the first-token
fold. Sizes stay small enough for the fp64 oracle to finish each case in well
under a second.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import layout
from oracle.backward import bwd as oracle_bwd
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


def _draw(seed, max_len=300):
    r = np.random.default_rng(seed)
    B = int(r.integers(1, 9))
    Hkv = int(r.choice([1, 2, 3]))
    G = int(r.choice([1, 2, 3, 4, 7, 8]))
    D = int(r.choice([64, 128]))
    causal = bool(r.integers(0, 2))
    lq = [int(x) for x in r.integers(0, max_len + 1, B)]
    if r.integers(0, 3) == 0:
        lq[int(r.integers(0, B))] = 0
    if r.integers(0, 2) == 0:
        lk = list(lq)
    else:
        lk = [int(x) for x in r.integers(0, max_len + 1, B)]
    if max(lq) == 0:
        lq[0] = 1
    bias = str(r.choice(["none", "key", "pair", "both", "pair_kv"]))
    shared_grid = bool(r.integers(0, 2))
    return dict(B=B, Hkv=Hkv, Hq=G * Hkv, G=G, D=D, causal=causal, lq=lq, lk=lk, bias=bias,
                shared_grid=shared_grid)


def _workload(c, seed):
    bias_key = c["bias"] in ("key", "both")
    grid = None
    if c["bias"] in ("pair", "both", "pair_kv"):
        if c["bias"] == "pair_kv":
            Hg = c["Hkv"]
        else:
            Hg = 1 if c["shared_grid"] else c["Hq"]
        grid = (c["B"], Hg, max(max(c["lq"]), 1), max(max(c["lk"]), 1))
    return workloads.make_custom(c["lq"], c["lk"], n_heads=c["Hq"], n_kv_heads=c["Hkv"],
                                 head_dim=c["D"], causal=c["causal"], seed=seed,
                                 bias_key=bias_key, bias_pair=grid, bias_key_std=0.5)


def _oracle_grid(w, c):
    """The grid the oracle reads: a per-K/V-head grid expanded to query heads."""
    if w.bias_pair is None:
        return None, None
    if c["bias"] == "pair_kv":
        e = layout.expand_kv_head_grid(w.bias_pair.numpy(), c["G"])
        B, H, R, C = e.shape
        return torch.from_numpy(e), (H * R * C, R * C, C, 1)
    return w.bias_pair, w.bias_strides


def _fwd_gpu(w, c, dev):
    return va.varlen_attn_fwd(dev["q"], dev["k"], dev["v"], dev["cu_q"], dev["cu_k"],
                              w.max_seqlen_q, w.max_seqlen_k, softmax_scale=w.softmax_scale,
                              causal=w.causal, bias_per_key=dev["bias_key"],
                              bias_pair=dev["bias_pair"],
                              bias_pair_strides=w.bias_strides if w.bias_pair is not None else None,
                              bias_pair_kv_heads=c["bias"] == "pair_kv")


@pytest.mark.parametrize("seed", range(40))
def test_random_pack_forward(seed):
    c = _draw(1000 + seed)
    w = _workload(c, 1000 + seed)
    dev = to_device(w)
    out = torch.full_like(dev["q"], float("nan"))
    lse = torch.full((w.n_heads, w.total_q), float("nan"), device="cuda")
    o, l = va.varlen_attn_fwd(dev["q"], dev["k"], dev["v"], dev["cu_q"], dev["cu_k"],
                              w.max_seqlen_q, w.max_seqlen_k, softmax_scale=w.softmax_scale,
                              causal=w.causal, bias_per_key=dev["bias_key"],
                              bias_pair=dev["bias_pair"],
                              bias_pair_strides=w.bias_strides if w.bias_pair is not None else None,
                              bias_pair_kv_heads=c["bias"] == "pair_kv", out=out, lse=lse)
    torch.cuda.synchronize()
    grid, strides = _oracle_grid(w, c)
    ref_o, ref_l = oracle.fwd(w.q, w.k, w.v, w.cu_q, w.cu_k, w.n_heads, w.n_kv_heads,
                              w.softmax_scale, w.causal, bias_key=w.bias_key, bias_pair=grid,
                              bias_strides=strides)
    compare(o, l, ref_o, ref_l)


@pytest.mark.parametrize("seed", range(10))
def test_random_pack_fp32_forward(seed):
    c = _draw(2000 + seed, max_len=200)
    if c["bias"] == "pair_kv":  # a bf16-path option
        c["bias"] = "pair"
    w = _workload(c, 2000 + seed)
    w.q, w.k, w.v = w.q.float(), w.k.float(), w.v.float()
    dev = to_device(w)
    o, l = _fwd_gpu(w, c, dev)
    torch.cuda.synchronize()
    assert o.dtype == torch.float32
    ref_o, ref_l = oracle.fwd(w.q, w.k, w.v, w.cu_q, w.cu_k, w.n_heads, w.n_kv_heads,
                              w.softmax_scale, w.causal, bias_key=w.bias_key,
                              bias_pair=w.bias_pair, bias_strides=w.bias_strides)
    compare(o, l, ref_o, ref_l, fp32=True)


def _close(name, got, ref, rel_l2=1e-2, max_abs_frac=2e-2):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, name
    assert np.isfinite(got).all(), name
    den = np.linalg.norm(ref)
    err = np.linalg.norm(got - ref)
    rel = err / den if den > 0 else err
    scale = np.abs(ref).max() if ref.size else 0.0
    mx = np.abs(got - ref).max() if got.size else 0.0
    assert rel <= rel_l2, (name, rel)
    assert mx <= max_abs_frac * max(scale, 1e-6), (name, mx, scale)


@pytest.mark.parametrize("seed", range(12))
def test_random_pack_backward(seed):
    c = _draw(3000 + seed, max_len=260)
    w = _workload(c, 3000 + seed)
    dev = to_device(w)
    o, l = _fwd_gpu(w, c, dev)
    g = torch.Generator().manual_seed(4000 + seed)
    dout = torch.randn(w.q.shape, generator=g).to(torch.bfloat16)
    has_bk, has_bp = w.bias_key is not None, w.bias_pair is not None
    dq, dk, dv, dbk, dbp = va.varlen_attn_bwd(
        dev["q"], dev["k"], dev["v"], o, l, dout.cuda(), dev["cu_q"], dev["cu_k"],
        w.max_seqlen_q, w.max_seqlen_k, softmax_scale=w.softmax_scale, causal=w.causal,
        bias_per_key=dev["bias_key"], bias_pair=dev["bias_pair"],
        bias_pair_strides=w.bias_strides if has_bp else None,
        bias_pair_kv_heads=c["bias"] == "pair_kv",
        need_dbias_per_key=has_bk, need_dbias_pair=has_bp)
    torch.cuda.synchronize()
    grid, strides = _oracle_grid(w, c)
    ref = oracle_bwd(w.q, w.k, w.v, dout, w.cu_q, w.cu_k, w.n_heads, w.n_kv_heads,
                     w.softmax_scale, w.causal, bias_key=w.bias_key, bias_pair=grid,
                     bias_strides=strides)
    _close("dq", dq.float().cpu().numpy(), ref["dq"])
    _close("dk", dk.float().cpu().numpy(), ref["dk"])
    _close("dv", dv.float().cpu().numpy(), ref["dv"])
    if has_bk:
        _close("dbias_key", dbk.cpu().numpy(), ref["dbias_key"])
    if has_bp:
        _close("dbias_pair", dbp.cpu().numpy(), ref["dbias_pair"])


@pytest.mark.parametrize("seed", range(10))
def test_random_decode(seed):
    r = np.random.default_rng(5000 + seed)
    B = int(r.integers(1, 12))
    Hkv = int(r.choice([1, 2, 4, 8]))
    G = int(r.choice([1, 2, 4, 7, 8]))
    Hq, D = G * Hkv, int(r.choice([64, 128]))
    max_q = int(max(1, min(32 // G, r.integers(1, 5))))
    lq = [int(x) for x in r.integers(1, max_q + 1, B)]
    cache_len = int(r.integers(64, 1500))
    new = bool(r.integers(0, 2))
    cl = [int(x) for x in r.integers(0, cache_len - (max_q if new else 0) + 1, B)]
    g = torch.Generator().manual_seed(6000 + seed)
    cu_q = torch.tensor(np.concatenate([[0], np.cumsum(lq)]), dtype=torch.int32)
    Tq = int(cu_q[-1])
    q = torch.randn(Tq, Hq, D, generator=g).to(torch.bfloat16)
    kc = torch.randn(B, cache_len, Hkv, D, generator=g).to(torch.bfloat16)
    vc = torch.randn(B, cache_len, Hkv, D, generator=g).to(torch.bfloat16)
    kn = torch.randn(Tq, Hkv, D, generator=g).to(torch.bfloat16) if new else None
    vn = torch.randn(Tq, Hkv, D, generator=g).to(torch.bfloat16) if new else None
    cs = torch.tensor(cl, dtype=torch.int32)
    kcd, vcd = kc.cuda(), vc.cuda()
    scale = 1.0 / np.sqrt(D)
    out, lse = va.varlen_attn_decode(q.cuda(), cu_q.cuda(), max(lq), kcd, vcd, cs.cuda(),
                                     None if kn is None else kn.cuda(),
                                     None if vn is None else vn.cuda(), softmax_scale=scale,
                                     causal=True, num_splits=int(r.integers(0, 4)))
    torch.cuda.synchronize()
    kcache, vcache = kc.clone(), vc.clone()
    if new:
        for i in range(B):
            a, b = int(cu_q[i]), int(cu_q[i + 1])
            kcache[i, cl[i]:cl[i] + (b - a)] = kn[a:b]
            vcache[i, cl[i]:cl[i] + (b - a)] = vn[a:b]
    assert torch.equal(kcd.cpu().view(torch.int16), kcache.view(torch.int16))
    lk = [cl[i] + (lq[i] if new else 0) for i in range(B)]
    k = torch.cat([kcache[i, :lk[i]] for i in range(B)])
    v = torch.cat([vcache[i, :lk[i]] for i in range(B)])
    cu_k = torch.tensor(np.concatenate([[0], np.cumsum(lk)]), dtype=torch.int32)
    ref_o, ref_l = oracle.fwd(q, k, v, cu_q, cu_k, Hq, Hkv, scale, True)
    compare(out, lse, ref_o, ref_l)


@pytest.mark.parametrize("seed", range(8))
def test_random_unpad_pad_bit_exact(seed):
    """Random masks (holes, prefixes, empty and full rows) and row shapes:
    unpadding metadata, gather and scatter bit for bit against the oracle."""
    r = np.random.default_rng(7000 + seed)
    B, S = int(r.integers(1, 10)), int(r.integers(1, 700))
    kind = int(r.integers(0, 3))
    if kind == 0:
        mask = r.random((B, S)) < r.uniform(0.05, 0.95)
    else:
        mask = np.zeros((B, S), dtype=bool)
        for b in range(B):
            L = int(r.integers(0, S + 1))
            mask[b, :L] = True
        if kind == 2:  # and a few holes
            mask &= r.random((B, S)) < 0.9
    H = int(r.choice([1, 2, 3, 8]))
    D = int(r.choice([8, 64, 128]))
    dtype = torch.bfloat16 if r.integers(0, 2) else torch.float32
    g = torch.Generator().manual_seed(8000 + seed)
    x = torch.randn(B, S, H, D, generator=g).to(dtype)
    packed, idx, cu, mx = va.unpad(x.cuda(), torch.from_numpy(mask).cuda())
    back = va.pad(packed, idx, cu, B, S)
    torch.cuda.synchronize()
    ref_cu, ref_idx, ref_mx = layout.mask_to_seqlens(mask)
    assert cu.cpu().numpy().tolist() == ref_cu.tolist()
    assert int(mx) == ref_mx
    bits = torch.int16 if dtype == torch.bfloat16 else torch.int32
    rows = x.view(bits).numpy().reshape(B * S, H, D)
    ref_packed = layout.gather_rows(rows, ref_idx)
    assert np.array_equal(packed.cpu().view(bits).numpy(), ref_packed)
    ref_back = layout.scatter_rows(ref_packed, ref_idx, B * S).reshape(B, S, H, D)
    assert np.array_equal(back.cpu().view(bits).numpy(), ref_back)


@pytest.mark.parametrize("seed", range(6))
def test_random_fold_matches_oracle(seed):
    """First-token fold of random strided grids (per query head or per K/V
    head, with and without a per-key bias to add to)."""
    r = np.random.default_rng(9000 + seed)
    B = int(r.integers(1, 9))
    lk = [int(x) for x in r.integers(0, 300, B)]
    if sum(lk) == 0:
        lk[0] = 1
    Hkv = int(r.choice([1, 2, 4]))
    G = int(r.choice([1, 2, 4]))
    Hq = Hkv * G
    kv_heads = bool(r.integers(0, 2))
    Hg = Hkv if kv_heads else Hq
    rows = int(r.integers(1, 4))
    row = int(r.integers(0, rows))
    with_key = bool(r.integers(0, 2))
    w = workloads.make_custom([1] * B, lk, n_heads=Hq, n_kv_heads=Hkv, head_dim=64, causal=False,
                              seed=9100 + seed, bias_pair=(B, Hg, rows, max(lk)),
                              bias_key=with_key)
    dev = to_device(w)
    head_div = G if kv_heads else 1
    folded = va.fold_pair_bias_row(dev["bias_pair"], dev["cu_k"], Hq, w.total_k, row=row,
                                   head_div=head_div,
                                   bias_in=dev["bias_key"] if with_key else None)
    torch.cuda.synchronize()
    gflat = w.bias_pair.numpy().reshape(-1)
    sb, sh, sr, sc = w.bias_strides
    cu = w.cu_k.numpy()
    want = np.zeros((w.total_k, Hq), dtype=np.float32)
    for i in range(B):
        for h in range(Hq):
            for c in range(lk[i]):
                v = np.float32(gflat[i * sb + (h // head_div) * sh + row * sr + c * sc])
                want[cu[i] + c, h] = (np.float32(w.bias_key[cu[i] + c, h].item()) + v
                                      if with_key else v)
    assert np.array_equal(folded.cpu().numpy(), want)
    ref = layout.fold_pair_row(w.bias_pair.numpy(), w.bias_strides, row, cu, Hq, w.total_k,
                               head_div=head_div,
                               bias_key=w.bias_key.numpy() if with_key else None)
    np.testing.assert_allclose(folded.cpu().numpy(), ref, rtol=1e-6, atol=1e-6)
