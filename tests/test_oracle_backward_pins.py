"""Pins of the backward oracle (oracle/backward.py), independent of its code.

- Central finite differences of the forward oracle (the C code, fp64 inputs):
  the loss sum(dO * O) is evaluated at x ± h for sampled entries of Q, K, V,
  the per-key bias and the pair grid; the oracle's gradient entry must match
  the difference quotient. A dropped term, a wrong sign, a transposed product
  or a wrong head/group index fails here.
- Invariants of the softmax Jacobian: every row of dS sums to zero (so the
  pair-grid gradient has zero row sums and the per-key bias gradient sums to
  zero over keys), and sum over keys of dV = sum over rows of dO for each
  (sequence, head group) whose rows all see a key.
- A one-key sequence has P = 1: dQ = dK = 0 and dV = sum of dO.
"""
import numpy as np
import pytest
from hypothesis import HealthCheck, given, settings, strategies as st

import oracle
from oracle.backward import bwd


def _case(seed, causal, with_bias):
    rng = np.random.default_rng(seed)
    lq = [3, 5, 1, 4, 4]   # the last one: Lq > Lk, so under causal its first rows see no key
    lk = [3, 7, 2, 4, 2]
    Hq, Hkv, D = 4, 2, 8
    cu_q = np.concatenate([[0], np.cumsum(lq)]).astype(np.int32)
    cu_k = np.concatenate([[0], np.cumsum(lk)]).astype(np.int32)
    Tq, Tk = int(cu_q[-1]), int(cu_k[-1])
    q = rng.standard_normal((Tq, Hq, D))
    k = rng.standard_normal((Tk, Hkv, D))
    v = rng.standard_normal((Tk, Hkv, D))
    dout = rng.standard_normal((Tq, Hq, D))
    bk = bp = strides = None
    if with_bias:
        bk = rng.standard_normal((Tk, Hq)) * 0.5
        R, C = max(lq), max(lk)
        bp = rng.standard_normal((len(lq), Hq, R, C))
        strides = (Hq * R * C, R * C, C, 1)
    return dict(q=q, k=k, v=v, dout=dout, cu_q=cu_q, cu_k=cu_k, Hq=Hq, Hkv=Hkv,
                scale=0.37, causal=causal, bk=bk, bp=bp, strides=strides)


def _loss(c, q=None, k=None, v=None, bk=None, bp=None):
    o, _ = oracle.fwd(c["q"] if q is None else q, c["k"] if k is None else k,
                      c["v"] if v is None else v, c["cu_q"], c["cu_k"], c["Hq"], c["Hkv"],
                      c["scale"], c["causal"],
                      bias_key=c["bk"] if bk is None else bk,
                      bias_pair=c["bp"] if bp is None else bp, bias_strides=c["strides"],
                      threads=1)
    return float((o * c["dout"]).sum())


def _grads(c):
    return bwd(c["q"], c["k"], c["v"], c["dout"], c["cu_q"], c["cu_k"], c["Hq"], c["Hkv"],
               c["scale"], c["causal"], bias_key=c["bk"], bias_pair=c["bp"],
               bias_strides=c["strides"])


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("with_bias", [False, True])
def test_finite_differences(causal, with_bias):
    c = _case(11 + 2 * causal + with_bias, causal, with_bias)
    g = _grads(c)
    rng = np.random.default_rng(5)
    h = 1e-5
    names = ["q", "k", "v"] + (["bk", "bp"] if with_bias else [])
    grad_of = {"q": g["dq"], "k": g["dk"], "v": g["dv"], "bk": g["dbias_key"]}
    checked = 0
    for name in names:
        x = c[name]
        for _ in range(12):
            idx = tuple(int(rng.integers(0, s)) for s in x.shape)
            if name == "bp":
                # only in-sequence grid entries are read by the forward
                i, hh, r, col = idx
                lq = int(c["cu_q"][i + 1] - c["cu_q"][i])
                lk = int(c["cu_k"][i + 1] - c["cu_k"][i])
                idx = (i, hh, r % lq, col % lk)
            xp = x.copy(); xp[idx] += h
            xm = x.copy(); xm[idx] -= h
            fd = (_loss(c, **{name: xp}) - _loss(c, **{name: xm})) / (2 * h)
            got = g["dbias_pair"][idx] if name == "bp" else grad_of[name][idx]
            assert abs(got - fd) <= 1e-6 * (1 + abs(fd)), (name, idx, got, fd)
            checked += 1
    assert checked == 12 * len(names)


def test_jacobian_invariants():
    c = _case(3, True, True)
    g = _grads(c)
    # rows of dS sum to zero
    np.testing.assert_allclose(g["dbias_pair"].sum(axis=3), 0.0, atol=1e-12)
    # per sequence and head, the per-key gradient sums to zero over keys
    for i in range(len(c["cu_k"]) - 1):
        k0, k1 = c["cu_k"][i], c["cu_k"][i + 1]
        np.testing.assert_allclose(g["dbias_key"][k0:k1].sum(axis=0), 0.0, atol=1e-12)
    # sum over keys of dV = sum over rows of dO where every row sees a key
    # (bottom-right causal with Lk >= Lq)
    G = c["Hq"] // c["Hkv"]
    for i in range(len(c["cu_q"]) - 1):
        q0, q1 = c["cu_q"][i], c["cu_q"][i + 1]
        k0, k1 = c["cu_k"][i], c["cu_k"][i + 1]
        if q1 - q0 > k1 - k0:
            # rows without a visible key get no gradient at all
            nv = (q1 - q0) - (k1 - k0)
            assert np.abs(g["dq"][q0:q0 + nv]).max() == 0.0
            assert np.abs(g["dbias_pair"][i, :, :nv]).max() == 0.0
            continue
        for kvh in range(c["Hkv"]):
            lhs = g["dv"][k0:k1, kvh].sum(axis=0)
            rhs = c["dout"][q0:q1, kvh * G:(kvh + 1) * G].sum(axis=(0, 1))
            np.testing.assert_allclose(lhs, rhs, rtol=1e-12, atol=1e-12)


def test_single_key_sequence():
    rng = np.random.default_rng(8)
    q = rng.standard_normal((3, 2, 4))
    k = rng.standard_normal((1, 2, 4))
    v = rng.standard_normal((1, 2, 4))
    dout = rng.standard_normal((3, 2, 4))
    g = bwd(q, k, v, dout, [0, 3], [0, 1], 2, 2, 0.5, False)
    assert np.abs(g["dq"]).max() == 0.0 and np.abs(g["dk"]).max() == 0.0
    np.testing.assert_allclose(g["dv"][0], dout.sum(axis=0), rtol=1e-14)


@settings(max_examples=15, deadline=None, suppress_health_check=[HealthCheck.too_slow])
@given(data=st.data())
def test_finite_differences_random_packs(data):
    """Random packs (empty members, Lq != Lk, GQA, biases): sampled gradient
    entries against central differences of the forward oracle."""
    B = data.draw(st.integers(1, 3))
    lq = data.draw(st.lists(st.integers(0, 6), min_size=B, max_size=B))
    lk = data.draw(st.lists(st.integers(1, 6), min_size=B, max_size=B))
    if sum(lq) == 0:
        lq[0] = 1
    hkv = data.draw(st.sampled_from([1, 2]))
    Hq = hkv * data.draw(st.sampled_from([1, 2]))
    D = 4
    causal = data.draw(st.booleans())
    with_bias = data.draw(st.booleans())
    rng = np.random.default_rng(data.draw(st.integers(0, 10_000)))
    cu_q = np.concatenate([[0], np.cumsum(lq)]).astype(np.int32)
    cu_k = np.concatenate([[0], np.cumsum(lk)]).astype(np.int32)
    c = dict(q=rng.standard_normal((int(cu_q[-1]), Hq, D)),
             k=rng.standard_normal((int(cu_k[-1]), hkv, D)),
             v=rng.standard_normal((int(cu_k[-1]), hkv, D)),
             dout=rng.standard_normal((int(cu_q[-1]), Hq, D)),
             cu_q=cu_q, cu_k=cu_k, Hq=Hq, Hkv=hkv, scale=0.41, causal=causal,
             bk=None, bp=None, strides=None)
    if with_bias:
        R, C = max(max(lq), 1), max(lk)
        c["bk"] = rng.standard_normal((int(cu_k[-1]), Hq)) * 0.5
        c["bp"] = rng.standard_normal((B, Hq, R, C))
        c["strides"] = (Hq * R * C, R * C, C, 1)
    g = _grads(c)
    h = 1e-5
    for name, key in (("q", "dq"), ("k", "dk"), ("v", "dv")) + ((("bk", "dbias_key"),) if with_bias else ()):
        x = c[name]
        idx = tuple(int(rng.integers(0, s)) for s in x.shape)
        xp = x.copy(); xp[idx] += h
        xm = x.copy(); xm[idx] -= h
        fd = (_loss(c, **{name: xp}) - _loss(c, **{name: xm})) / (2 * h)
        assert abs(g[key][idx] - fd) <= 1e-6 * (1 + abs(fd)), (name, idx, g[key][idx], fd)
