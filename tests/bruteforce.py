"""Brute-force padded attention with an explicit mask (numpy, fp64).

Independent of the oracle: it pads the packed stream into [B, H, maxL, D],
repeats each K/V head G times, builds the boolean mask [B, maxLq, maxLk]
(in-sequence and bottom-right causal) and the bias grid element by element,
and runs textbook softmax attention with matrix products. Used only to pin
the oracle on tiny inputs.
"""
import numpy as np
import torch


def _f64(x):
    if isinstance(x, torch.Tensor):
        return x.detach().to(torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def padded_attention(q, k, v, cu_q, cu_k, n_heads, n_kv_heads, scale, causal,
                     bias_key=None, bias_pair=None, bias_strides=(0, 0, 0, 0)):
    q, k, v = _f64(q), _f64(k), _f64(v)
    cu_q = [int(x) for x in cu_q]
    cu_k = [int(x) for x in cu_k]
    B = len(cu_q) - 1
    D = q.shape[-1]
    G = n_heads // n_kv_heads
    Lq = [cu_q[i + 1] - cu_q[i] for i in range(B)]
    Lk = [cu_k[i + 1] - cu_k[i] for i in range(B)]
    mq, mk = max(Lq + [1]), max(Lk + [1])
    Qp = np.zeros((B, n_heads, mq, D))
    Kp = np.zeros((B, n_heads, mk, D))
    Vp = np.zeros((B, n_heads, mk, D))
    for i in range(B):
        Qp[i, :, :Lq[i]] = q[cu_q[i]:cu_q[i + 1]].transpose(1, 0, 2)
        kk = np.repeat(k[cu_k[i]:cu_k[i + 1]].transpose(1, 0, 2), G, axis=0)
        vv = np.repeat(v[cu_k[i]:cu_k[i + 1]].transpose(1, 0, 2), G, axis=0)
        Kp[i, :, :Lk[i]] = kk
        Vp[i, :, :Lk[i]] = vv
    mask = np.zeros((B, mq, mk), dtype=bool)
    for i in range(B):
        rr = np.arange(mq)[:, None]
        cc = np.arange(mk)[None, :]
        m = (rr < Lq[i]) & (cc < Lk[i])
        if causal:
            m &= cc - rr <= Lk[i] - Lq[i]
        mask[i] = m
    S = scale * np.einsum("bhrd,bhcd->bhrc", Qp, Kp)
    if bias_key is not None:
        bk = _f64(bias_key)
        for i in range(B):
            S[i, :, :, :Lk[i]] += bk[cu_k[i]:cu_k[i + 1]].T[:, None, :]
    if bias_pair is not None:
        flat = _f64(bias_pair).reshape(-1)
        sb, sh, sr, sc = bias_strides
        for i in range(B):
            for h in range(n_heads):
                for r in range(Lq[i]):
                    for c in range(Lk[i]):
                        S[i, h, r, c] += flat[i * sb + h * sh + r * sr + c * sc]
    S = np.where(mask[:, None], S, -np.inf)
    mx = S.max(axis=-1, keepdims=True)
    empty = ~np.isfinite(mx)
    mx = np.where(empty, 0.0, mx)
    E = np.exp(S - mx)
    Z = E.sum(axis=-1, keepdims=True)
    P = np.where(empty, 0.0, E / np.where(Z == 0, 1.0, Z))
    O = np.einsum("bhrc,bhcd->bhrd", P, Vp)
    L = np.where(empty[..., 0], -np.inf, mx[..., 0] + np.log(np.where(Z[..., 0] == 0, 1.0, Z[..., 0])))
    Tq = cu_q[-1]
    out = np.zeros((Tq, n_heads, D))
    lse = np.zeros((n_heads, Tq))
    for i in range(B):
        out[cu_q[i]:cu_q[i + 1]] = O[i, :, :Lq[i]].transpose(1, 0, 2)
        lse[:, cu_q[i]:cu_q[i + 1]] = L[i, :, :Lq[i]]
    return out, lse
