"""CPU oracle for the backward pass of packed variable-length attention
(TEST INFRASTRUCTURE: only tests/, the smoke check and bench.py's CPU leg may
import it; it never imports the product).

What it computes, per sequence i and query head h (K/V head kvh = h / G):
with P the softmax probabilities of the forward pass (taken from the
forward oracle, ``oracle.probs``: scores scale·QKᵀ + biases, visible keys
only, rows without a visible key all zero) and dO the gradient of the loss
with respect to the output O = P V,

    dV[kvh]  += Pᵀ dO                      (summed over the G heads of the group)
    dP        = dO Vᵀ
    dS        = P ∘ (dP − rowsum(P ∘ dP))  (the softmax Jacobian applied to dP)
    dQ[h]     = scale · dS K
    dK[kvh]  += scale · dSᵀ Q
    dbias_key[c, h]        = Σ_r dS[r, c]  (the per-key bias enters every row)
    dbias_pair[i, h, r, c] = dS[r, c]

This is the chain rule through the forward definition: the gradients that
the TorchEasyRec PR 663 page (GenRec, "Test plan") checks for the packed path,
that the ASpec PR 25 page ("Verification") bounds against a dense math backend
(Q/K/V relative L2 error under 1%), and that the GiGL PR 858 page
("Approach") lists as missing for a per-sequence bias. It is written as
plain per-(sequence, head) fp64 matrix products, with no tiling or
recomputation. Its pins (tests/test_oracle_backward_pins.py) are central
finite differences of the forward oracle and invariants of the softmax
Jacobian, not this code.
"""
from __future__ import annotations

import numpy as np

from . import _as_np, BF16, probs


def _widen(x):
    a, t = _as_np(x)
    if t == BF16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def bwd(q, k, v, dout, cu_q, cu_k, n_heads, n_kv_heads, scale, causal, bias_key=None,
        bias_pair=None, bias_strides=None):
    """Gradients of sum(dout * O) with respect to q, k, v and the biases.

    Returns a dict with ``dq`` [Tq,Hq,D], ``dk``/``dv`` [Tk,Hkv,D],
    ``dbias_key`` [Tk,Hq] and ``dbias_pair`` [B,Hq,maxLq,maxLk] (entries
    outside a sequence are 0), all fp64.
    """
    Q, K, V, dO = _widen(q), _widen(k), _widen(v), _widen(dout)
    cu_q = np.asarray(cu_q, dtype=np.int64)
    cu_k = np.asarray(cu_k, dtype=np.int64)
    B = len(cu_q) - 1
    Hq, Hkv = int(n_heads), int(n_kv_heads)
    G = Hq // Hkv
    Tq, Tk, D = Q.shape[0], K.shape[0], Q.shape[2]
    lq = np.diff(cu_q)
    lk = np.diff(cu_k)
    dq = np.zeros((Tq, Hq, D))
    dk = np.zeros((Tk, Hkv, D))
    dv = np.zeros((Tk, Hkv, D))
    dbk = np.zeros((Tk, Hq))
    dbp = np.zeros((B, Hq, int(lq.max(initial=0)), int(lk.max(initial=0))))
    for i in range(B):
        q0, k0, Lq, Lk = int(cu_q[i]), int(cu_k[i]), int(lq[i]), int(lk[i])
        if Lq == 0:
            continue
        for h in range(Hq):
            kvh = h // G
            P = probs(q, k, v, cu_q, cu_k, Hq, Hkv, scale, causal, i, h, bias_key=bias_key,
                      bias_pair=bias_pair, bias_strides=bias_strides)
            Qh = Q[q0:q0 + Lq, h, :]
            Kh = K[k0:k0 + Lk, kvh, :]
            Vh = V[k0:k0 + Lk, kvh, :]
            dOh = dO[q0:q0 + Lq, h, :]
            dv[k0:k0 + Lk, kvh, :] += P.T @ dOh
            dP = dOh @ Vh.T
            dS = P * (dP - (P * dP).sum(axis=1, keepdims=True))
            dq[q0:q0 + Lq, h, :] = scale * (dS @ Kh)
            dk[k0:k0 + Lk, kvh, :] += scale * (dS.T @ Qh)
            dbk[k0:k0 + Lk, h] = dS.sum(axis=0)
            dbp[i, h, :Lq, :Lk] = dS
    return {"dq": dq, "dk": dk, "dv": dv, "dbias_key": dbk, "dbias_pair": dbp}
