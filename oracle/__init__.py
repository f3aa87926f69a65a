"""CPU oracle for packed variable-length attention forward (TEST INFRASTRUCTURE).

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The product path (the CUDA library and
its Python binding) never imports, links or calls it, and this package never
imports the product.

The arithmetic lives in ``varlen_attn_oracle.c`` (plain C, fp64, OpenMP over
(sequence, head)); this module only compiles it with gcc and marshals numpy /
torch CPU arrays into it. What it computes, with the pages each step follows,
is written at the top of the C file.

Functions
---------
``fwd``    full forward: O [Tq, Hq, D] fp64 and LSE [Hq, Tq] fp64.
``rows``   the same for a list of (sequence, head, local row) samples.
``probs``  the softmax probability matrix of one (sequence, head).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "varlen_attn_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

BF16, F32, F64 = 0, 1, 2

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/liboracle.so`` (gcc, -O2, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-fopenmp", "-std=c99", "-Wall", "-shared", "-fPIC",
               _SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        vp, i32, i64, dbl = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_double
        common = [vp, vp, vp, i32, vp, vp, i32, i32, i32, i32, dbl, i32, vp, vp, i32,
                  i64, i64, i64, i64]
        lib.oracle_varlen_attn_fwd.argtypes = common + [vp, vp, i32]
        lib.oracle_varlen_attn_fwd.restype = i32
        lib.oracle_varlen_attn_rows.argtypes = common + [i64, vp, vp, vp, vp, vp, i32]
        lib.oracle_varlen_attn_rows.restype = i32
        lib.oracle_varlen_attn_probs.argtypes = common + [i32, i32, vp]
        lib.oracle_varlen_attn_probs.restype = i32
        _lib = lib
    return _lib


def default_threads() -> int:
    return len(os.sched_getaffinity(0))


def _as_np(x):
    """torch CPU tensor or numpy array -> contiguous numpy array (bf16 kept as raw bits)."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().contiguous()
            if x.dtype == torch.bfloat16:
                return x.view(torch.int16).numpy().view(np.uint16), BF16
            x = x.numpy()
    except ImportError:  # pragma: no cover
        pass
    x = np.ascontiguousarray(x)
    if x.dtype == np.uint16:
        return x, BF16
    if x.dtype == np.float32:
        return x, F32
    if x.dtype == np.float64:
        return x, F64
    raise TypeError(f"unsupported oracle element type {x.dtype}")


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


class _Args:
    """Marshalled common arguments; keeps the numpy buffers alive."""

    def __init__(self, q, k, v, cu_q, cu_k, n_heads, n_kv_heads, scale, causal,
                 bias_key, bias_pair, bias_strides):
        self.q, dq = _as_np(q)
        self.k, dk = _as_np(k)
        self.v, dv = _as_np(v)
        if not (dq == dk == dv):
            raise TypeError("q, k, v must share one element type")
        self.qkv_dtype = dq
        self.cu_q = np.ascontiguousarray(np.asarray(cu_q, dtype=np.int32))
        self.cu_k = np.ascontiguousarray(np.asarray(cu_k, dtype=np.int32))
        self.batch = len(self.cu_q) - 1
        self.head_dim = self.q.shape[-1]
        self.n_heads = int(n_heads)
        self.n_kv_heads = int(n_kv_heads)
        self.bias_dtype = F32
        self.bias_key = None
        self.bias_pair = None
        if bias_key is not None:
            self.bias_key, self.bias_dtype = _as_np(bias_key)
        if bias_pair is not None:
            self.bias_pair, bd = _as_np(bias_pair)
            if bias_key is not None and bd != self.bias_dtype:
                raise TypeError("bias_key and bias_pair must share one element type")
            self.bias_dtype = bd
        self.strides = tuple(int(s) for s in (bias_strides or (0, 0, 0, 0)))
        self.scale = float(scale)
        self.causal = int(bool(causal))

    def common(self):
        return (_ptr(self.q), _ptr(self.k), _ptr(self.v), self.qkv_dtype,
                _ptr(self.cu_q), _ptr(self.cu_k), self.batch, self.n_heads, self.n_kv_heads,
                self.head_dim, self.scale, self.causal, _ptr(self.bias_key),
                _ptr(self.bias_pair), self.bias_dtype, *self.strides)


def fwd(q, k, v, cu_q, cu_k, n_heads, n_kv_heads, scale, causal, bias_key=None,
        bias_pair=None, bias_strides=None, threads=None):
    """Full oracle forward. Returns (out [Tq,Hq,D] fp64, lse [Hq,Tq] fp64).

    ``q`` [Tq,Hq,D], ``k``/``v`` [Tk,Hkv,D] (bf16 torch tensors, or uint16 bit
    patterns, fp32 or fp64); ``bias_key`` [Tk,Hq]; ``bias_pair`` any buffer
    addressed through ``bias_strides`` = (sb, sh, sr, sc) in elements.
    """
    a = _Args(q, k, v, cu_q, cu_k, n_heads, n_kv_heads, scale, causal, bias_key, bias_pair,
              bias_strides)
    Tq = int(a.cu_q[-1])
    out = np.zeros((Tq, a.n_heads, a.head_dim), dtype=np.float64)
    lse = np.zeros((a.n_heads, Tq), dtype=np.float64)
    rc = _load().oracle_varlen_attn_fwd(*a.common(), _ptr(out), _ptr(lse),
                                        threads or default_threads())
    if rc != 0:
        raise ValueError(f"oracle rejected its arguments (code {rc})")
    return out, lse


def rows(q, k, v, cu_q, cu_k, n_heads, n_kv_heads, scale, causal, seq, head, row,
         bias_key=None, bias_pair=None, bias_strides=None, threads=None):
    """Oracle output rows for samples (seq[n], head[n], local row[n]).

    Returns (out [N, D] fp64, lse [N] fp64)."""
    a = _Args(q, k, v, cu_q, cu_k, n_heads, n_kv_heads, scale, causal, bias_key, bias_pair,
              bias_strides)
    seq = np.ascontiguousarray(np.asarray(seq, dtype=np.int32))
    head = np.ascontiguousarray(np.asarray(head, dtype=np.int32))
    row = np.ascontiguousarray(np.asarray(row, dtype=np.int32))
    n = len(seq)
    out = np.zeros((n, a.head_dim), dtype=np.float64)
    lse = np.zeros((n,), dtype=np.float64)
    rc = _load().oracle_varlen_attn_rows(*a.common(), n, _ptr(seq), _ptr(head), _ptr(row),
                                         _ptr(out), _ptr(lse), threads or default_threads())
    if rc != 0:
        raise ValueError(f"oracle rejected its arguments (code {rc})")
    return out, lse


def probs(q, k, v, cu_q, cu_k, n_heads, n_kv_heads, scale, causal, i, h, bias_key=None,
          bias_pair=None, bias_strides=None):
    """Softmax probability matrix [Lq_i, Lk_i] of sequence ``i``, head ``h``."""
    a = _Args(q, k, v, cu_q, cu_k, n_heads, n_kv_heads, scale, causal, bias_key, bias_pair,
              bias_strides)
    lq = int(a.cu_q[i + 1] - a.cu_q[i])
    lk = int(a.cu_k[i + 1] - a.cu_k[i])
    p = np.zeros((lq, lk), dtype=np.float64)
    rc = _load().oracle_varlen_attn_probs(*a.common(), int(i), int(h), _ptr(p))
    if rc != 0:
        raise ValueError(f"oracle rejected its arguments (code {rc})")
    return p
