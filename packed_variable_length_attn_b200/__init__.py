"""Packed variable-length attention for NVIDIA B200 (sm_100a).

Thin Python binding over the C ABI of ``libvarlen_attn.so`` (declared in
``include/varlen_attn.h``). This module only checks and marshals arguments:
every step of the computation runs in the library's CUDA kernels. PyTorch
provides device memory and the current stream. There is no fallback: if the
library is missing or the device is not sm_100, calls raise.

    out, lse = varlen_attn_fwd(q, k, v, cu_seqlens_q, cu_seqlens_k,
                               max_seqlen_q, max_seqlen_k, causal=True)

``q`` is ``[total_q, n_heads, head_dim]``, ``k``/``v`` are
``[total_k, n_kv_heads, head_dim]`` (bf16, or fp32 for the fp32 path),
``cu_seqlens_*`` are int32 ``[batch + 1]`` on the same device. ``out`` has
q's shape and dtype; ``lse`` is fp32 ``[n_heads, total_q]``.

Also: ``varlen_attn_bwd`` (gradients of q, k, v and the biases from the
forward's ``out`` and ``lse`` and the output gradient), ``varlen_attn_decode``
(a decode step over a per-sequence K/V cache), ``unpad`` / ``pad`` /
``mask_to_seqlens`` / ``gather_rows`` / ``scatter_rows`` (packed-layout
helpers) and ``fold_pair_bias_row`` (first-token bias fold).

    dq, dk, dv, _, _ = varlen_attn_bwd(q, k, v, out, lse, dout, cu_seqlens_q,
                                       cu_seqlens_k, max_seqlen_q, max_seqlen_k,
                                       causal=True)

``varlen_attn`` wraps the two in a ``torch.autograd.Function`` for training
loops (bf16; gradients for q, k, v and the biases that require them).
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional, Sequence, Tuple

__all__ = ["varlen_attn_fwd", "varlen_attn_fwd_noalloc", "library_path", "load_library", "VarlenAttnError",
           "get_device_error", "set_profile_events", "launches_per_call", "exported_symbols",
           "mask_to_seqlens", "gather_rows", "scatter_rows", "unpad", "pad", "fold_pair_bias_row",
           "varlen_attn_decode", "varlen_attn_bwd", "set_wait_limit", "set_test_stall",
           "BIAS_PAIR_KV_HEADS", "varlen_attn"]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libvarlen_attn.so")
_lib = None

# Status codes and flags of include/varlen_attn.h
BIAS_PAIR_KV_HEADS = 1
OK = 0
ERR_BAD_SEQLENS = 9
ERR_DEVICE_TIMEOUT = 10


class VarlenAttnError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"varlen_attn error {status}: {message}")
        self.status = status


def library_path() -> str:
    return _LIB_PATH


def exported_symbols() -> Tuple[str, ...]:
    return ("varlen_attn_fwd", "varlen_attn_fwd_f32", "varlen_attn_strerror",
            "varlen_attn_get_device_error", "varlen_attn_set_profile_events",
            "varlen_attn_launches_per_call", "varlen_attn_version",
            "varlen_attn_last_error_detail", "varlen_attn_fwd_noalloc", "varlen_attn_fwd_ex",
            "varlen_mask_to_seqlens", "varlen_gather_rows", "varlen_scatter_rows",
            "varlen_fold_pair_bias_row", "varlen_attn_decode", "varlen_attn_bwd",
            "varlen_attn_set_wait_limit", "varlen_attn_set_test_stall")


def load_library():
    """Load libvarlen_attn.so (built by build.py / __graft_entry__.build())."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise ImportError(f"CUDA library not built: {_LIB_PATH} is missing "
                          "(run packed_variable_length_attn_b200/build.py)")
    lib = ctypes.CDLL(_LIB_PATH)
    vp, i32, i64, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float
    fwd_args = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, i32, f32, i32, vp, vp,
                i64, i64, i64, i64, vp, vp, vp]
    lib.varlen_attn_fwd.argtypes = fwd_args
    lib.varlen_attn_fwd.restype = i32
    lib.varlen_attn_fwd_f32.argtypes = fwd_args
    lib.varlen_attn_fwd_f32.restype = i32
    lib.varlen_attn_fwd_noalloc.argtypes = fwd_args
    lib.varlen_attn_fwd_noalloc.restype = i32
    lib.varlen_attn_fwd_ex.argtypes = fwd_args[:21] + [ctypes.c_uint] + fwd_args[21:]
    lib.varlen_attn_fwd_ex.restype = i32
    lib.varlen_mask_to_seqlens.argtypes = [vp, i32, i32, vp, vp, vp, vp]
    lib.varlen_mask_to_seqlens.restype = i32
    lib.varlen_gather_rows.argtypes = [vp, i64, i64, vp, vp, i32, vp, i64, vp]
    lib.varlen_gather_rows.restype = i32
    lib.varlen_scatter_rows.argtypes = [vp, i64, i64, vp, vp, i32, vp, i64, vp]
    lib.varlen_scatter_rows.restype = i32
    lib.varlen_fold_pair_bias_row.argtypes = [vp, i64, i64, i64, i64, i32, i32, vp, i32, i32,
                                              i32, vp, vp, vp]
    lib.varlen_fold_pair_bias_row.restype = i32
    lib.varlen_attn_decode.argtypes = [vp, vp, i32, i32, i32, vp, vp, i32, vp, vp, vp, i32, i32,
                                       i32, f32, i32, i32, vp, vp, vp]
    lib.varlen_attn_decode.restype = i32
    lib.varlen_attn_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32,
                                    i32, i32, ctypes.c_float, i32, vp, vp, i64, i64, i64, i64,
                                    ctypes.c_uint, vp, vp, vp, vp, vp, i64, i64, i64, vp]
    lib.varlen_attn_bwd.restype = i32
    lib.varlen_attn_strerror.argtypes = [i32]
    lib.varlen_attn_strerror.restype = ctypes.c_char_p
    lib.varlen_attn_get_device_error.argtypes = [vp]
    lib.varlen_attn_get_device_error.restype = i32
    lib.varlen_attn_set_profile_events.argtypes = [vp, vp]
    lib.varlen_attn_set_profile_events.restype = i32
    lib.varlen_attn_set_wait_limit.argtypes = [ctypes.c_longlong]
    lib.varlen_attn_set_wait_limit.restype = i32
    lib.varlen_attn_set_test_stall.argtypes = [i32]
    lib.varlen_attn_set_test_stall.restype = i32
    lib.varlen_attn_launches_per_call.argtypes = [i32]
    lib.varlen_attn_launches_per_call.restype = i32
    lib.varlen_attn_version.argtypes = []
    lib.varlen_attn_version.restype = i32
    lib.varlen_attn_last_error_detail.argtypes = []
    lib.varlen_attn_last_error_detail.restype = ctypes.c_char_p
    _lib = lib
    return lib


def strerror(status: int) -> str:
    return load_library().varlen_attn_strerror(int(status)).decode()


def _check(status: int):
    if status != OK:
        msg = strerror(status)
        if status in (7, 12):
            msg += " [" + load_library().varlen_attn_last_error_detail().decode() + "]"
        raise VarlenAttnError(status, msg)


def _stream_handle(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def get_device_error(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device error word."""
    return int(load_library().varlen_attn_get_device_error(_stream_handle(stream)))


def set_profile_events(start=None, stop=None):
    """Record ``start``/``stop`` (torch.cuda.Event) around later attention-kernel
    launches from this thread; ``set_profile_events()`` switches it off."""
    lib = load_library()
    if start is None or stop is None:
        _check(lib.varlen_attn_set_profile_events(None, None))
    else:
        if not start.cuda_event or not stop.cuda_event:
            raise ValueError("record the events once first (torch creates them lazily)")
        _check(lib.varlen_attn_set_profile_events(ctypes.c_void_p(start.cuda_event),
                                                  ctypes.c_void_p(stop.cuda_event)))


def set_wait_limit(cycles: int = 0):
    """Limit, in SM clock cycles, of every bounded barrier wait of the
    tensor-core kernels launched afterwards (process-wide); 0 restores the
    default (2^33). A wait that runs out raises status 10 in the device error
    word and the call's outputs are undefined."""
    _check(load_library().varlen_attn_set_wait_limit(int(cycles)))


def set_test_stall(on: bool = False):
    """Test hook of the abort path: while on, every tensor-core forward and
    backward launch first waits on a barrier phase that nothing completes, so
    the call ends with status 10 after the wait limit. Off by default."""
    _check(load_library().varlen_attn_set_test_stall(1 if on else 0))


def launches_per_call(fp32: bool = False) -> int:
    return int(load_library().varlen_attn_launches_per_call(1 if fp32 else 0))


def _grid_strides(bias_pair, bias_pair_strides: Optional[Sequence[int]]):
    if bias_pair_strides is not None:
        return tuple(int(s) for s in bias_pair_strides)
    if bias_pair.dim() != 4:
        raise ValueError("bias_pair must be 4-D [batch, heads or 1, rows, cols] "
                         "or come with explicit bias_pair_strides")
    sb, sh, sr, sc = bias_pair.stride()
    if bias_pair.shape[1] == 1:
        sh = 0
    return (sb, sh, sr, sc)


def varlen_attn_fwd(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q: int, max_seqlen_k: int,
                    softmax_scale: Optional[float] = None, causal: bool = False,
                    bias_per_key=None, bias_pair=None, bias_pair_strides=None,
                    out=None, lse=None, return_lse: bool = True, stream=None,
                    bias_pair_kv_heads: bool = False):
    """Packed variable-length attention forward through the C ABI.

    bf16 q/k/v run the tensor-core kernel; fp32 q/k/v run the fp32 kernel.
    ``bias_per_key``: fp32 ``[total_k, n_heads]``. ``bias_pair``: fp32 grid
    read at ``i*sb + h*sh + r*sq + c*sk``; strides default to the tensor's own
    (a 4-D ``[B, 1 or H, R, C]`` view, permuted views included; a size-1 head
    axis broadcasts). ``bias_pair_kv_heads``: the grid is per K/V head
    (``[B, n_kv_heads, R, C]``; query head h reads grid head h // G; bf16 only).
    Returns ``(out, lse)`` (``lse`` None if not requested).
    """
    import torch
    lib = load_library()
    if q.dim() != 3 or k.dim() != 3 or v.dim() != 3:
        raise ValueError("q, k, v must be [tokens, heads, head_dim]")
    if q.dtype not in (torch.bfloat16, torch.float32) or k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("q, k, v must all be bf16 or all fp32")
    tensors = [q, k, v, cu_seqlens_q, cu_seqlens_k]
    for t in (bias_per_key, bias_pair, out, lse):
        if t is not None:
            tensors.append(t)
    dev = q.device
    if dev.type != "cuda" or any(t.device != dev for t in tensors):
        raise ValueError("all tensors must be on the same CUDA device")
    for name, t in (("q", q), ("k", k), ("v", v), ("cu_seqlens_q", cu_seqlens_q),
                    ("cu_seqlens_k", cu_seqlens_k)):
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    if cu_seqlens_q.dtype != torch.int32 or cu_seqlens_k.dtype != torch.int32:
        raise ValueError("cu_seqlens must be int32")
    if cu_seqlens_q.numel() != cu_seqlens_k.numel() or cu_seqlens_q.numel() < 2:
        raise ValueError("cu_seqlens_q and cu_seqlens_k must both have batch + 1 entries")
    total_q, n_heads, head_dim = q.shape
    total_k, n_kv_heads, dk = k.shape
    if v.shape != k.shape or dk != head_dim:
        raise ValueError("k and v must be [total_k, n_kv_heads, head_dim] like q's head_dim")
    batch = cu_seqlens_q.numel() - 1
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(head_dim)
    if bias_per_key is not None:
        if bias_per_key.dtype != torch.float32 or not bias_per_key.is_contiguous() or \
                tuple(bias_per_key.shape) != (total_k, n_heads):
            raise ValueError("bias_per_key must be contiguous fp32 [total_k, n_heads]")
    strides = (0, 0, 0, 0)
    if bias_pair is not None:
        if bias_pair.dtype != torch.float32:
            raise ValueError("bias_pair must be fp32")
        strides = _grid_strides(bias_pair, bias_pair_strides)
    if out is None:
        out = torch.empty_like(q)
    elif out.shape != q.shape or out.dtype != q.dtype or not out.is_contiguous():
        raise ValueError("out must be contiguous with q's shape and dtype")
    if lse is None and return_lse:
        lse = torch.empty((n_heads, total_q), dtype=torch.float32, device=dev)
    elif lse is not None and (lse.shape != (n_heads, total_q) or lse.dtype != torch.float32
                              or not lse.is_contiguous()):
        raise ValueError("lse must be contiguous fp32 [n_heads, total_q]")
    ptr = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    args = (ptr(q), ptr(k), ptr(v), ptr(cu_seqlens_q), ptr(cu_seqlens_k), batch, total_q,
            total_k, int(max_seqlen_q), int(max_seqlen_k), n_heads, n_kv_heads, head_dim,
            float(softmax_scale), 1 if causal else 0, ptr(bias_per_key), ptr(bias_pair), *strides)
    tail = (ptr(out), ptr(lse), _stream_handle(stream))
    with torch.cuda.device(dev):
        if bias_pair_kv_heads:
            if q.dtype != torch.bfloat16:
                raise ValueError("bias_pair_kv_heads is a bf16-path option")
            status = lib.varlen_attn_fwd_ex(*args, BIAS_PAIR_KV_HEADS, *tail)
        elif q.dtype == torch.bfloat16:
            status = lib.varlen_attn_fwd(*args, *tail)
        else:
            status = lib.varlen_attn_fwd_f32(*args, *tail)
    _check(status)
    return out, lse


def varlen_attn_fwd_noalloc(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q: int,
                            max_seqlen_k: int, out, lse, softmax_scale: Optional[float] = None,
                            causal: bool = False, bias_per_key=None, bias_pair=None,
                            bias_pair_strides=None, stream=None):
    """The same forward through ``varlen_attn_fwd_noalloc``: no device memory is
    allocated, neither by the library (its work list sits in a fixed array of
    the library, limited to 16384 (sequence, q-block group) pairs) nor here
    (``out`` and ``lse`` must be given). For callers whose device memory is
    managed elsewhere and must not be allocated behind their back. Calls that
    can run concurrently on one device share that array and must be ordered.
    bf16 only."""
    import torch
    lib = load_library()
    if q.dtype != torch.bfloat16 or k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("varlen_attn_fwd_noalloc takes bf16 q, k, v")
    total_q, n_heads, head_dim = q.shape
    total_k, n_kv_heads, _ = k.shape
    if out is None or lse is None:
        raise ValueError("out and lse must be provided (this path allocates nothing)")
    if out.shape != q.shape or out.dtype != q.dtype or not out.is_contiguous():
        raise ValueError("out must be contiguous with q's shape and dtype")
    if lse.shape != (n_heads, total_q) or lse.dtype != torch.float32 or not lse.is_contiguous():
        raise ValueError("lse must be contiguous fp32 [n_heads, total_q]")
    for name, t in (("q", q), ("k", k), ("v", v), ("cu_seqlens_q", cu_seqlens_q),
                    ("cu_seqlens_k", cu_seqlens_k)):
        if not t.is_contiguous() or t.device != q.device:
            raise ValueError(f"{name} must be contiguous and on q's device")
    batch = cu_seqlens_q.numel() - 1
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(head_dim)
    strides = (0, 0, 0, 0) if bias_pair is None else _grid_strides(bias_pair, bias_pair_strides)
    ptr = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    with torch.cuda.device(q.device):
        status = lib.varlen_attn_fwd_noalloc(
            ptr(q), ptr(k), ptr(v), ptr(cu_seqlens_q), ptr(cu_seqlens_k), batch, total_q,
            total_k, int(max_seqlen_q), int(max_seqlen_k), n_heads, n_kv_heads, head_dim,
            float(softmax_scale), 1 if causal else 0, ptr(bias_per_key), ptr(bias_pair),
            *strides, ptr(out), ptr(lse), _stream_handle(stream))
    _check(status)
    return out, lse


# ----------------------------------------------------------------------------- layout helpers

def _dev_ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def mask_to_seqlens(mask, stream=None):
    """Unpadding metadata from a [batch, seqlen] validity mask (bool or uint8,
    CUDA, contiguous): ``(cu_seqlens [B+1], indices [B*S], max_seqlen [1])``,
    int32 device tensors; the first ``cu_seqlens[-1]`` indices are the flat
    padded positions of the packed rows. Nothing is read back to the host."""
    import torch
    if mask.dim() != 2 or mask.device.type != "cuda":
        raise ValueError("mask must be a 2-D CUDA tensor [batch, seqlen]")
    m = mask.to(torch.uint8).contiguous()
    B, S = m.shape
    cu = torch.empty(B + 1, dtype=torch.int32, device=m.device)
    idx = torch.empty(B * S, dtype=torch.int32, device=m.device)
    mx = torch.empty(1, dtype=torch.int32, device=m.device)
    with torch.cuda.device(m.device):
        _check(load_library().varlen_mask_to_seqlens(_dev_ptr(m), B, S, _dev_ptr(cu),
                                                     _dev_ptr(idx), _dev_ptr(mx),
                                                     _stream_handle(stream)))
    return cu, idx, mx


def _rows_view(t):
    if not t.is_contiguous() or t.dim() < 1:
        raise ValueError("row tensors must be contiguous")
    row_bytes = t.element_size() * (t.numel() // max(1, t.shape[0])) if t.shape[0] else 0
    return t.shape[0], row_bytes


def gather_rows(src, indices, cu_seqlens, out, stream=None):
    """out[t] = src[indices[t]] for t < cu_seqlens[-1] (rows = first dimension;
    row size a multiple of 16 bytes)."""
    import torch
    n_src, rb = _rows_view(src)
    n_dst, rb2 = _rows_view(out)
    if rb != rb2 or src.dtype != out.dtype:
        raise ValueError("src and out rows must match in size and dtype")
    with torch.cuda.device(src.device):
        _check(load_library().varlen_gather_rows(
            _dev_ptr(src), n_src, rb, _dev_ptr(indices), _dev_ptr(cu_seqlens),
            cu_seqlens.numel() - 1, _dev_ptr(out), n_dst, _stream_handle(stream)))
    return out


def scatter_rows(src, indices, cu_seqlens, out, stream=None):
    """out = 0, then out[indices[t]] = src[t] for t < cu_seqlens[-1]."""
    import torch
    n_src, rb = _rows_view(src)
    n_dst, rb2 = _rows_view(out)
    if rb != rb2 or src.dtype != out.dtype:
        raise ValueError("src and out rows must match in size and dtype")
    with torch.cuda.device(src.device):
        _check(load_library().varlen_scatter_rows(
            _dev_ptr(src), n_src, rb, _dev_ptr(indices), _dev_ptr(cu_seqlens),
            cu_seqlens.numel() - 1, _dev_ptr(out), n_dst, _stream_handle(stream)))
    return out


def unpad(x, mask, stream=None):
    """Padded ``x [B, S, ...]`` + mask ``[B, S]`` -> ``(packed [T, ...], indices,
    cu_seqlens, max_seqlen)``. Sizing the packed tensor reads T back to the host
    (one synchronisation), as the padded-to-packed conversion of the
    FlashAttention pipeline does."""
    import torch
    B, S = mask.shape
    cu, idx, mx = mask_to_seqlens(mask, stream)
    T = int(cu[-1].item())
    packed = torch.empty((T,) + tuple(x.shape[2:]), dtype=x.dtype, device=x.device)
    if T:
        gather_rows(x.reshape((B * S,) + tuple(x.shape[2:])), idx, cu, packed, stream)
    return packed, idx[:T], cu, int(mx.item())


def pad(packed, indices, cu_seqlens, batch, seqlen, stream=None):
    """Packed ``[T, ...]`` -> padded ``[batch, seqlen, ...]`` (zeros elsewhere)."""
    import torch
    out = torch.empty((batch * seqlen,) + tuple(packed.shape[1:]), dtype=packed.dtype,
                      device=packed.device)
    scatter_rows(packed, indices, cu_seqlens, out, stream)
    return out.reshape((batch, seqlen) + tuple(packed.shape[1:]))


def fold_pair_bias_row(bias_pair, cu_seqlens_k, n_heads, total_k, row=0, head_div=1,
                       bias_pair_strides=None, bias_in=None, out=None, stream=None):
    """Per-key bias ``[total_k, n_heads]`` = ``bias_in`` (or 0) + row ``row`` of
    the per-pair grid (first-token fold; ``head_div`` = G for a grid over K/V
    heads)."""
    import torch
    strides = _grid_strides(bias_pair, bias_pair_strides)
    if out is None:
        out = torch.empty((total_k, n_heads), dtype=torch.float32, device=bias_pair.device)
    with torch.cuda.device(bias_pair.device):
        _check(load_library().varlen_fold_pair_bias_row(
            _dev_ptr(bias_pair), *strides, int(row), int(head_div), _dev_ptr(cu_seqlens_k),
            cu_seqlens_k.numel() - 1, int(total_k), int(n_heads),
            None if bias_in is None else _dev_ptr(bias_in), _dev_ptr(out),
            _stream_handle(stream)))
    return out


def varlen_attn_bwd(q, k, v, out, lse, dout, cu_seqlens_q, cu_seqlens_k, max_seqlen_q: int,
                    max_seqlen_k: int, softmax_scale: Optional[float] = None,
                    causal: bool = False, bias_per_key=None, bias_pair=None,
                    bias_pair_strides=None, bias_pair_kv_heads: bool = False,
                    need_dbias_per_key: bool = False, need_dbias_pair: bool = False,
                    dq=None, dk=None, dv=None, stream=None):
    """Backward of ``varlen_attn_fwd`` (bf16) through the C ABI.

    ``out`` and ``lse`` are the forward's results for the same arguments,
    ``dout`` the gradient of the loss w.r.t. ``out``. Returns
    ``(dq, dk, dv, dbias_per_key, dbias_pair)``: ``dq`` like q, ``dk``/``dv``
    like k/v (bf16); ``dbias_per_key`` fp32 ``[total_k, n_heads]`` when
    requested; ``dbias_pair`` fp32 ``[batch, n_heads, max_seqlen_q,
    max_seqlen_k]`` per query head when requested (zeros outside the
    sequences; sum over the heads that share a broadcast or per-K/V-head
    grid for that grid's gradient). Unrequested ones are None.
    """
    import torch
    lib = load_library()
    for name, t in (("q", q), ("k", k), ("v", v), ("out", out), ("dout", dout)):
        if t.dim() != 3 or t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous bf16 [tokens, heads, head_dim] tensor")
    if out.shape != q.shape or dout.shape != q.shape or v.shape != k.shape:
        raise ValueError("out and dout must have q's shape, v k's shape")
    dev = q.device
    tensors = [q, k, v, out, lse, dout, cu_seqlens_q, cu_seqlens_k] + \
        [t for t in (bias_per_key, bias_pair, dq, dk, dv) if t is not None]
    if dev.type != "cuda" or any(t.device != dev for t in tensors):
        raise ValueError("all tensors must be on the same CUDA device")
    if cu_seqlens_q.dtype != torch.int32 or cu_seqlens_k.dtype != torch.int32 or \
            not cu_seqlens_q.is_contiguous() or not cu_seqlens_k.is_contiguous():
        raise ValueError("cu_seqlens must be contiguous int32")
    if cu_seqlens_q.numel() != cu_seqlens_k.numel() or cu_seqlens_q.numel() < 2:
        raise ValueError("cu_seqlens_q and cu_seqlens_k must both have batch + 1 entries")
    total_q, n_heads, head_dim = q.shape
    total_k, n_kv_heads, _ = k.shape
    batch = cu_seqlens_q.numel() - 1
    if lse.shape != (n_heads, total_q) or lse.dtype != torch.float32 or not lse.is_contiguous():
        raise ValueError("lse must be contiguous fp32 [n_heads, total_q]")
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(head_dim)
    if bias_per_key is not None and (bias_per_key.dtype != torch.float32 or
                                     not bias_per_key.is_contiguous() or
                                     tuple(bias_per_key.shape) != (total_k, n_heads)):
        raise ValueError("bias_per_key must be contiguous fp32 [total_k, n_heads]")
    strides = (0, 0, 0, 0)
    if bias_pair is not None:
        if bias_pair.dtype != torch.float32:
            raise ValueError("bias_pair must be fp32")
        strides = _grid_strides(bias_pair, bias_pair_strides)
    for name, t, ref in (("dq", dq, q), ("dk", dk, k), ("dv", dv, v)):
        if t is not None and (t.shape != ref.shape or t.dtype != torch.bfloat16 or
                              not t.is_contiguous()):
            raise ValueError(f"{name} must be contiguous bf16 with the shape of its input")
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    dbk = torch.empty((total_k, n_heads), dtype=torch.float32, device=dev) \
        if need_dbias_per_key else None
    dbp = None
    dstr = (0, 0, 0)
    if need_dbias_pair:
        dbp = torch.zeros((batch, n_heads, max(int(max_seqlen_q), 1), max(int(max_seqlen_k), 1)),
                          dtype=torch.float32, device=dev)
        dstr = dbp.stride()[:3]
    ptr = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    flags = BIAS_PAIR_KV_HEADS if bias_pair_kv_heads else 0
    with torch.cuda.device(dev):
        status = lib.varlen_attn_bwd(
            ptr(q), ptr(k), ptr(v), ptr(out), ptr(lse), ptr(dout), ptr(cu_seqlens_q),
            ptr(cu_seqlens_k), batch, total_q, total_k, int(max_seqlen_q), int(max_seqlen_k),
            n_heads, n_kv_heads, head_dim, float(softmax_scale), 1 if causal else 0,
            ptr(bias_per_key), ptr(bias_pair), *strides, flags, ptr(dq), ptr(dk), ptr(dv),
            ptr(dbk), ptr(dbp), *dstr, _stream_handle(stream))
    _check(status)
    return dq, dk, dv, dbk, dbp


def varlen_attn_decode(q, cu_seqlens_q, max_seqlen_q: int, k_cache, v_cache, cache_seqlens,
                       k_new=None, v_new=None, softmax_scale: Optional[float] = None,
                       causal: bool = True, num_splits: int = 0, out=None, lse=None,
                       return_lse: bool = True, stream=None):
    """Decode attention over a K/V cache ``[batch, cache_len, n_kv_heads, D]``
    (bf16). ``k_new``/``v_new`` ``[total_q, n_kv_heads, D]`` are written into
    the cache after ``cache_seqlens[i]`` rows and attended to. Returns
    ``(out, lse)``."""
    import torch
    lib = load_library()
    if q.dtype != torch.bfloat16 or k_cache.dtype != q.dtype or v_cache.dtype != q.dtype:
        raise ValueError("q and the cache must be bf16")
    if k_cache.dim() != 4 or v_cache.shape != k_cache.shape:
        raise ValueError("k_cache and v_cache must be [batch, cache_len, n_kv_heads, head_dim]")
    for t in (q, k_cache, v_cache, cu_seqlens_q, cache_seqlens):
        if not t.is_contiguous() or t.device != q.device:
            raise ValueError("all tensors must be contiguous and on q's device")
    total_q, n_heads, head_dim = q.shape
    batch, cache_len, n_kv_heads, dk = k_cache.shape
    if dk != head_dim or cu_seqlens_q.numel() != batch + 1 or cache_seqlens.numel() != batch:
        raise ValueError("shapes of q, the cache, cu_seqlens_q and cache_seqlens disagree")
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(head_dim)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and return_lse:
        lse = torch.empty((n_heads, total_q), dtype=torch.float32, device=q.device)
    ptr = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    with torch.cuda.device(q.device):
        status = lib.varlen_attn_decode(
            ptr(q), ptr(cu_seqlens_q), batch, total_q, int(max_seqlen_q), ptr(k_cache),
            ptr(v_cache), cache_len, ptr(cache_seqlens), ptr(k_new), ptr(v_new), n_heads,
            n_kv_heads, head_dim, float(softmax_scale), 1 if causal else 0, int(num_splits),
            ptr(out), ptr(lse), _stream_handle(stream))
    _check(status)
    return out, lse


def _autograd_function():
    import torch

    class _VarlenAttn(torch.autograd.Function):
        """Forward and backward both run through the C ABI; this class only
        keeps the forward's output and LSE for the backward and reshapes the
        per-query-head pair-grid gradient to the grid the caller passed."""

        @staticmethod
        def forward(ctx, q, k, v, bias_per_key, bias_pair, cu_seqlens_q, cu_seqlens_k,
                    max_seqlen_q, max_seqlen_k, softmax_scale, causal, bias_pair_kv_heads):
            out, lse = varlen_attn_fwd(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q,
                                       max_seqlen_k, softmax_scale=softmax_scale, causal=causal,
                                       bias_per_key=bias_per_key, bias_pair=bias_pair,
                                       bias_pair_kv_heads=bias_pair_kv_heads)
            ctx.save_for_backward(q, k, v, out, lse, bias_per_key, bias_pair, cu_seqlens_q,
                                  cu_seqlens_k)
            ctx.args = (max_seqlen_q, max_seqlen_k, softmax_scale, causal, bias_pair_kv_heads)
            ctx.mark_non_differentiable(lse)
            return out, lse

        @staticmethod
        def backward(ctx, dout, _dlse):
            q, k, v, out, lse, bk, bp, cu_q, cu_k = ctx.saved_tensors
            max_q, max_k, scale, causal, kv_heads = ctx.args
            need_bk = bk is not None and ctx.needs_input_grad[3]
            need_bp = bp is not None and ctx.needs_input_grad[4]
            dq, dk, dv, dbk, dbp = varlen_attn_bwd(
                q, k, v, out, lse, dout.contiguous(), cu_q, cu_k, max_q, max_k,
                softmax_scale=scale, causal=causal, bias_per_key=bk, bias_pair=bp,
                bias_pair_kv_heads=kv_heads, need_dbias_per_key=need_bk,
                need_dbias_pair=need_bp)
            if need_bp:
                # per query head [B, Hq, max_q, max_k] -> the grid's own heads
                # (a broadcast or per-K/V-head grid sums the heads that read
                # it) and rows / columns (zeros outside the sequences)
                B, Hq, R, C = dbp.shape
                Hg = bp.shape[1]
                dbp = dbp.view(B, Hg, Hq // Hg, R, C).sum(dim=2)
                grad = torch.zeros(bp.shape, dtype=torch.float32, device=bp.device)
                r, c = min(R, bp.shape[2]), min(C, bp.shape[3])
                grad[:, :, :r, :c] = dbp[:, :, :r, :c]
                dbp = grad
            return (dq, dk, dv, dbk if need_bk else None, dbp if need_bp else None,
                    None, None, None, None, None, None, None)

    return _VarlenAttn


_VARLEN_ATTN_FN = None


def varlen_attn(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q: int, max_seqlen_k: int,
                softmax_scale: Optional[float] = None, causal: bool = False, bias_per_key=None,
                bias_pair=None, bias_pair_kv_heads: bool = False):
    """Differentiable packed attention (bf16): ``(out, lse)`` with gradients
    for ``q``, ``k``, ``v``, ``bias_per_key`` and ``bias_pair`` (a 4-D
    ``[batch, 1 | n_heads | n_kv_heads, rows, cols]`` tensor; a head axis of 1
    broadcasts, ``bias_pair_kv_heads`` reads it per K/V head) through
    ``varlen_attn_fwd`` and ``varlen_attn_bwd``."""
    global _VARLEN_ATTN_FN
    if _VARLEN_ATTN_FN is None:
        _VARLEN_ATTN_FN = _autograd_function()
    if bias_pair is not None and bias_pair.dim() != 4:
        raise ValueError("varlen_attn takes bias_pair as a 4-D [batch, heads, rows, cols] tensor")
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(q.shape[-1])
    return _VARLEN_ATTN_FN.apply(q, k, v, bias_per_key, bias_pair, cu_seqlens_q, cu_seqlens_k,
                                 int(max_seqlen_q), int(max_seqlen_k), float(softmax_scale),
                                 bool(causal), bool(bias_pair_kv_heads))
