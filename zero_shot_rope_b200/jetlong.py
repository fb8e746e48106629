"""Thin Python binding of the C ABI in include/jetlong.h (argument marshalling
only: every step of the attention runs in the CUDA library).

The names match the C entry points.  Tensors are torch CUDA tensors; the call
is enqueued on the current torch stream (or ``stream``).  A non-OK status
raises :class:`JetLongError` carrying ``jl_last_error()``.  There is no CPU
fallback: if ``libjetlong.so`` is missing, the first call raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libjetlong.so")

JL_OK, JL_ERR_INVALID_ARG, JL_ERR_UNSUPPORTED, JL_ERR_CUDA, JL_ERR_WORKSPACE = range(5)
JL_BF16, JL_FP32 = 0, 1
JL_FLAG_PLAIN_CAUSAL = 0x1
JL_FLAG_SIMT = 0x2
JL_FLAG_PREROTATE_K = 0x4

_lib = None


class JetLongError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{status_string(status) if _lib else status}: {msg}")
        self.status = status


def lib() -> ctypes.CDLL:
    """Load libjetlong.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"{LIB_PATH} is missing: build it with `python -m zero_shot_rope_b200.build` "
            "(there is no CPU fallback)")
    L = ctypes.CDLL(LIB_PATH)
    c_i32, c_i64, c_u32, c_sz, c_p, c_d = (ctypes.c_int32, ctypes.c_int64, ctypes.c_uint32,
                                           ctypes.c_size_t, ctypes.c_void_p, ctypes.c_double)
    L.jl_status_string.restype = ctypes.c_char_p
    L.jl_status_string.argtypes = [ctypes.c_int]
    L.jl_last_error.restype = ctypes.c_char_p
    L.jl_last_error.argtypes = []
    L.jl_version.restype = ctypes.c_char_p
    L.jl_version.argtypes = []
    L.jl_group_size.restype = ctypes.c_int
    L.jl_group_size.argtypes = [c_i64, c_i64, ctypes.POINTER(c_i64)]
    L.jl_bifocal_prefill_workspace_size.restype = c_sz
    L.jl_bifocal_prefill_workspace_size.argtypes = [c_i32, c_i32, c_i32, c_i32, c_i32, ctypes.c_int, c_u32]
    L.jl_bifocal_prefill.restype = ctypes.c_int
    L.jl_bifocal_prefill.argtypes = [c_p, c_p, c_p, c_p, c_p, c_p, c_i32, c_i32, c_i32, c_i32, c_i32,
                                     c_i32, c_i64, c_i32, c_d, ctypes.c_int, c_u32, c_p, c_sz, c_p]
    L.jl_bifocal_prefill_kv.restype = ctypes.c_int
    L.jl_bifocal_prefill_kv.argtypes = [c_p, c_p, c_p, c_p, c_p, c_p, c_p, c_i32, c_i32, c_i32, c_i32, c_i32,
                                        c_i32, c_i32, c_i64, c_i32, c_i32, c_d, ctypes.c_int, c_u32, c_p, c_sz,
                                        c_p]
    L.jl_bifocal_decode_workspace_size.restype = c_sz
    L.jl_bifocal_decode_workspace_size.argtypes = [c_i32, c_i32, c_i32, c_i32, c_i32]
    L.jl_bifocal_decode.restype = ctypes.c_int
    L.jl_bifocal_decode.argtypes = [c_p, c_p, c_p, c_p, c_i32, c_i32, c_i32, c_i32, c_i32, c_i32, c_i64,
                                    c_i32, c_d, c_p, c_p, c_p, c_sz, ctypes.c_int, c_u32, c_p]
    L.jl_bifocal_decode_window.restype = ctypes.c_int
    L.jl_bifocal_decode_window.argtypes = [c_p, c_p, c_p, c_p, c_i32, c_i32, c_i32, c_i32, c_i32, c_i32, c_i64,
                                           c_i32, c_i32, c_d, c_p, c_p, c_p, c_sz, ctypes.c_int, c_u32, c_p]
    L.jl_bifocal_decode_noalloc.restype = ctypes.c_int
    L.jl_bifocal_decode_noalloc.argtypes = [c_p, c_p, c_p, c_p, c_i32, c_i32, c_i32, c_i32, c_i32, c_i32,
                                            c_i64, c_i32, c_d, c_p, c_p, ctypes.c_int, c_u32, c_p]
    L.jl_bifocal_decode_noalloc_error.restype = ctypes.c_int
    L.jl_bifocal_decode_noalloc_error.argtypes = [ctypes.POINTER(c_i32), c_p]
    L.jl_debug_set_wait_limit.restype = ctypes.c_int
    L.jl_debug_set_wait_limit.argtypes = [ctypes.c_ulonglong]
    _lib = L
    return L


def status_string(s: int) -> str:
    return lib().jl_status_string(int(s)).decode()


def last_error() -> str:
    return lib().jl_last_error().decode()


def _check(status: int):
    if status != JL_OK:
        raise JetLongError(status, last_error())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return JL_BF16
    if t.dtype == torch.float32:
        return JL_FP32
    raise TypeError(f"unsupported dtype {t.dtype}")


def jl_group_size(L: int, w_pretrained: int) -> int:
    g = ctypes.c_int64(0)
    _check(lib().jl_group_size(int(L), int(w_pretrained), ctypes.byref(g)))
    return int(g.value)


def jl_bifocal_prefill_workspace_size(batch, total_tokens, n_q_heads, n_kv_heads, head_dim,
                                      dtype=torch.bfloat16, flags=0) -> int:
    code = JL_BF16 if dtype == torch.bfloat16 else JL_FP32
    return int(lib().jl_bifocal_prefill_workspace_size(batch, total_tokens, n_q_heads, n_kv_heads,
                                                       head_dim, code, flags))


def jl_bifocal_decode_workspace_size(batch, n_q_heads, n_kv_heads, head_dim, max_seqlen) -> int:
    return int(lib().jl_bifocal_decode_workspace_size(batch, n_q_heads, n_kv_heads, head_dim, max_seqlen))


def _workspace(nbytes, device, workspace):
    if nbytes == 0:
        return None
    if workspace is not None:
        return workspace
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def jl_bifocal_prefill(q, k, v, cu_seqlens, max_seqlen, w_pretrained, w0, rope_theta, out=None,
                       lse=None, flags=0, workspace=None, stream=None):
    """Causal GQA prefill with Dynamic Bifocal RoPE over packed sequences.

    q [T, Hq, D], k/v [T, Hkv, D] (standard-RoPE q and k), cu_seqlens int32
    [B+1] on the device.  Returns (out [T, Hq, D], lse [Hq, T] or None).
    """
    T, Hq, D = q.shape
    Hkv = k.shape[1]
    B = cu_seqlens.numel() - 1
    if out is None:
        out = torch.empty_like(q)
    ws_bytes = jl_bifocal_prefill_workspace_size(B, T, Hq, Hkv, D, q.dtype, flags)
    ws = _workspace(ws_bytes, q.device, workspace)
    _check(lib().jl_bifocal_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(cu_seqlens),
                                    B, T, int(max_seqlen), Hq, Hkv, D, int(w_pretrained), int(w0),
                                    float(rope_theta), _dtype_code(q), int(flags), _ptr(ws),
                                    0 if ws is None else ws.numel() * ws.element_size(),
                                    _stream(stream)))
    return out, lse


def jl_bifocal_prefill_kv(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, w_pretrained, w0, rope_theta,
                          out=None, lse=None, flags=0, workspace=None, stream=None, window=0):
    """Prefill of new tokens against keys that include an existing cache:
    sequence s has its Lq queries at the last positions of its Lk keys.
    ``window`` > 0: sliding-window layer (keys at distance >= window hidden).

    q [Tq, Hq, D]; k, v [Tk, Hkv, D]; cu_seqlens_q / cu_seqlens_k int32 [B+1]
    on the device.  Returns (out [Tq, Hq, D], lse [Hq, Tq] or None).
    """
    Tq, Hq, D = q.shape
    Tk, Hkv = k.shape[0], k.shape[1]
    B = cu_seqlens_q.numel() - 1
    if out is None:
        out = torch.empty_like(q)
    ws_bytes = jl_bifocal_prefill_workspace_size(B, Tk, Hq, Hkv, D, q.dtype, flags)
    ws = _workspace(ws_bytes, q.device, workspace)
    _check(lib().jl_bifocal_prefill_kv(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(cu_seqlens_q),
                                       _ptr(cu_seqlens_k), B, Tq, Tk, int(max_seqlen_q), Hq, Hkv, D,
                                       int(w_pretrained), int(w0), int(window), float(rope_theta), _dtype_code(q),
                                       int(flags),
                                       _ptr(ws), 0 if ws is None else ws.numel() * ws.element_size(),
                                       _stream(stream)))
    return out, lse


def jl_bifocal_decode(q, k_cache, v_cache, seqlens, max_seqlen, w_pretrained, w0, rope_theta,
                      out=None, lse=None, flags=0, workspace=None, stream=None):
    """One decode step: q [B, Hq, D] at position L_b - 1 against the cache
    [B, Lcap, Hkv, D] (rows 0 .. L_b - 1).  Returns (out [B, Hq, D], lse)."""
    B, Hq, D = q.shape
    Lcap, Hkv = k_cache.shape[1], k_cache.shape[2]
    if out is None:
        out = torch.empty_like(q)
    ws_bytes = jl_bifocal_decode_workspace_size(B, Hq, Hkv, D, int(max_seqlen))
    ws = _workspace(ws_bytes, q.device, workspace)
    _check(lib().jl_bifocal_decode(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seqlens), B, Lcap,
                                   int(max_seqlen), Hq, Hkv, D, int(w_pretrained), int(w0),
                                   float(rope_theta), _ptr(out), _ptr(lse), _ptr(ws),
                                   0 if ws is None else ws.numel() * ws.element_size(),
                                   _dtype_code(q), int(flags), _stream(stream)))
    return out, lse


def jl_bifocal_decode_window(q, k_cache, v_cache, seqlens, max_seqlen, w_pretrained, w0, window, rope_theta,
                             out=None, lse=None, flags=0, workspace=None, stream=None):
    """jl_bifocal_decode for a sliding-window layer: the new query attends to
    the last ``window`` keys of its sequence (0: all keys)."""
    B, Hq, D = q.shape
    Lcap, Hkv = k_cache.shape[1], k_cache.shape[2]
    if out is None:
        out = torch.empty_like(q)
    ws_bytes = jl_bifocal_decode_workspace_size(B, Hq, Hkv, D, int(max_seqlen))
    ws = _workspace(ws_bytes, q.device, workspace)
    _check(lib().jl_bifocal_decode_window(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seqlens), B, Lcap,
                                          int(max_seqlen), Hq, Hkv, D, int(w_pretrained), int(w0), int(window),
                                          float(rope_theta), _ptr(out), _ptr(lse), _ptr(ws),
                                          0 if ws is None else ws.numel() * ws.element_size(),
                                          _dtype_code(q), int(flags), _stream(stream)))
    return out, lse


JL_DECODE_NOALLOC_SCRATCH_BYTES = 4 << 20


def jl_bifocal_decode_noalloc(q, k_cache, v_cache, seqlens, max_seqlen, w_pretrained, w0, rope_theta,
                              out, lse=None, flags=0, stream=None):
    """jl_bifocal_decode for callers that cannot allocate device memory: the
    library supplies the scratch from a fixed array in its device image
    (JL_DECODE_NOALLOC_SCRATCH_BYTES), so ``out`` must be given and nothing
    is allocated.  Calls that overlap on the GPU share that array and race."""
    B, Hq, D = q.shape
    Lcap, Hkv = k_cache.shape[1], k_cache.shape[2]
    _check(lib().jl_bifocal_decode_noalloc(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seqlens), B, Lcap,
                                           int(max_seqlen), Hq, Hkv, D, int(w_pretrained), int(w0),
                                           float(rope_theta), _ptr(out), _ptr(lse), _dtype_code(q), int(flags),
                                           _stream(stream)))
    return out, lse


def jl_bifocal_decode_noalloc_error(stream=None) -> int:
    """The kernel error word of the last jl_bifocal_decode_noalloc call (0: no
    error).  Enqueues the copy on ``stream`` and synchronises it."""
    word = ctypes.c_int32(-1)
    st = _stream(stream)
    _check(lib().jl_bifocal_decode_noalloc_error(ctypes.byref(word), st))
    (stream or torch.cuda.current_stream()).synchronize()
    return int(word.value)
