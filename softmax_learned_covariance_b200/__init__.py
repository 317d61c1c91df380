"""Parallax attention on B200 (sm_100a): Python binding of the C ABI in include/parallax.h.

Parallax keeps exact softmax attention and subtracts the softmax-weighted
key/value covariance projected by a learned probe rho_i = W_R x_i (zubnet.ai
news item on Parallax, paragraph 2):  y_i = o_i - (m_i - o_i abar_i).

This module only marshals torch tensors to the shared library
``libparallax.so`` (built by ``softmax_learned_covariance_b200.build``); every
step of the computation runs in its CUDA kernels.  There is no fallback: if the
library is missing or a call fails, a ``ParallaxError`` is raised.

Functions keep the C names:
    parallax_fwd(q, k, v, rho=None, causal=True, out_dtype=torch.float32) -> (y, lse)
    parallax_fwd_fused(q, k, v, x, W_R, causal=True) -> (y, lse)     probe rho = x W_R in the kernel
    parallax_fwd_train(q, k, v, rho, causal=True) -> (y, lse, o, abar)  the forward kept for the backward
    parallax_bwd(q, k, v, rho, y, o, abar, lse, dy, causal=True) -> (dq, dk, dv, drho)
    parallax_decode(q, rho, kcache, vcache, seqlens, out_dtype=torch.float32) -> (y, lse)
    parallax_softmax_decode(q, kcache, vcache, seqlens) -> (y, lse)   reference: softmax attention, d 64/128/256
    parallax_decode_ex(..., workspace) -> (y, lse)          caller-owned split scratch
    parallax_decode_paged(q, rho, kpages, vpages, block_table, seqlens) -> (y, lse)
                                                            paged cache, grouped query heads
    parallax_rho_proj(x, W_R, H, d) -> rho
"""
from __future__ import annotations

import ctypes
import os
import threading

__all__ = [
    "ParallaxError", "lib", "parallax_fwd", "parallax_fwd_fused", "parallax_fwd_train", "parallax_bwd",
    "parallax_decode", "parallax_softmax_decode", "parallax_decode_ex", "parallax_decode_paged",
    "parallax_rho_proj", "parallax_decode_workspace_bytes", "parallax_last_device_error",
    "parallax_strerror", "parallax_device_sm_count", "LIB_PATH", "F32", "BF16",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libparallax.so")
F32, BF16 = 0, 1
_lock = threading.Lock()
_lib = None


class ParallaxError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {parallax_strerror(status)} (status {status})")


def lib() -> ctypes.CDLL:
    """The loaded C library (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise ParallaxError(-1, f"{LIB_PATH} is missing; build it with "
                                        "`python -m softmax_learned_covariance_b200.build`")
            L = ctypes.CDLL(LIB_PATH)
            P, I, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
            L.parallax_fwd.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, I, P]
            L.parallax_fwd_fused.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, P]
            L.parallax_fwd_train.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, I, P]
            L.parallax_bwd.argtypes = [P, P, P, P, P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, P]
            L.parallax_decode.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, P]
            L.parallax_softmax_decode.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, P]
            L.parallax_decode_ex.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, P, S, P]
            L.parallax_decode_paged.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, I, P]
            L.parallax_decode_workspace_bytes.argtypes = [I, I, I, I]
            L.parallax_decode_workspace_bytes.restype = S
            L.parallax_rho_proj.argtypes = [P, P, P, I, I, I, I, I, I, P]
            L.parallax_strerror.argtypes = [I]
            L.parallax_strerror.restype = ctypes.c_char_p
            L.parallax_last_device_error.argtypes = [P]
            L.parallax_device_sm_count.argtypes = []
            for f in (L.parallax_fwd, L.parallax_fwd_fused, L.parallax_fwd_train, L.parallax_bwd, L.parallax_decode,
                      L.parallax_softmax_decode, L.parallax_decode_ex, L.parallax_decode_paged,
                      L.parallax_rho_proj,
                      L.parallax_last_device_error, L.parallax_device_sm_count):
                f.restype = I
            _lib = L
    return _lib


def parallax_strerror(status: int) -> str:
    if status == -1:
        return "library not built"
    return lib().parallax_strerror(int(status)).decode()


def _torch():
    import torch

    return torch


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    torch = _torch()
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype_code(dt):
    torch = _torch()
    if dt == torch.float32:
        return F32
    if dt == torch.bfloat16:
        return BF16
    raise TypeError(f"unsupported dtype {dt}")


def _check(status, what):
    if status != 0:
        raise ParallaxError(status, what)


def _need(t, name):
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA tensor")


def parallax_fwd(q, k, v, rho=None, causal: bool = True, out_dtype=None, y=None, lse=None,
                 stream=None, want_lse: bool = True):
    """Prefill/forward.  q,k,v,rho: [B,H,T,d]; returns (y [B,H,T,d], lse [B,H,T] fp32 or None).

    rho=None runs the softmax-only instantiation.  bf16 inputs run on the tensor
    cores (d = 128); fp32 inputs run the fp32 CUDA-core kernel.
    """
    torch = _torch()
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n)
    if rho is not None:
        _need(rho, "rho")
    B, H, T, d = q.shape
    out_dtype = out_dtype or torch.float32
    if y is None:
        y = torch.empty((B, H, T, d), dtype=out_dtype, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((B, H, T), dtype=torch.float32, device=q.device)
    st = lib().parallax_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(rho), _ptr(y), _ptr(lse), B, H, T, d,
                            int(bool(causal)), _dtype_code(q.dtype), _dtype_code(y.dtype), _stream(stream))
    _check(st, "parallax_fwd")
    return y, lse


def parallax_fwd_fused(q, k, v, x, W_R, causal: bool = True, out_dtype=None, y=None, lse=None, stream=None,
                       want_lse: bool = True):
    """Prefill with the probe rho = x W_R computed in the kernel.

    q, k, v: [B, H, T, d] bf16 (d = 128); x: [B, T, d_model] bf16; W_R: [d_model, H*d] bf16.
    """
    torch = _torch()
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (x, "x"), (W_R, "W_R")):
        _need(t, n)
    B, H, T, d = q.shape
    d_model = x.shape[-1]
    out_dtype = out_dtype or torch.float32
    if y is None:
        y = torch.empty((B, H, T, d), dtype=out_dtype, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((B, H, T), dtype=torch.float32, device=q.device)
    st = lib().parallax_fwd_fused(_ptr(q), _ptr(k), _ptr(v), _ptr(x), _ptr(W_R), _ptr(y), _ptr(lse), B, H, T, d,
                                  d_model, int(bool(causal)), _dtype_code(q.dtype), _dtype_code(y.dtype),
                                  _stream(stream))
    _check(st, "parallax_fwd_fused")
    return y, lse


def parallax_fwd_train(q, k, v, rho, causal: bool = True, stream=None):
    """Training forward: (y, lse, o, abar), fp32; o and abar are what parallax_bwd needs."""
    torch = _torch()
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (rho, "rho")):
        _need(t, n)
    B, H, T, d = q.shape
    f32 = dict(dtype=torch.float32, device=q.device)
    y, o = torch.empty((B, H, T, d), **f32), torch.empty((B, H, T, d), **f32)
    lse, abar = torch.empty((B, H, T), **f32), torch.empty((B, H, T), **f32)
    st = lib().parallax_fwd_train(_ptr(q), _ptr(k), _ptr(v), _ptr(rho), _ptr(y), _ptr(lse), _ptr(o), _ptr(abar),
                                  B, H, T, d, int(bool(causal)), _dtype_code(q.dtype), _stream(stream))
    _check(st, "parallax_fwd_train")
    return y, lse, o, abar


def parallax_bwd(q, k, v, rho, y, o, abar, lse, dy, causal: bool = True, stream=None, out=None):
    """Gradients (dq, dk, dv, drho), fp32, for an upstream dy (bf16, [B, H, T, d]).

    ``out``: optional (dq, dk, dv, drho) fp32 [B, H, T, d] tensors to write into."""
    torch = _torch()
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (rho, "rho"), (y, "y"), (o, "o"), (abar, "abar"), (lse, "lse"),
                 (dy, "dy")):
        _need(t, n)
    B, H, T, d = q.shape
    if out is None:
        outs = [torch.empty((B, H, T, d), dtype=torch.float32, device=q.device) for _ in range(4)]
    else:
        outs = list(out)
        for t, n in zip(outs, ("dq", "dk", "dv", "drho")):
            _need(t, n)
            if t.dtype != torch.float32 or tuple(t.shape) != (B, H, T, d):
                raise ValueError(f"{n} must be float32 of shape {(B, H, T, d)}")
    st = lib().parallax_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(rho), _ptr(y), _ptr(o), _ptr(abar), _ptr(lse), _ptr(dy),
                            *(_ptr(t) for t in outs), B, H, T, d, int(bool(causal)), _dtype_code(q.dtype),
                            _stream(stream))
    _check(st, "parallax_bwd")
    return tuple(outs)


def parallax_decode(q, rho, kcache, vcache, seqlens, out_dtype=None, y=None, lse=None, stream=None,
                    want_lse: bool = True):
    """Decode one token per sequence.  q,rho: [B,H,d]; caches [B,H,Tcap,d]; seqlens int32 [B] on device."""
    torch = _torch()
    for t, n in ((q, "q"), (rho, "rho"), (kcache, "kcache"), (vcache, "vcache"), (seqlens, "seqlens")):
        _need(t, n)
    if seqlens.dtype != torch.int32:
        raise TypeError("seqlens must be int32")
    B, H, Tcap, d = kcache.shape
    out_dtype = out_dtype or torch.float32
    if y is None:
        y = torch.empty((B, H, d), dtype=out_dtype, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((B, H), dtype=torch.float32, device=q.device)
    st = lib().parallax_decode(_ptr(q), _ptr(rho), _ptr(kcache), _ptr(vcache), _ptr(seqlens), _ptr(y),
                               _ptr(lse), B, H, Tcap, d, _dtype_code(q.dtype), _dtype_code(y.dtype),
                               _stream(stream))
    _check(st, "parallax_decode")
    return y, lse


def parallax_softmax_decode(q, kcache, vcache, seqlens, out_dtype=None, y=None, lse=None, stream=None,
                            want_lse: bool = True):
    """Plain softmax attention decode (no probe), head dims 64, 128, 256: the pages' reference point."""
    torch = _torch()
    for t, n in ((q, "q"), (kcache, "kcache"), (vcache, "vcache"), (seqlens, "seqlens")):
        _need(t, n)
    B, H, Tcap, d = kcache.shape
    out_dtype = out_dtype or torch.float32
    if y is None:
        y = torch.empty((B, H, d), dtype=out_dtype, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((B, H), dtype=torch.float32, device=q.device)
    st = lib().parallax_softmax_decode(_ptr(q), _ptr(kcache), _ptr(vcache), _ptr(seqlens), _ptr(y), _ptr(lse), B, H,
                                       Tcap, d, _dtype_code(q.dtype), _dtype_code(y.dtype), _stream(stream))
    _check(st, "parallax_softmax_decode")
    return y, lse


def parallax_decode_workspace_bytes(B: int, H: int, Tcap: int, d: int) -> int:
    return int(lib().parallax_decode_workspace_bytes(B, H, Tcap, d))


def parallax_decode_ex(q, rho, kcache, vcache, seqlens, workspace, out_dtype=None, y=None, lse=None,
                       stream=None, want_lse: bool = True):
    """parallax_decode with a caller-owned workspace tensor (any dtype, >= the required bytes)."""
    torch = _torch()
    B, H, Tcap, d = kcache.shape
    out_dtype = out_dtype or torch.float32
    if y is None:
        y = torch.empty((B, H, d), dtype=out_dtype, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((B, H), dtype=torch.float32, device=q.device)
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib().parallax_decode_ex(_ptr(q), _ptr(rho), _ptr(kcache), _ptr(vcache), _ptr(seqlens), _ptr(y),
                                  _ptr(lse), B, H, Tcap, d, _dtype_code(q.dtype), _dtype_code(y.dtype),
                                  _ptr(workspace), nbytes, _stream(stream))
    _check(st, "parallax_decode_ex")
    return y, lse


def parallax_decode_paged(q, rho, kpages, vpages, block_table, seqlens, out_dtype=None, y=None, lse=None,
                          stream=None, want_lse: bool = True):
    """Decode over a paged cache with grouped query heads.

    q, rho: [B, Hq, d]; kpages, vpages: [num_pages, Hkv, page_size, d];
    block_table: int32 [B, max_pages] and seqlens: int32 [B], both on the device.
    """
    torch = _torch()
    for t, n in ((q, "q"), (rho, "rho"), (kpages, "kpages"), (vpages, "vpages"), (block_table, "block_table"),
                 (seqlens, "seqlens")):
        _need(t, n)
    if seqlens.dtype != torch.int32 or block_table.dtype != torch.int32:
        raise TypeError("seqlens and block_table must be int32")
    B, Hq, d = q.shape
    num_pages, Hkv, page_size, _ = kpages.shape
    max_pages = block_table.shape[1]
    out_dtype = out_dtype or torch.float32
    if y is None:
        y = torch.empty((B, Hq, d), dtype=out_dtype, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    st = lib().parallax_decode_paged(_ptr(q), _ptr(rho), _ptr(kpages), _ptr(vpages), _ptr(block_table),
                                     _ptr(seqlens), _ptr(y), _ptr(lse), B, Hq, Hkv, page_size, max_pages,
                                     num_pages, d, _dtype_code(q.dtype), _dtype_code(y.dtype), _stream(stream))
    _check(st, "parallax_decode_paged")
    return y, lse


def parallax_rho_proj(x, W_R, H: int, d: int, rho=None, stream=None):
    """rho [B,H,T,d] bf16 = per-head slices of x [B,T,d_model] @ W_R [d_model, H*d]."""
    torch = _torch()
    _need(x, "x")
    _need(W_R, "W_R")
    B, T, dm = x.shape
    if rho is None:
        rho = torch.empty((B, H, T, d), dtype=torch.bfloat16, device=x.device)
    st = lib().parallax_rho_proj(_ptr(x), _ptr(W_R), _ptr(rho), B, T, dm, H, d, _dtype_code(x.dtype),
                                 _stream(stream))
    _check(st, "parallax_rho_proj")
    return rho


def parallax_last_device_error(stream=None) -> int:
    """Sync the stream; return and clear the device error word (0 or a status code)."""
    return int(lib().parallax_last_device_error(_stream(stream)))


def parallax_device_sm_count() -> int:
    return int(lib().parallax_device_sm_count())
