"""Causal grouped-query attention with RoPE for NVIDIA B200 (sm_100a).

Thin ctypes binding over ``libnea.so`` (C ABI in ``include/nea_attn.h``).
This module only checks and marshals arguments; every step of the
computation runs in the library's CUDA kernels.  There is no fallback: if the
library is missing, importing this package raises.

Tensors are torch CUDA tensors, contiguous, in the library layout:
``q, o, do, dq: [B, T, Hq, D]``, ``k, v, dk, dv: [B, T, Hkv, D]``,
``lse: [B, Hq, T]`` (float32); dtype float32 or bfloat16.
"""
from __future__ import annotations

import ctypes
import os

__all__ = [
    "nea_attn_fwd", "nea_attn_bwd", "nea_device_status", "nea_set_wait_limit_ns", "nea_debug_inject",
    "nea_status_string", "nea_version", "nea_set_profile_events", "NeaError", "LIB_PATH", "NEA_OK", "NEA_ERR_ARG", "NEA_ERR_CUDA",
    "NEA_ERR_TIMEOUT", "NEA_ERR_UNSUPPORTED", "NEA_ERR_NOMEM", "NEA_ERR_SCRATCH_LIMIT", "NEA_F32", "NEA_BF16",
    "nea_attn_bwd_noalloc", "nea_attn_decode", "nea_attn_saved_bytes", "nea_attn_fwd_save", "nea_attn_bwd_saved",
    "nea_block_qkv_fwd", "nea_block_qkv_bwd", "nea_block_out_fwd", "nea_block_out_bwd", "nea_block_ffn_fwd",
    "nea_block_ffn_bwd",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libnea.so")

NEA_F32, NEA_BF16 = 0, 1
NEA_OK, NEA_ERR_ARG, NEA_ERR_CUDA, NEA_ERR_TIMEOUT, NEA_ERR_UNSUPPORTED, NEA_ERR_NOMEM, NEA_ERR_SCRATCH_LIMIT = range(7)

if not os.path.exists(LIB_PATH):
    raise ImportError(f"libnea.so not built ({LIB_PATH}); run `python causal_gqa_attention_sm_b200/build.py`")

_lib = ctypes.CDLL(LIB_PATH)
_vp, _i, _f, _ll = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_longlong
_lib.nea_attn_fwd.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _i, _vp]
_lib.nea_attn_fwd.restype = _i
_lib.nea_attn_bwd.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _i, _vp]
_lib.nea_attn_bwd.restype = _i
_lib.nea_device_status.argtypes = [_vp]
_lib.nea_device_status.restype = _i
_lib.nea_set_wait_limit_ns.argtypes = [_ll]
_lib.nea_set_wait_limit_ns.restype = _ll
_lib.nea_debug_inject.argtypes = [_i]
_lib.nea_debug_inject.restype = None
_lib.nea_status_string.argtypes = [_i]
_lib.nea_status_string.restype = ctypes.c_char_p
_lib.nea_set_profile_events.argtypes = [ctypes.POINTER(ctypes.c_void_p), _i]
_lib.nea_set_profile_events.restype = None
_lib.nea_attn_bwd_noalloc.argtypes = list(_lib.nea_attn_bwd.argtypes)
_lib.nea_attn_bwd_noalloc.restype = _i
_lib.nea_attn_decode.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _vp]
_lib.nea_attn_decode.restype = _i
_lib.nea_attn_saved_bytes.argtypes = [_i, _i, _i, _i, _i, _i, _f]
_lib.nea_attn_saved_bytes.restype = _ll
_lib.nea_attn_fwd_save.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _i, _vp]
_lib.nea_attn_fwd_save.restype = _i
_lib.nea_attn_bwd_saved.argtypes = [_vp] * 10 + [_i, _i, _i, _i, _i, _i, _f, _i, _vp]
_lib.nea_attn_bwd_saved.restype = _i
_lib.nea_block_qkv_fwd.argtypes = [_vp] * 8 + [_i] * 6 + [_vp]
_lib.nea_block_qkv_fwd.restype = _i
_lib.nea_block_qkv_bwd.argtypes = [_vp] * 14 + [_i] * 6 + [_vp]
_lib.nea_block_qkv_bwd.restype = _i
_lib.nea_block_out_fwd.argtypes = [_vp] * 4 + [_i] * 5 + [_vp]
_lib.nea_block_out_fwd.restype = _i
_lib.nea_block_out_bwd.argtypes = [_vp] * 5 + [_i] * 5 + [_vp]
_lib.nea_block_out_bwd.restype = _i
_lib.nea_block_ffn_fwd.argtypes = [_vp] * 8 + [_i] * 4 + [_vp]
_lib.nea_block_ffn_fwd.restype = _i
_lib.nea_block_ffn_bwd.argtypes = [_vp] * 13 + [_i] * 4 + [_vp]
_lib.nea_block_ffn_bwd.restype = _i
_lib.nea_version.argtypes = []
_lib.nea_version.restype = _i


class NeaError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {nea_status_string(status)}")
        self.status = status


def nea_status_string(status: int) -> str:
    return _lib.nea_status_string(int(status)).decode()


def nea_version() -> int:
    return int(_lib.nea_version())


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None and t.numel() > 0 else None


def _stream(stream):
    import torch

    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype_code(t):
    import torch

    if t.dtype == torch.float32:
        return NEA_F32
    if t.dtype == torch.bfloat16:
        return NEA_BF16
    raise TypeError(f"unsupported dtype {t.dtype}; expected float32 or bfloat16")


def _check(t, name, shape, dtype, device):
    if not t.is_cuda or t.device != device:
        raise ValueError(f"{name} must be a CUDA tensor on {device}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if t.dtype != dtype:
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _shapes(q, k, v):
    if q.dim() != 4 or k.dim() != 4:
        raise ValueError("q, k, v must be [B, T, H, D]")
    B, T, Hq, D = q.shape
    Hkv = k.shape[2]
    return B, T, Hq, Hkv, D


def nea_attn_fwd(q, k, v, rope_base: float = 10000.0, causal: bool = True, o=None, lse=None, stream=None):
    """Forward: returns ``(o, lse)``.  ``o``/``lse`` may be passed preallocated."""
    import torch

    B, T, Hq, Hkv, D = _shapes(q, k, v)
    dev, dt = q.device, q.dtype
    code = _dtype_code(q)
    _check(q, "q", (B, T, Hq, D), dt, dev)
    _check(k, "k", (B, T, Hkv, D), dt, dev)
    _check(v, "v", (B, T, Hkv, D), dt, dev)
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, T), dtype=torch.float32, device=dev)
    _check(o, "o", (B, T, Hq, D), dt, dev)
    _check(lse, "lse", (B, Hq, T), torch.float32, dev)
    rc = _lib.nea_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, T, Hq, Hkv, D, code,
                           float(rope_base), int(bool(causal)), _stream(stream))
    if rc != NEA_OK:
        raise NeaError(rc, "nea_attn_fwd")
    return o, lse


def nea_attn_bwd(q, k, v, o, lse, do, rope_base: float = 10000.0, causal: bool = True,
                 dq=None, dk=None, dv=None, stream=None):
    """Backward: returns ``(dq, dk, dv)`` (gradients w.r.t. un-rotated q, k and v)."""
    import torch

    B, T, Hq, Hkv, D = _shapes(q, k, v)
    dev, dt = q.device, q.dtype
    code = _dtype_code(q)
    _check(q, "q", (B, T, Hq, D), dt, dev)
    _check(k, "k", (B, T, Hkv, D), dt, dev)
    _check(v, "v", (B, T, Hkv, D), dt, dev)
    _check(o, "o", (B, T, Hq, D), dt, dev)
    _check(do, "do", (B, T, Hq, D), dt, dev)
    _check(lse, "lse", (B, Hq, T), torch.float32, dev)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    _check(dq, "dq", (B, T, Hq, D), dt, dev)
    _check(dk, "dk", (B, T, Hkv, D), dt, dev)
    _check(dv, "dv", (B, T, Hkv, D), dt, dev)
    rc = _lib.nea_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(do), _ptr(dq), _ptr(dk), _ptr(dv),
                           B, T, Hq, Hkv, D, code, float(rope_base), int(bool(causal)), _stream(stream))
    if rc != NEA_OK:
        raise NeaError(rc, "nea_attn_bwd")
    return dq, dk, dv


def nea_attn_bwd_noalloc(q, k, v, o, lse, do, dq, dk, dv, rope_base: float = 10000.0, causal: bool = True,
                         stream=None):
    """Backward that allocates no device memory (for callers that may not call
    cudaMalloc): the outputs ``dq, dk, dv`` must be passed preallocated; the
    scratch is a fixed 4 MiB array inside the library (see include/nea_attn.h
    for its limit and the rule that concurrent calls must be serialised)."""
    import torch

    B, T, Hq, Hkv, D = _shapes(q, k, v)
    dev, dt = q.device, q.dtype
    code = _dtype_code(q)
    for t, n, shp in ((q, "q", (B, T, Hq, D)), (k, "k", (B, T, Hkv, D)), (v, "v", (B, T, Hkv, D)),
                      (o, "o", (B, T, Hq, D)), (do, "do", (B, T, Hq, D)), (dq, "dq", (B, T, Hq, D)),
                      (dk, "dk", (B, T, Hkv, D)), (dv, "dv", (B, T, Hkv, D))):
        _check(t, n, shp, dt, dev)
    _check(lse, "lse", (B, Hq, T), torch.float32, dev)
    rc = _lib.nea_attn_bwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(do), _ptr(dq), _ptr(dk),
                                   _ptr(dv), B, T, Hq, Hkv, D, code, float(rope_base), int(bool(causal)),
                                   _stream(stream))
    if rc != NEA_OK:
        raise NeaError(rc, "nea_attn_bwd_noalloc")
    return dq, dk, dv


def nea_attn_saved_bytes(B: int, T: int, Hq: int, Hkv: int, D: int, dtype, rope_base: float = 10000.0) -> int:
    """Bytes of the save-for-backward buffer (``dtype`` a torch dtype or NEA_F32/NEA_BF16)."""
    import torch

    code = dtype if isinstance(dtype, int) else {torch.float32: NEA_F32, torch.bfloat16: NEA_BF16}[dtype]
    n = int(_lib.nea_attn_saved_bytes(B, T, Hq, Hkv, D, code, float(rope_base)))
    if n < 0:
        raise NeaError(NEA_ERR_ARG, "nea_attn_saved_bytes")
    return n


def _check_saved(saved, need, device):
    if need == 0:
        return
    if saved is None or not saved.is_cuda or saved.device != device or not saved.is_contiguous():
        raise ValueError(f"saved must be a contiguous CUDA tensor on {device}")
    if saved.numel() * saved.element_size() < need:
        raise ValueError(f"saved holds {saved.numel() * saved.element_size()} bytes, needs {need}")


def nea_attn_fwd_save(q, k, v, rope_base: float = 10000.0, causal: bool = True, o=None, lse=None, saved=None,
                      stream=None):
    """Forward that keeps its operand planes for the backward: returns
    ``(o, lse, saved)``; ``saved`` (a uint8 CUDA tensor of
    ``nea_attn_saved_bytes`` bytes) is passed to ``nea_attn_bwd_saved``."""
    import torch

    B, T, Hq, Hkv, D = _shapes(q, k, v)
    dev, dt = q.device, q.dtype
    code = _dtype_code(q)
    _check(q, "q", (B, T, Hq, D), dt, dev)
    _check(k, "k", (B, T, Hkv, D), dt, dev)
    _check(v, "v", (B, T, Hkv, D), dt, dev)
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, T), dtype=torch.float32, device=dev)
    _check(o, "o", (B, T, Hq, D), dt, dev)
    _check(lse, "lse", (B, Hq, T), torch.float32, dev)
    need = nea_attn_saved_bytes(B, T, Hq, Hkv, D, code, rope_base)
    if saved is None:
        saved = torch.empty(need, dtype=torch.uint8, device=dev)
    _check_saved(saved, need, dev)
    rc = _lib.nea_attn_fwd_save(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(saved), B, T, Hq, Hkv, D, code,
                                float(rope_base), int(bool(causal)), _stream(stream))
    if rc != NEA_OK:
        raise NeaError(rc, "nea_attn_fwd_save")
    return o, lse, saved


def nea_attn_bwd_saved(q, k, v, o, lse, do, saved, rope_base: float = 10000.0, causal: bool = True,
                       dq=None, dk=None, dv=None, stream=None):
    """Backward reading Q, K, V operands from ``saved`` (what ``nea_attn_fwd_save``
    wrote for the same q, k, v and rope_base): returns ``(dq, dk, dv)``."""
    import torch

    B, T, Hq, Hkv, D = _shapes(q, k, v)
    dev, dt = q.device, q.dtype
    code = _dtype_code(q)
    for t, n, shp in ((q, "q", (B, T, Hq, D)), (k, "k", (B, T, Hkv, D)), (v, "v", (B, T, Hkv, D)),
                      (o, "o", (B, T, Hq, D)), (do, "do", (B, T, Hq, D))):
        _check(t, n, shp, dt, dev)
    _check(lse, "lse", (B, Hq, T), torch.float32, dev)
    _check_saved(saved, nea_attn_saved_bytes(B, T, Hq, Hkv, D, code, rope_base), dev)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    _check(dq, "dq", (B, T, Hq, D), dt, dev)
    _check(dk, "dk", (B, T, Hkv, D), dt, dev)
    _check(dv, "dv", (B, T, Hkv, D), dt, dev)
    rc = _lib.nea_attn_bwd_saved(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(do), _ptr(saved), _ptr(dq),
                                 _ptr(dk), _ptr(dv), B, T, Hq, Hkv, D, code, float(rope_base), int(bool(causal)),
                                 _stream(stream))
    if rc != NEA_OK:
        raise NeaError(rc, "nea_attn_bwd_saved")
    return dq, dk, dv


def _block_check(name, t, shape, dt, dev):
    _check(t, name, shape, dt, dev)


def nea_block_qkv_fwd(x, g, Wq, Wk, Wv, Hq: int, Hkv: int, D: int, q=None, k=None, v=None, stream=None):
    """Pre-norm and projections: returns ``(q, k, v)`` as ``[B, T, H, D]`` for
    ``x`` of shape ``[B, T, C]`` (RMSNorm with gain ``g`` applied inside)."""
    import torch

    B, T, C = x.shape
    dev, dt = x.device, x.dtype
    code = _dtype_code(x)
    for t, n, shp in ((x, "x", (B, T, C)), (g, "g", (C,)), (Wq, "Wq", (C, Hq * D)), (Wk, "Wk", (C, Hkv * D)),
                      (Wv, "Wv", (C, Hkv * D))):
        _block_check(n, t, shp, dt, dev)
    q = torch.empty((B, T, Hq, D), dtype=dt, device=dev) if q is None else q
    k = torch.empty((B, T, Hkv, D), dtype=dt, device=dev) if k is None else k
    v = torch.empty((B, T, Hkv, D), dtype=dt, device=dev) if v is None else v
    for t, n, shp in ((q, "q", (B, T, Hq, D)), (k, "k", (B, T, Hkv, D)), (v, "v", (B, T, Hkv, D))):
        _block_check(n, t, shp, dt, dev)
    rc = _lib.nea_block_qkv_fwd(_ptr(x), _ptr(g), _ptr(Wq), _ptr(Wk), _ptr(Wv), _ptr(q), _ptr(k), _ptr(v), B * T, C,
                                Hq, Hkv, D, code, _stream(stream))
    if rc != NEA_OK:
        raise NeaError(rc, "nea_block_qkv_fwd")
    return q, k, v


def nea_block_qkv_bwd(x, g, Wq, Wk, Wv, dq, dk, dv, dres=None, stream=None):
    """Backward of ``nea_block_qkv_fwd``: returns ``(dx, dg, dWq, dWk, dWv)``;
    ``dres`` (the residual branch's gradient) is added to ``dx`` when given."""
    import torch

    B, T, C = x.shape
    Hq, D = dq.shape[2], dq.shape[3]
    Hkv = dk.shape[2]
    dev, dt = x.device, x.dtype
    code = _dtype_code(x)
    for t, n, shp in ((x, "x", (B, T, C)), (g, "g", (C,)), (Wq, "Wq", (C, Hq * D)), (Wk, "Wk", (C, Hkv * D)),
                      (Wv, "Wv", (C, Hkv * D)), (dq, "dq", (B, T, Hq, D)), (dk, "dk", (B, T, Hkv, D)),
                      (dv, "dv", (B, T, Hkv, D))):
        _block_check(n, t, shp, dt, dev)
    if dres is not None:
        _block_check("dres", dres, (B, T, C), dt, dev)
    dx, dg = torch.empty_like(x), torch.empty_like(g)
    dWq, dWk, dWv = torch.empty_like(Wq), torch.empty_like(Wk), torch.empty_like(Wv)
    rc = _lib.nea_block_qkv_bwd(_ptr(x), _ptr(g), _ptr(Wq), _ptr(Wk), _ptr(Wv), _ptr(dq), _ptr(dk), _ptr(dv),
                                _ptr(dres), _ptr(dx), _ptr(dg), _ptr(dWq), _ptr(dWk), _ptr(dWv), B * T, C, Hq, Hkv, D,
                                code, _stream(stream))
    if rc != NEA_OK:
        raise NeaError(rc, "nea_block_qkv_bwd")
    return dx, dg, dWq, dWk, dWv


def nea_block_out_fwd(x, o, Wo, h=None, stream=None):
    """Output projection with the residual: ``h = x + o Wo`` for ``o`` of shape
    ``[B, T, Hq, D]``."""
    import torch

    B, T, C = x.shape
    Hq, D = o.shape[2], o.shape[3]
    dev, dt = x.device, x.dtype
    code = _dtype_code(x)
    for t, n, shp in ((x, "x", (B, T, C)), (o, "o", (B, T, Hq, D)), (Wo, "Wo", (Hq * D, C))):
        _block_check(n, t, shp, dt, dev)
    h = torch.empty_like(x) if h is None else h
    _block_check("h", h, (B, T, C), dt, dev)
    rc = _lib.nea_block_out_fwd(_ptr(x), _ptr(o), _ptr(Wo), _ptr(h), B * T, C, Hq, D, code, _stream(stream))
    if rc != NEA_OK:
        raise NeaError(rc, "nea_block_out_fwd")
    return h


def nea_block_out_bwd(o, Wo, dh, stream=None):
    """Backward of ``nea_block_out_fwd``: returns ``(do, dWo)`` (the residual's
    gradient is ``dh``)."""
    import torch

    B, T, Hq, D = o.shape
    C = dh.shape[2]
    dev, dt = o.device, o.dtype
    code = _dtype_code(o)
    for t, n, shp in ((o, "o", (B, T, Hq, D)), (Wo, "Wo", (Hq * D, C)), (dh, "dh", (B, T, C))):
        _block_check(n, t, shp, dt, dev)
    do, dWo = torch.empty_like(o), torch.empty_like(Wo)
    rc = _lib.nea_block_out_bwd(_ptr(o), _ptr(Wo), _ptr(dh), _ptr(do), _ptr(dWo), B * T, C, Hq, D, code,
                                _stream(stream))
    if rc != NEA_OK:
        raise NeaError(rc, "nea_block_out_bwd")
    return do, dWo


def nea_block_ffn_fwd(x, g, Wg, Wu, Wd, h=None, save=True, stream=None):
    """Pre-norm SwiGLU feed-forward with the residual: ``h = x + (silu(y Wg) *
    (y Wu)) Wd`` for ``x`` of shape ``[B, T, C]``, ``y`` the RMSNorm of ``x``
    with gain ``g``.  Returns ``(h, a, b)``, ``a = y Wg`` and ``b = y Wu`` of
    shape ``[B, T, F]`` saved for the backward (``None`` when ``save`` is
    false)."""
    import torch

    B, T, C = x.shape
    F = Wg.shape[1]
    dev, dt = x.device, x.dtype
    code = _dtype_code(x)
    for t, n, shp in ((x, "x", (B, T, C)), (g, "g", (C,)), (Wg, "Wg", (C, F)), (Wu, "Wu", (C, F)),
                      (Wd, "Wd", (F, C))):
        _block_check(n, t, shp, dt, dev)
    h = torch.empty_like(x) if h is None else h
    _block_check("h", h, (B, T, C), dt, dev)
    a = torch.empty((B, T, F), dtype=dt, device=dev) if save else None
    b = torch.empty((B, T, F), dtype=dt, device=dev) if save else None
    rc = _lib.nea_block_ffn_fwd(_ptr(x), _ptr(g), _ptr(Wg), _ptr(Wu), _ptr(Wd), _ptr(h), _ptr(a), _ptr(b), B * T,
                                C, F, code, _stream(stream))
    if rc != NEA_OK:
        raise NeaError(rc, "nea_block_ffn_fwd")
    return h, a, b


def nea_block_ffn_bwd(x, g, Wg, Wu, Wd, a, b, dh, stream=None):
    """Backward of ``nea_block_ffn_fwd`` from its saved ``a`` and ``b``:
    returns ``(dx, dg, dWg, dWu, dWd)``, ``dx`` including the residual's
    ``dh``."""
    import torch

    B, T, C = x.shape
    F = Wg.shape[1]
    dev, dt = x.device, x.dtype
    code = _dtype_code(x)
    for t, n, shp in ((x, "x", (B, T, C)), (g, "g", (C,)), (Wg, "Wg", (C, F)), (Wu, "Wu", (C, F)),
                      (Wd, "Wd", (F, C)), (a, "a", (B, T, F)), (b, "b", (B, T, F)), (dh, "dh", (B, T, C))):
        _block_check(n, t, shp, dt, dev)
    dx, dg = torch.empty_like(x), torch.empty_like(g)
    dWg, dWu, dWd = torch.empty_like(Wg), torch.empty_like(Wu), torch.empty_like(Wd)
    rc = _lib.nea_block_ffn_bwd(_ptr(x), _ptr(g), _ptr(Wg), _ptr(Wu), _ptr(Wd), _ptr(a), _ptr(b), _ptr(dh),
                                _ptr(dx), _ptr(dg), _ptr(dWg), _ptr(dWu), _ptr(dWd), B * T, C, F, code,
                                _stream(stream))
    if rc != NEA_OK:
        raise NeaError(rc, "nea_block_ffn_bwd")
    return dx, dg, dWg, dWu, dWd


def nea_device_status(stream=None) -> int:
    """Synchronises the stream and returns (and clears) the device status."""
    return int(_lib.nea_device_status(_stream(stream)))


def nea_set_wait_limit_ns(ns: int) -> int:
    return int(_lib.nea_set_wait_limit_ns(int(ns)))


def nea_debug_inject(flags: int) -> None:
    _lib.nea_debug_inject(int(flags))


_prof_keep = None


def nea_set_profile_events(events) -> None:
    """Records the given torch.cuda.Event objects at kernel boundaries of later
    calls (see include/nea_attn.h); ``None`` disables."""
    global _prof_keep
    if not events:
        _prof_keep = None
        _lib.nea_set_profile_events(None, 0)
        return
    arr = (ctypes.c_void_p * len(events))(*[ctypes.c_void_p(e.cuda_event) for e in events])
    _prof_keep = (arr, list(events))
    _lib.nea_set_profile_events(arr, len(events))


def nea_attn_decode(q, kc, vc, lens, rope_base: float = 10000.0, o=None, lse=None, stream=None):
    """Decode attention of one query per sequence over a key/value cache:
    ``q [B, Hq, D]`` (un-rotated, the token at position ``lens[b]-1``),
    ``kc, vc [B, Tc, Hkv, D]`` (keys already rotated at their positions),
    ``lens`` int32 ``[B]`` on the same device.  Returns ``(o [B, Hq, D],
    lse [B, Hq])``."""
    import torch

    if q.dim() != 3 or kc.dim() != 4:
        raise ValueError("q must be [B, Hq, D] and kc, vc [B, Tc, Hkv, D]")
    B, Hq, D = q.shape
    Tc, Hkv = kc.shape[1], kc.shape[2]
    dev, dt = q.device, q.dtype
    code = _dtype_code(q)
    _check(kc, "kc", (B, Tc, Hkv, D), dt, dev)
    _check(vc, "vc", (B, Tc, Hkv, D), dt, dev)
    _check(lens, "lens", (B,), torch.int32, dev)
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=dev)
    _check(o, "o", (B, Hq, D), dt, dev)
    _check(lse, "lse", (B, Hq), torch.float32, dev)
    rc = _lib.nea_attn_decode(_ptr(q), _ptr(kc), _ptr(vc), _ptr(lens), _ptr(o), _ptr(lse), B, Tc, Hq, Hkv, D, code,
                              float(rope_base), _stream(stream))
    if rc != NEA_OK:
        raise NeaError(rc, "nea_attn_decode")
    return o, lse

