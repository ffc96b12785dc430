"""fp64 CPU oracle for causal GQA attention with RoPE, forward and backward.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``, never by the product package.  The
arithmetic lives in ``attn_ref.c`` (plain C, double precision, the full
T x T score matrix per head); this module only marshals numpy arrays.

Every function takes and returns float64 arrays in the library's layout:
Q, O, dO, dQ ``[B, T, Hq, D]``; K, V, dK, dV ``[B, T, Hkv, D]``;
LSE and the row term ``Dvec`` ``[B, Hq, T]``.

``block_ref`` (numpy, float64) holds the steps on either side of the
attention in a decoder block: the RMSNorm pre-norm with the Q/K/V
projections, and the output projection with the residual add; its pins are
in ``tests/test_block_oracle.py``.

Parity pins: every function here is checked in ``tests/test_oracle.py``
against closed forms, invariants, central finite differences and a library
cross-check; see the header of ``attn_ref.c`` for the passages each step
follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_ref.c")
_LIB = os.path.join(_HERE, "liboracle.so")

_dp = ctypes.POINTER(ctypes.c_double)


def build(force: bool = False) -> str:
    """Compiles ``attn_ref.c`` into ``liboracle.so`` with gcc and OpenMP."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-Wall",
               "-o", _LIB + ".tmp", _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        i = ctypes.c_int
        d = ctypes.c_double
        lib.oracle_attn_fwd.argtypes = [_dp, _dp, _dp, _dp, _dp, i, i, i, i, i, d, i]
        lib.oracle_attn_bwd.argtypes = [_dp, _dp, _dp, _dp, _dp, _dp, _dp, _dp, _dp, _dp,
                                        i, i, i, i, i, d, i]
        lib.oracle_attn_probs.argtypes = [_dp, _dp, _dp, i, i, i, i, i, d, i, i, i]
        lib.oracle_rope.argtypes = [_dp, _dp, i, i, i, i, d]
        lib.oracle_attn_decode.argtypes = [_dp, _dp, _dp, ctypes.POINTER(ctypes.c_int), _dp, _dp,
                                           i, i, i, i, i, d]
        lib.oracle_set_threads.argtypes = [i]
        lib.oracle_get_threads.restype = i
        for f in (lib.oracle_attn_fwd, lib.oracle_attn_bwd, lib.oracle_attn_probs, lib.oracle_rope,
                  lib.oracle_attn_decode):
            f.restype = i
        _lib = lib
    return _lib


def _c(a: np.ndarray) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float64)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(_dp)


def set_threads(n: int) -> None:
    """Sets the OpenMP thread count the oracle uses."""
    _load().oracle_set_threads(int(n))


def get_threads() -> int:
    return int(_load().oracle_get_threads())


def _shape(q, k):
    B, T, Hq, D = q.shape
    Bk, Tk, Hkv, Dk = k.shape
    if (Bk, Tk, Dk) != (B, T, D):
        raise ValueError("Q and K/V shapes disagree")
    return B, T, Hq, Hkv, D


def _check(rc: int) -> None:
    if rc != 0:
        raise ValueError(f"oracle returned status {rc}")


def rope(x: np.ndarray, base: float) -> np.ndarray:
    """R_t x for every head vector of ``x [B, T, H, D]`` (interleaved pairs)."""
    x = _c(x)
    y = np.empty_like(x)
    B, T, H, D = x.shape
    _check(_load().oracle_rope(_ptr(x), _ptr(y), B, T, H, D, float(base)))
    return y


def attn_fwd(q, k, v, rope_base: float = 10000.0, causal: bool = True):
    """Returns ``(O, LSE)`` of causal (or full) GQA attention with RoPE."""
    q, k, v = _c(q), _c(k), _c(v)
    B, T, Hq, Hkv, D = _shape(q, k)
    o = np.zeros_like(q)
    lse = np.zeros((B, Hq, T), dtype=np.float64)
    _check(_load().oracle_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                                   B, T, Hq, Hkv, D, float(rope_base), int(bool(causal))))
    return o, lse


def attn_bwd(q, k, v, do, rope_base: float = 10000.0, causal: bool = True, extras: bool = False):
    """Returns ``(dQ, dK, dV)``; with ``extras`` also ``(O, LSE, Dvec)``."""
    q, k, v, do = _c(q), _c(k), _c(v), _c(do)
    B, T, Hq, Hkv, D = _shape(q, k)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    o = np.zeros_like(q) if extras else None
    lse = np.zeros((B, Hq, T)) if extras else None
    dvec = np.zeros((B, Hq, T)) if extras else None
    _check(_load().oracle_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(do), _ptr(dq), _ptr(dk),
                                   _ptr(dv), _ptr(o), _ptr(lse), _ptr(dvec),
                                   B, T, Hq, Hkv, D, float(rope_base), int(bool(causal))))
    if extras:
        return dq, dk, dv, o, lse, dvec
    return dq, dk, dv


def attn_probs(q, k, b: int, h: int, rope_base: float = 10000.0, causal: bool = True):
    """Dense ``[T, T]`` softmax probabilities of batch ``b``, query head ``h``."""
    q, k = _c(q), _c(k)
    B, T, Hq, Hkv, D = _shape(q, k)
    p = np.zeros((T, T), dtype=np.float64)
    _check(_load().oracle_attn_probs(_ptr(q), _ptr(k), _ptr(p), B, T, Hq, Hkv, D,
                                     float(rope_base), int(bool(causal)), int(b), int(h)))
    return p


def attn_decode(q, kc, vc, lens, rope_base: float = 10000.0):
    """Decode attention of one query per sequence over a key/value cache.

    ``q [B, Hq, D]`` un-rotated query of the token at position ``lens[b]-1``;
    ``kc, vc [B, Tc, Hkv, D]`` the cache (keys already rotated at their
    positions); ``lens [B]`` valid lengths.  Returns ``(O [B, Hq, D],
    LSE [B, Hq])``; an empty cache gives O = 0 and LSE = -inf.
    """
    q, kc, vc = _c(q), _c(kc), _c(vc)
    B, Hq, D = q.shape
    _, Tc, Hkv, _ = kc.shape
    ln = np.ascontiguousarray(lens, dtype=np.int32)
    o = np.zeros_like(q)
    lse = np.zeros((B, Hq), dtype=np.float64)
    _check(_load().oracle_attn_decode(_ptr(q), _ptr(kc), _ptr(vc), ln.ctypes.data_as(ctypes.POINTER(ctypes.c_int)),
                                      _ptr(o), _ptr(lse), B, Tc, Hq, Hkv, D, float(rope_base)))
    return o, lse
