"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every function include/nea_attn.h declares, and rejects bad arguments before
touching the device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "nea_attn.h")
LIB = os.path.join(ROOT, "causal_gqa_attention_sm_b200", "libnea.so")


@pytest.fixture(scope="module")
def lib():
    import __graft_entry__

    __graft_entry__.build()
    return ctypes.CDLL(LIB)


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(nea_[a-z_0-9]+)\s*\(", src)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("nea_attn_fwd", "nea_attn_bwd", "nea_status_string", "nea_device_status"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for n in declared_functions():
        assert hasattr(lib, n), n


def _fwd(lib, B=1, T=4, Hq=4, Hkv=2, D=64, dtype=0, causal=1, ptr=16, base=10000.0):
    f = lib.nea_attn_fwd
    vp = ctypes.c_void_p
    f.argtypes = [vp] * 5 + [ctypes.c_int] * 6 + [ctypes.c_float, ctypes.c_int, vp]
    p = vp(ptr) if ptr is not None else None
    return f(p, p, p, p, p, B, T, Hq, Hkv, D, dtype, base, causal, None)


def _bwd(lib, B=1, T=4, Hq=4, Hkv=2, D=64, dtype=0, causal=1, ptr=16):
    f = lib.nea_attn_bwd
    vp = ctypes.c_void_p
    f.argtypes = [vp] * 9 + [ctypes.c_int] * 6 + [ctypes.c_float, ctypes.c_int, vp]
    p = vp(ptr) if ptr is not None else None
    return f(*([p] * 9), B, T, Hq, Hkv, D, dtype, 10000.0, causal, None)


@pytest.mark.parametrize("kw", [
    dict(D=48), dict(D=128), dict(Hq=5, Hkv=2), dict(Hkv=0), dict(B=-1), dict(T=-3), dict(dtype=7),
    dict(causal=2), dict(ptr=None), dict(ptr=8), dict(ptr=20),
])
def test_bad_arguments_are_rejected_without_launch(lib, kw):
    assert _fwd(lib, **kw) == 1  # NEA_ERR_ARG
    assert _bwd(lib, **kw) == 1


def test_d128_is_a_bf16_variant(lib):
    """D = 128 passes the checks with bfloat16 storage only."""
    assert _fwd(lib, D=128, dtype=1, B=0, ptr=None) == 0  # accepted: the empty problem is a no-op
    assert _bwd(lib, D=128, dtype=1, B=0, ptr=None) == 0
    assert _fwd(lib, D=128, dtype=1, ptr=None) == 1       # and its pointers are checked
    assert _bwd(lib, D=128, dtype=1, ptr=None) == 1
    assert _fwd(lib, D=128, dtype=0) == 1
    assert _bwd(lib, D=128, dtype=0) == 1
    nq, nk = 2 * 100 * 6 * 128, 2 * 100 * 2 * 128  # bf16 with the rotation: rotated Q and K
    assert _saved_bytes(lib, D=128, dtype=1) == (2 * nq + 255) // 256 * 256 + (2 * nk + 255) // 256 * 256
    assert _saved_bytes(lib, D=128, dtype=0) == -1


def test_nonfinite_rope_base_rejected(lib):
    assert _fwd(lib, base=float("nan")) == 1


def test_empty_problem_is_a_noop(lib):
    assert _fwd(lib, B=0, ptr=None) == 0
    assert _fwd(lib, T=0, ptr=None) == 0
    assert _bwd(lib, B=0, ptr=None) == 0


def _saved_bytes(lib, B=2, T=100, Hq=6, Hkv=2, D=64, dtype=0, base=10000.0):
    f = lib.nea_attn_saved_bytes
    f.argtypes = [ctypes.c_int] * 6 + [ctypes.c_float]
    f.restype = ctypes.c_longlong
    return f(B, T, Hq, Hkv, D, dtype, base)


def test_saved_bytes_closed_form(lib):
    def r256(x):
        return (x + 255) // 256 * 256

    nq, nk = 2 * 100 * 6 * 64, 2 * 100 * 2 * 64
    # float32: hi and lo bf16 planes of rotated Q, K and of V
    assert _saved_bytes(lib) == 2 * (r256(2 * nq) + 2 * r256(2 * nk))
    # bfloat16 with the rotation on: rotated Q and K only
    assert _saved_bytes(lib, dtype=1) == r256(2 * nq) + r256(2 * nk)
    # bfloat16 without rotation: nothing to save; float32 keeps its planes
    assert _saved_bytes(lib, dtype=1, base=0.0) == 0
    assert _saved_bytes(lib, base=0.0) == _saved_bytes(lib)
    assert _saved_bytes(lib, B=0) == 0
    assert _saved_bytes(lib, D=48) == -1
    assert _saved_bytes(lib, base=float("inf")) == -1


def test_saved_pair_rejects_missing_buffer(lib):
    vp = ctypes.c_void_p
    f = lib.nea_attn_fwd_save
    f.argtypes = [vp] * 6 + [ctypes.c_int] * 6 + [ctypes.c_float, ctypes.c_int, vp]
    p = vp(16)
    assert f(p, p, p, p, p, None, 1, 4, 4, 2, 64, 0, 10000.0, 1, None) == 1   # saved needed, NULL
    assert f(p, p, p, p, p, vp(24), 1, 4, 4, 2, 64, 0, 10000.0, 1, None) == 1  # misaligned
    g = lib.nea_attn_bwd_saved
    g.argtypes = [vp] * 10 + [ctypes.c_int] * 6 + [ctypes.c_float, ctypes.c_int, vp]
    assert g(p, p, p, p, p, p, None, p, p, p, 1, 4, 4, 2, 64, 0, 10000.0, 1, None) == 1
    assert g(p, p, p, p, p, p, p, p, p, p, 1, 4, 4, 2, 48, 0, 10000.0, 1, None) == 1
    assert g(*([None] * 10), 0, 4, 4, 2, 64, 0, 10000.0, 1, None) == 0  # empty: no-op


def test_status_strings(lib):
    lib.nea_status_string.restype = ctypes.c_char_p
    for code in range(6):
        assert lib.nea_status_string(code).startswith(b"NEA_")
    assert lib.nea_version() >= 100
