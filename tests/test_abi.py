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


def test_nonfinite_rope_base_rejected(lib):
    assert _fwd(lib, base=float("nan")) == 1


def test_empty_problem_is_a_noop(lib):
    assert _fwd(lib, B=0, ptr=None) == 0
    assert _fwd(lib, T=0, ptr=None) == 0
    assert _bwd(lib, B=0, ptr=None) == 0


def test_status_strings(lib):
    lib.nea_status_string.restype = ctypes.c_char_p
    for code in range(6):
        assert lib.nea_status_string(code).startswith(b"NEA_")
    assert lib.nea_version() >= 100
