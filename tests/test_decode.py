"""Decode attention over a key/value cache (nea_attn_decode): host-side
argument checks (no GPU) and GPU parity with the fp64 oracle."""
import ctypes
import os

import numpy as np
import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIB = os.path.join(ROOT, "causal_gqa_attention_sm_b200", "libnea.so")
BASE = 10000.0


@pytest.fixture(scope="module")
def lib():
    import __graft_entry__

    __graft_entry__.build()
    return ctypes.CDLL(LIB)


def _decode(lib, B=2, Tc=8, Hq=4, Hkv=2, D=64, dtype=0, ptr=16, lens=16, base=10000.0):
    f = lib.nea_attn_decode
    vp = ctypes.c_void_p
    f.argtypes = [vp] * 6 + [ctypes.c_int] * 6 + [ctypes.c_float, vp]
    p = vp(ptr) if ptr is not None else None
    return f(p, p, p, vp(lens) if lens is not None else None, p, p, B, Tc, Hq, Hkv, D, dtype, base, None)


@pytest.mark.parametrize("kw", [
    dict(D=48), dict(Hq=5, Hkv=2), dict(Hq=18, Hkv=2), dict(Hkv=0), dict(B=-1), dict(Tc=0), dict(dtype=3),
    dict(ptr=None), dict(ptr=8), dict(lens=None), dict(lens=18), dict(base=float("inf")),
])
def test_decode_bad_arguments_rejected_without_launch(lib, kw):
    assert _decode(lib, **kw) == 1  # NEA_ERR_ARG


def test_decode_empty_batch_is_a_noop(lib):
    assert _decode(lib, B=0, ptr=None, lens=None) == 0


# ----------------------------------------------------------------- GPU parity
TOL = {"f32": (2e-3, 2e-3), "bf16": (2e-2, 2e-2)}  # (O max-abs, LSE max-abs)


def _case(B, Tc, Hq, Hkv, D, dtype, lens, seed, rope=True):
    """Seeded cache (keys rotated by the oracle at their positions, then
    stored in the storage type) and queries; the oracle sees exactly the
    stored values."""
    import torch

    tdt = {"f32": torch.float32, "bf16": torch.bfloat16}[dtype]
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, Hq, D, generator=g).to(tdt)
    k = torch.randn(B, Tc, Hkv, D, generator=g)
    v = torch.randn(B, Tc, Hkv, D, generator=g).to(tdt)
    base = BASE if rope else 0.0
    kc = torch.from_numpy(oracle.rope(k.double().numpy(), base) if rope else k.double().numpy()).to(tdt)
    lens = np.asarray(lens, dtype=np.int32)
    o_ref, lse_ref = oracle.attn_decode(q.double().numpy(), kc.double().numpy(), v.double().numpy(), lens, base)
    return q, kc, v, lens, base, o_ref, lse_ref


def _run(nea, q, kc, v, lens, base):
    import torch

    o, lse = nea.nea_attn_decode(q.cuda(), kc.cuda(), v.cuda(), torch.from_numpy(lens).cuda(), base)
    torch.cuda.synchronize()
    assert nea.nea_device_status() == nea.NEA_OK
    return o.double().cpu().numpy(), lse.double().cpu().numpy()


def _compare(o, lse, o_ref, lse_ref, dtype):
    to, tl = TOL[dtype]
    live = np.isfinite(lse_ref)
    assert np.all(np.isneginf(lse[~live])) and np.all(o[~live] == 0.0)
    assert np.abs(o - o_ref).max() <= to, np.abs(o - o_ref).max()
    assert np.abs(lse[live] - lse_ref[live]).max() <= tl


CASES = [
    # B, Tc, Hq, Hkv, D, dtype, lens
    (3, 300, 12, 4, 64, "f32", [1, 129, 300]),
    (3, 300, 12, 4, 64, "bf16", [300, 128, 7]),
    (2, 257, 4, 2, 32, "f32", [257, 256]),
    (2, 257, 8, 1, 32, "bf16", [1, 200]),
    (4, 128, 6, 6, 64, "bf16", [128, 127, 64, 0]),
    # G = 4 .. 7 (lanes per row 4 or 8, pieces of 64 or 32 rows)
    (2, 190, 8, 2, 64, "f32", [190, 31]),
    (2, 190, 10, 2, 64, "bf16", [33, 190]),
    (2, 150, 12, 2, 32, "f32", [150, 65]),
    (2, 150, 14, 2, 32, "bf16", [1, 150]),
    # one (sequence, kv head) spread over every CTA (ranges of a few pieces each)
    (1, 20000, 3, 1, 64, "bf16", [19999]),
    (1, 9000, 3, 1, 64, "f32", [9000]),
    # many short sequences: one CTA's range crosses several (sequence, kv head) pairs
    (300, 70, 6, 2, 32, "bf16", [(7 * i) % 71 for i in range(300)]),
    (40, 5, 8, 2, 64, "f32", [i % 6 for i in range(40)]),
    # head dimension 128 (two 64-column arrays per cached line for bf16, four for fp32)
    (3, 300, 8, 2, 128, "bf16", [300, 129, 1]),
    (3, 300, 8, 2, 128, "f32", [1, 257, 300]),
    (2, 190, 8, 8, 128, "bf16", [190, 64]),
    (2, 190, 16, 2, 128, "bf16", [33, 190]),
    (2, 190, 16, 2, 128, "f32", [190, 2]),
    (1, 9000, 4, 1, 128, "bf16", [8999]),
]


@pytest.mark.gpu
@pytest.mark.parametrize("case", CASES, ids=[f"{c[5]}-T{c[1]}-G{c[2] // c[3]}-D{c[4]}" for c in CASES])
def test_decode_parity(cuda_lib, case):
    B, Tc, Hq, Hkv, D, dtype, lens = case
    q, kc, v, ln, base, o_ref, lse_ref = _case(B, Tc, Hq, Hkv, D, dtype, lens, seed=sum(lens) + Tc)
    o, lse = _run(cuda_lib, q, kc, v, ln, base)
    _compare(o, lse, o_ref, lse_ref, dtype)


@pytest.mark.gpu
def test_decode_calls_of_different_shapes_in_turn(cuda_lib):
    """The per-(sequence, kv head) piece counts are left at zero by every call:
    calls of different shapes, one after another on one stream, each match the
    oracle."""
    cases = [(3, 300, 12, 4, 64, "f32", [300, 1, 0]), (9, 1000, 6, 3, 64, "bf16", [1000, 999, 500] * 3),
             (3, 300, 12, 4, 64, "f32", [300, 1, 0]), (1, 64, 2, 2, 32, "f32", [64])]
    prepared = [_case(*c, seed=17 + i) for i, c in enumerate(cases)]
    for c, (q, kc, v, ln, base, o_ref, lse_ref) in zip(cases, prepared):
        o, lse = _run(cuda_lib, q, kc, v, ln, base)
        _compare(o, lse, o_ref, lse_ref, c[5])


@pytest.mark.gpu
def test_decode_without_rotation(cuda_lib):
    q, kc, v, ln, base, o_ref, lse_ref = _case(2, 200, 12, 4, 64, "f32", [200, 33], seed=5, rope=False)
    o, lse = _run(cuda_lib, q, kc, v, ln, base)
    _compare(o, lse, o_ref, lse_ref, "f32")


@pytest.mark.gpu
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_decode_full_size(cuda_lib, dtype):
    """The benchmark's decode shape (B=16, Tc=4096, Hq=12, Hkv=4, D=64) with
    ragged lengths over the whole range."""
    rng = np.random.default_rng(11)
    lens = np.concatenate([[1, 4096, 4095, 128, 129], rng.integers(1, 4097, size=11)])
    q, kc, v, ln, base, o_ref, lse_ref = _case(16, 4096, 12, 4, 64, dtype, lens, seed=99)
    o, lse = _run(cuda_lib, q, kc, v, ln, base)
    _compare(o, lse, o_ref, lse_ref, dtype)


@pytest.mark.gpu
def test_decode_length_out_of_range_is_reported(cuda_lib):
    """A cache length above Tc is clamped on the device and reported by the
    next status read; the context stays usable."""
    import torch

    q, kc, v, ln, base, o_ref, lse_ref = _case(2, 64, 4, 2, 64, "f32", [64, 10], seed=3)
    bad = torch.tensor([65, 10], dtype=torch.int32, device="cuda")
    cuda_lib.nea_attn_decode(q.cuda(), kc.cuda(), v.cuda(), bad, base)
    assert cuda_lib.nea_device_status() == cuda_lib.NEA_ERR_ARG
    o, lse = _run(cuda_lib, q, kc, v, ln, base)
    _compare(o, lse, o_ref, lse_ref, "f32")
