"""The decoder-block steps beside the attention (nea_block_*): host-side
argument checks (no GPU) and GPU parity with the fp64 oracle
(``oracle.block_ref``) on seeded inputs.

Tolerances, relative Frobenius per output: float32 storage 2e-4 (every
product in split bf16, about 2^-16 relative, fp32 accumulation over at most a
few thousand terms); bfloat16 storage 2e-2 (the normalised input y and the
operands in bf16, as in the attention's bf16 path)."""
import ctypes
import os

import numpy as np
import pytest

from oracle import block_ref

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIB = os.path.join(ROOT, "causal_gqa_attention_sm_b200", "libnea.so")
TOL = {"f32": 2e-4, "bf16": 2e-2}


@pytest.fixture(scope="module")
def lib():
    import __graft_entry__

    __graft_entry__.build()
    return ctypes.CDLL(LIB)


@pytest.mark.parametrize("kw", [dict(C=96), dict(C=0), dict(D=4), dict(Hq=5), dict(Hkv=3), dict(M=-1),
                                dict(dtype=4), dict(ptr=None), dict(ptr=8)])
def test_block_bad_arguments_rejected_without_launch(lib, kw):
    a = dict(M=256, C=128, Hq=4, Hkv=2, D=32, dtype=0, ptr=16)
    a.update(kw)
    vp = ctypes.c_void_p
    p = vp(a["ptr"]) if a["ptr"] is not None else None
    f = lib.nea_block_qkv_fwd
    f.argtypes = [vp] * 8 + [ctypes.c_int] * 6 + [vp]
    assert f(*([p] * 8), a["M"], a["C"], a["Hq"], a["Hkv"], a["D"], a["dtype"], None) == 1
    f = lib.nea_block_out_fwd
    f.argtypes = [vp] * 4 + [ctypes.c_int] * 5 + [vp]
    if "Hkv" not in kw:
        assert f(*([p] * 4), a["M"], a["C"], a["Hq"], a["D"], a["dtype"], None) == 1


def test_block_empty_is_a_noop(lib):
    vp = ctypes.c_void_p
    f = lib.nea_block_qkv_bwd
    f.argtypes = [vp] * 14 + [ctypes.c_int] * 6 + [vp]
    assert f(*([None] * 14), 0, 128, 4, 2, 32, 0, None) == 0


# ----------------------------------------------------------------- GPU parity
def make(B, T, C, Hq, Hkv, D, dtype, seed):
    import torch

    tdt = {"f32": torch.float32, "bf16": torch.bfloat16}[dtype]
    g = torch.Generator().manual_seed(seed)
    r = lambda *s, std=1.0: (torch.randn(*s, generator=g) * std).to(tdt)
    return dict(x=r(B, T, C), g=(1.0 + 0.1 * torch.randn(C, generator=g)).to(tdt),
                Wq=r(C, Hq * D, std=C ** -0.5), Wk=r(C, Hkv * D, std=C ** -0.5), Wv=r(C, Hkv * D, std=C ** -0.5),
                Wo=r(Hq * D, C, std=(Hq * D) ** -0.5), o=r(B, T, Hq, D), dq=r(B, T, Hq, D), dk=r(B, T, Hkv, D),
                dv=r(B, T, Hkv, D), dh=r(B, T, C))


def to64(t):
    return t.detach().float().cpu().double().numpy()


def rel(a, b):
    return float(np.linalg.norm((a - b).ravel()) / max(np.linalg.norm(b.ravel()), 1e-30))


CASES = [
    (1, 128, 128, 4, 2, 32, "f32"),
    (1, 128, 128, 4, 2, 32, "bf16"),
    (2, 100, 256, 8, 2, 64, "f32"),      # M = 200: a ragged token tile
    (2, 100, 256, 8, 2, 64, "bf16"),
    (8, 512, 768, 12, 4, 64, "f32"),     # the GPU model layer
    (8, 512, 768, 12, 4, 64, "bf16"),
]


@pytest.mark.gpu
@pytest.mark.parametrize("case", CASES, ids=[f"{c[6]}-M{c[0] * c[1]}-C{c[2]}" for c in CASES])
def test_block_steps_match_oracle(cuda_lib, case):
    import torch

    nea = cuda_lib
    B, T, C, Hq, Hkv, D, dtype = case
    inp = make(B, T, C, Hq, Hkv, D, dtype, seed=B * T + C)
    d = {n: t.cuda() for n, t in inp.items()}
    q, k, v = nea.nea_block_qkv_fwd(d["x"], d["g"], d["Wq"], d["Wk"], d["Wv"], Hq, Hkv, D)
    h = nea.nea_block_out_fwd(d["x"], d["o"], d["Wo"])
    do, dWo = nea.nea_block_out_bwd(d["o"], d["Wo"], d["dh"])
    dx, dg, dWq, dWk, dWv = nea.nea_block_qkv_bwd(d["x"], d["g"], d["Wq"], d["Wk"], d["Wv"], d["dq"], d["dk"],
                                                  d["dv"], dres=d["dh"])
    torch.cuda.synchronize()
    assert nea.nea_device_status() == nea.NEA_OK
    a = {n: to64(t) for n, t in inp.items()}
    rq, rk, rv, y, rstd = block_ref.qkv_fwd(a["x"], a["g"], a["Wq"], a["Wk"], a["Wv"], Hq, Hkv, D)
    rh = block_ref.out_fwd(a["x"], a["o"], a["Wo"])
    rdres, rdo, rdWo = block_ref.out_bwd(a["o"], a["Wo"], a["dh"])
    rdx, rdg, rdWq, rdWk, rdWv = block_ref.qkv_bwd(a["x"], a["g"], a["Wq"], a["Wk"], a["Wv"], y, rstd, a["dq"],
                                                   a["dk"], a["dv"])
    rdx = rdx + rdres
    tol = TOL[dtype]
    errs = {n: rel(to64(got), ref) for n, got, ref in (
        ("q", q, rq), ("k", k, rk), ("v", v, rv), ("h", h, rh), ("do", do, rdo), ("dWo", dWo, rdWo),
        ("dx", dx, rdx), ("dg", dg, rdg), ("dWq", dWq, rdWq), ("dWk", dWk, rdWk), ("dWv", dWv, rdWv))}
    assert all(e <= tol for e in errs.values()), errs


@pytest.mark.gpu
def test_block_backward_without_residual_gradient(cuda_lib):
    """dres = NULL: dx is the norm's input gradient alone."""
    import torch

    nea = cuda_lib
    B, T, C, Hq, Hkv, D = 1, 256, 128, 4, 2, 32
    inp = make(B, T, C, Hq, Hkv, D, "f32", seed=7)
    d = {n: t.cuda() for n, t in inp.items()}
    dx, dg, *_ = nea.nea_block_qkv_bwd(d["x"], d["g"], d["Wq"], d["Wk"], d["Wv"], d["dq"], d["dk"], d["dv"])
    torch.cuda.synchronize()
    a = {n: to64(t) for n, t in inp.items()}
    _, _, _, y, rstd = block_ref.qkv_fwd(a["x"], a["g"], a["Wq"], a["Wk"], a["Wv"], Hq, Hkv, D)
    rdx, rdg, *_ = block_ref.qkv_bwd(a["x"], a["g"], a["Wq"], a["Wk"], a["Wv"], y, rstd, a["dq"], a["dk"], a["dv"])
    assert rel(to64(dx), rdx) <= TOL["f32"] and rel(to64(dg), rdg) <= TOL["f32"]


# ----------------------------------------------------------------- SwiGLU feed-forward
@pytest.mark.parametrize("kw", [dict(C=96), dict(F=96), dict(F=0), dict(C=8192), dict(M=-1), dict(dtype=4),
                                dict(ptr=None), dict(ptr=8)])
def test_ffn_bad_arguments_rejected_without_launch(lib, kw):
    a = dict(M=256, C=128, F=256, dtype=0, ptr=16)
    a.update(kw)
    vp = ctypes.c_void_p
    p = vp(a["ptr"]) if a["ptr"] is not None else None
    f = lib.nea_block_ffn_fwd
    f.argtypes = [vp] * 8 + [ctypes.c_int] * 4 + [vp]
    assert f(*([p] * 8), a["M"], a["C"], a["F"], a["dtype"], None) == 1
    f = lib.nea_block_ffn_bwd
    f.argtypes = [vp] * 13 + [ctypes.c_int] * 4 + [vp]
    assert f(*([p] * 13), a["M"], a["C"], a["F"], a["dtype"], None) == 1


def test_ffn_empty_is_a_noop(lib):
    vp = ctypes.c_void_p
    f = lib.nea_block_ffn_bwd
    f.argtypes = [vp] * 13 + [ctypes.c_int] * 4 + [vp]
    assert f(*([None] * 13), 0, 128, 256, 0, None) == 0


def make_ffn(B, T, C, F, dtype, seed):
    import torch

    tdt = {"f32": torch.float32, "bf16": torch.bfloat16}[dtype]
    g = torch.Generator().manual_seed(seed)
    r = lambda *s, std=1.0: (torch.randn(*s, generator=g) * std).to(tdt)
    return dict(x=r(B, T, C), g=(1.0 + 0.1 * torch.randn(C, generator=g)).to(tdt), Wg=r(C, F, std=C ** -0.5),
                Wu=r(C, F, std=C ** -0.5), Wd=r(F, C, std=F ** -0.5), dh=r(B, T, C))


FFN_CASES = [
    (1, 128, 128, 256, "f32"),
    (1, 128, 128, 256, "bf16"),
    (2, 100, 256, 320, "f32"),      # M = 200 and F = 320: ragged token and width tiles
    (2, 100, 256, 320, "bf16"),
    (1, 64, 64, 64, "f32"),         # one partial tile everywhere
    (1, 1000, 768, 3072, "f32"),    # ragged token tiles in split-K products of 256-wide tiles
    (1, 1000, 768, 3072, "bf16"),
    (8, 512, 768, 3072, "f32"),     # the GPU model layer, F = 4 C
    (8, 512, 768, 3072, "bf16"),
]


@pytest.mark.gpu
@pytest.mark.parametrize("case", FFN_CASES, ids=[f"{c[4]}-M{c[0] * c[1]}-C{c[2]}-F{c[3]}" for c in FFN_CASES])
def test_ffn_matches_oracle(cuda_lib, case):
    import torch

    nea = cuda_lib
    B, T, C, F, dtype = case
    inp = make_ffn(B, T, C, F, dtype, seed=B * T + C + F)
    d = {n: t.cuda() for n, t in inp.items()}
    h, ga, gb = nea.nea_block_ffn_fwd(d["x"], d["g"], d["Wg"], d["Wu"], d["Wd"])
    dx, dg, dWg, dWu, dWd = nea.nea_block_ffn_bwd(d["x"], d["g"], d["Wg"], d["Wu"], d["Wd"], ga, gb, d["dh"])
    h2, none_a, none_b = nea.nea_block_ffn_fwd(d["x"], d["g"], d["Wg"], d["Wu"], d["Wd"], save=False)
    torch.cuda.synchronize()
    assert nea.nea_device_status() == nea.NEA_OK
    assert none_a is None and none_b is None and torch.equal(h, h2)  # saving a and b does not change h
    a = {n: to64(t) for n, t in inp.items()}
    rh, sv = block_ref.ffn_fwd(a["x"], a["g"], a["Wg"], a["Wu"], a["Wd"])
    rdx, rdg, rdWg, rdWu, rdWd = block_ref.ffn_bwd(a["x"], a["g"], a["Wg"], a["Wu"], a["Wd"], sv, a["dh"])
    tol = TOL[dtype]
    errs = {n: rel(to64(got).reshape(ref.shape), ref) for n, got, ref in (
        ("h", h, rh), ("a", ga, sv["a"]), ("b", gb, sv["b"]), ("dx", dx, rdx), ("dg", dg, rdg), ("dWg", dWg, rdWg),
        ("dWu", dWu, rdWu), ("dWd", dWd, rdWd))}
    assert all(e <= tol for e in errs.values()), errs


@pytest.mark.gpu
def test_ffn_saturated_gate(cuda_lib):
    """Gate pre-activations far in both tails (|a| up to ~100): silu and its
    derivative stay finite and match the oracle (exp(-a) overflows to inf for
    a < -88 in fp32; silu and the derivative then go to 0)."""
    import torch

    nea = cuda_lib
    B, T, C, F = 1, 128, 128, 128
    inp = make_ffn(B, T, C, F, "f32", seed=11)
    inp["Wg"] = inp["Wg"] * 40.0
    d = {n: t.cuda() for n, t in inp.items()}
    h, ga, gb = nea.nea_block_ffn_fwd(d["x"], d["g"], d["Wg"], d["Wu"], d["Wd"])
    dx, dg, dWg, dWu, dWd = nea.nea_block_ffn_bwd(d["x"], d["g"], d["Wg"], d["Wu"], d["Wd"], ga, gb, d["dh"])
    torch.cuda.synchronize()
    a = {n: to64(t) for n, t in inp.items()}
    rh, sv = block_ref.ffn_fwd(a["x"], a["g"], a["Wg"], a["Wu"], a["Wd"])
    assert np.abs(sv["a"]).max() > 88.0  # the test reaches the overflow region
    ref = block_ref.ffn_bwd(a["x"], a["g"], a["Wg"], a["Wu"], a["Wd"], sv, a["dh"])
    for got, r in zip((h, dx, dg, dWg, dWu, dWd), (rh,) + tuple(ref)):
        assert torch.isfinite(got).all()
        assert rel(to64(got).reshape(r.shape), r) <= TOL["f32"]
