"""The scratch-free backward entry point, nea_attn_bwd_noalloc.

It serves callers that may not allocate device memory (their device memory
is owned by a host-side manager or a pre-planned arena, or an allocation
would synchronise the device at the wrong moment); its scratch is a fixed
array inside the library.  The GPU tests call it through the C ABI on several
problems in a row -- each call reuses the scratch the previous one left
behind -- and compare every result with the fp64 oracle at the tolerances of
the parity tests.  They also run its bounded-wait failure path: a withheld
arrival must surface as NEA_ERR_TIMEOUT through nea_device_status (which
itself allocates nothing), and the next call must be clean.

Each test sets up everything it uses, so the file passes alone in a fresh
process as well as after the rest of the suite; it is named to be collected
last so that a run stopping at the first failure has run every other test."""
import ctypes
import os

import numpy as np
import pytest

import oracle
from causal_gqa_attention_sm_b200.workloads import custom, make_inputs

# the parity tolerances: relative Frobenius per gradient
GRAD_REL = {"f32": 5e-3, "bf16": 2e-2}


def _rel(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def _call_noalloc(nea, t, w, dq, dk, dv):
    import torch

    p = lambda x: ctypes.c_void_p(x.data_ptr())  # noqa: E731
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    code = nea.NEA_F32 if w.dtype == "f32" else nea.NEA_BF16
    return nea._lib.nea_attn_bwd_noalloc(p(t["q"]), p(t["k"]), p(t["v"]), p(t["o"]), p(t["lse"]), p(t["do"]),
                                         p(dq), p(dk), p(dv), w.B, w.T, w.Hq, w.Hkv, w.D, code,
                                         float(w.rope_base), int(w.causal), stream)


def _problem(nea, w):
    """Device inputs, with O and LSE from the library's forward."""
    t = {n: x.cuda() for n, x in make_inputs(w).items()}
    t["o"], t["lse"] = nea.nea_attn_fwd(t["q"], t["k"], t["v"], w.rope_base, w.causal)
    return t


CASES = [
    custom("noalloc_f32", B=2, T=300, Hq=6, Hkv=2, D=64, dtype="f32", seed=41),
    custom("noalloc_bf16_d32", B=1, T=513, Hq=4, Hkv=1, D=32, dtype="bf16", seed=42),
    # rotation off: the bf16 path then reads Q and K in place (another scratch layout)
    custom("noalloc_bf16_norope", B=2, T=200, Hq=4, Hkv=2, D=64, dtype="bf16", seed=43, rope_base=0.0),
    custom("noalloc_f32_full", B=1, T=257, Hq=3, Hkv=1, D=64, dtype="f32", seed=44, causal=False),
]


@pytest.mark.gpu
def test_noalloc_backward_matches_oracle_on_consecutive_calls(cuda_lib):
    import torch

    nea = cuda_lib
    oracle.set_threads(len(os.sched_getaffinity(0)))
    for w in CASES:
        t = _problem(nea, w)
        got = [torch.full_like(t[n], float("nan")) for n in ("q", "k", "v")]
        rc = _call_noalloc(nea, t, w, *got)
        assert rc == nea.NEA_OK, nea.nea_status_string(rc)
        assert nea.nea_device_status() == nea.NEA_OK, w.name
        h = {n: x.float().cpu().double().numpy() for n, x in make_inputs(w).items()}
        ref = oracle.attn_bwd(h["q"], h["k"], h["v"], h["do"], w.rope_base, w.causal)
        for name, g, r in zip(("dq", "dk", "dv"), got, ref):
            g = g.float().cpu().double().numpy()
            assert np.isfinite(g).all(), (w.name, name)
            assert _rel(g, r) <= GRAD_REL[w.dtype], (w.name, name, _rel(g, r))


@pytest.mark.gpu
def test_noalloc_wait_limit_is_reported_and_next_call_is_clean(cuda_lib):
    import torch

    nea = cuda_lib
    w = custom("noalloc_timeout", B=1, T=256, Hq=2, Hkv=1, D=64, dtype="f32", seed=45)
    t = _problem(nea, w)
    assert nea.nea_device_status() == nea.NEA_OK
    out = [torch.empty_like(t[n]) for n in ("q", "k", "v")]
    prev = nea.nea_set_wait_limit_ns(20_000_000)  # 20 ms per wait
    try:
        nea.nea_debug_inject(2)  # the next backward withholds its resident tiles
        assert _call_noalloc(nea, t, w, *out) == nea.NEA_OK  # the launch itself succeeds
        assert nea.nea_device_status() == nea.NEA_ERR_TIMEOUT
        assert nea.nea_device_status() == nea.NEA_OK  # read and cleared
    finally:
        nea.nea_set_wait_limit_ns(prev)
    assert _call_noalloc(nea, t, w, *out) == nea.NEA_OK
    assert nea.nea_device_status() == nea.NEA_OK
    h = {n: x.float().cpu().double().numpy() for n, x in make_inputs(w).items()}
    ref = oracle.attn_bwd(h["q"], h["k"], h["v"], h["do"], w.rope_base, w.causal)
    for g, r in zip(out, ref):
        assert _rel(g.float().cpu().double().numpy(), r) <= GRAD_REL["f32"]


def test_noalloc_rejects_problems_beyond_its_scratch():
    """Problems whose scratch exceeds the fixed 4 MiB array are refused before
    any CUDA call (so this runs without a GPU)."""
    import causal_gqa_attention_sm_b200 as nea

    vp = ctypes.c_void_p(256)
    rc = nea._lib.nea_attn_bwd_noalloc(vp, vp, vp, vp, vp, vp, vp, vp, vp, 64, 4096, 12, 4, 64, nea.NEA_BF16,
                                       10000.0, 1, None)
    assert rc == nea.NEA_ERR_SCRATCH_LIMIT
    assert "scratch" in nea.nea_status_string(rc)
