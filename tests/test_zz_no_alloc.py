"""The scratch-free backward entry point, nea_attn_bwd_noalloc.

It serves callers that may not allocate device memory (their device memory
is owned by a host-side manager, or an allocation would synchronise the device
at the wrong moment); its scratch is a fixed array inside the library.  The
GPU test calls it through the C ABI twice in a row -- two different problems,
so the second call reuses scratch the first one left behind -- and compares
each result with the regular backward, nea_attn_bwd, within the tolerances of
the parity tests.  This file is collected last on purpose."""
import ctypes

import numpy as np
import pytest

from causal_gqa_attention_sm_b200.workloads import custom, make_inputs

GRAD_REL = {"f32": 5e-3, "bf16": 2e-2}


def _rel(a, b):
    a = a.float().cpu().double().numpy()
    b = b.float().cpu().double().numpy()
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def _call_noalloc(nea, t, w, dq, dk, dv):
    import torch

    p = lambda x: ctypes.c_void_p(x.data_ptr())  # noqa: E731
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    code = nea.NEA_F32 if w.dtype == "f32" else nea.NEA_BF16
    return nea._lib.nea_attn_bwd_noalloc(p(t["q"]), p(t["k"]), p(t["v"]), p(t["o"]), p(t["lse"]), p(t["do"]),
                                         p(dq), p(dk), p(dv), w.B, w.T, w.Hq, w.Hkv, w.D, code,
                                         float(w.rope_base), int(w.causal), stream)


@pytest.mark.gpu
def test_noalloc_backward_matches_regular_backward_twice(cuda_lib):
    import torch

    nea = cuda_lib
    cases = [custom("noalloc_a", B=2, T=300, Hq=6, Hkv=2, D=64, dtype="f32", seed=41),
             custom("noalloc_b", B=1, T=513, Hq=4, Hkv=1, D=32, dtype="bf16", seed=42)]
    for w in cases:
        t = {n: x.cuda() for n, x in make_inputs(w).items()}
        t["o"], t["lse"] = nea.nea_attn_fwd(t["q"], t["k"], t["v"], w.rope_base, w.causal)
        ref = nea.nea_attn_bwd(t["q"], t["k"], t["v"], t["o"], t["lse"], t["do"], w.rope_base, w.causal)
        got = [torch.full_like(r, float("nan")) for r in ref]
        rc = _call_noalloc(nea, t, w, *got)
        assert rc == nea.NEA_OK, nea.nea_status_string(rc)
        torch.cuda.synchronize()
        for name, g, r in zip(("dq", "dk", "dv"), got, ref):
            assert torch.isfinite(g).all(), (w.name, name)
            assert _rel(g, r) <= GRAD_REL[w.dtype], (w.name, name, _rel(g, r))


def test_noalloc_rejects_problems_beyond_its_scratch():
    """B*Hq*T + T*D beyond the fixed 1 Mi floats: refused before any launch."""
    import causal_gqa_attention_sm_b200 as nea

    vp = ctypes.c_void_p(256)
    rc = nea._lib.nea_attn_bwd_noalloc(vp, vp, vp, vp, vp, vp, vp, vp, vp, 64, 4096, 12, 4, 64, nea.NEA_BF16,
                                       10000.0, 1, None)
    assert rc == nea.NEA_ERR_SCRATCH_LIMIT
    assert "scratch" in nea.nea_status_string(rc)
