"""GPU tests of the save-for-backward pair (nea_attn_fwd_save, nea_attn_bwd_saved):
their outputs are bit-identical to nea_attn_fwd / nea_attn_bwd on the same
inputs, they agree with the oracle, and the backward reads only the caller's
buffer -- calls that reuse the library workspace in between change nothing."""
import numpy as np
import pytest

from causal_gqa_attention_sm_b200.workloads import WORKLOADS, custom, make_inputs
from test_parity import compare, oracle_ref, to64

pytestmark = pytest.mark.gpu

CASES = [
    custom("saved_f32_D64", B=2, T=300, Hq=6, Hkv=2, D=64, dtype="f32", seed=21),
    custom("saved_bf16_D64", B=2, T=257, Hq=4, Hkv=2, D=64, dtype="bf16", seed=22),
    custom("saved_f32_D32_noncausal", B=1, T=200, Hq=4, Hkv=1, D=32, dtype="f32", causal=False, seed=23),
    custom("saved_bf16_norope", B=1, T=190, Hq=4, Hkv=1, D=64, dtype="bf16", rope_base=0.0, seed=24),
    custom("saved_f32_norope", B=1, T=129, Hq=2, Hkv=2, D=64, dtype="f32", rope_base=0.0, seed=25),
]


def _dev(inp):
    return {n: t.cuda() for n, t in inp.items()}


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_saved_pair_matches_regular_calls_bitwise(cuda_lib, w):
    import torch

    nea = cuda_lib
    d = _dev(make_inputs(w))
    o0, lse0 = nea.nea_attn_fwd(d["q"], d["k"], d["v"], w.rope_base, w.causal)
    dq0, dk0, dv0 = nea.nea_attn_bwd(d["q"], d["k"], d["v"], o0, lse0, d["do"], w.rope_base, w.causal)
    o1, lse1, saved = nea.nea_attn_fwd_save(d["q"], d["k"], d["v"], w.rope_base, w.causal)
    assert saved.numel() == nea.nea_attn_saved_bytes(w.B, w.T, w.Hq, w.Hkv, w.D, w.torch_dtype, w.rope_base)
    dq1, dk1, dv1 = nea.nea_attn_bwd_saved(d["q"], d["k"], d["v"], o1, lse1, d["do"], saved, w.rope_base, w.causal)
    torch.cuda.synchronize()
    assert nea.nea_device_status() == nea.NEA_OK
    for a, b in ((o0, o1), (lse0, lse1), (dq0, dq1), (dk0, dk1), (dv0, dv1)):
        assert torch.equal(a, b)
    got = {"o": to64(o1), "lse": to64(lse1), "dq": to64(dq1), "dk": to64(dk1), "dv": to64(dv1)}
    compare(w, got, oracle_ref(w, make_inputs(w)))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_saved_planes_survive_other_calls(cuda_lib, dtype):
    """fwd_save(A), then a full forward and backward of another problem B (same
    shapes, so the workspace is reused), then bwd_saved(A): A's gradients are
    those of A."""
    import torch

    nea = cuda_lib
    wa = custom(f"order_a_{dtype}", B=1, T=256, Hq=4, Hkv=2, D=64, dtype=dtype, seed=31)
    wb = custom(f"order_b_{dtype}", B=1, T=256, Hq=4, Hkv=2, D=64, dtype=dtype, seed=32)
    a, b = _dev(make_inputs(wa)), _dev(make_inputs(wb))
    oa, lsea, saved = nea.nea_attn_fwd_save(a["q"], a["k"], a["v"], wa.rope_base, wa.causal)
    ob, lseb = nea.nea_attn_fwd(b["q"], b["k"], b["v"], wb.rope_base, wb.causal)
    nea.nea_attn_bwd(b["q"], b["k"], b["v"], ob, lseb, b["do"], wb.rope_base, wb.causal)
    dqa, dka, dva = nea.nea_attn_bwd_saved(a["q"], a["k"], a["v"], oa, lsea, a["do"], saved, wa.rope_base,
                                           wa.causal)
    ref = nea.nea_attn_bwd(a["q"], a["k"], a["v"], oa, lsea, a["do"], wa.rope_base, wa.causal)
    torch.cuda.synchronize()
    assert nea.nea_device_status() == nea.NEA_OK
    for x, y in zip((dqa, dka, dva), ref):
        assert torch.equal(x, y)


def test_saved_bench_workload_sampled(cuda_lib):
    """The benchmarked step (float32 storage, B=4 T=1024 Hq=12 Hkv=4 D=64) through
    the saved pair equals the regular calls bit for bit."""
    import torch

    nea = cuda_lib
    w = WORKLOADS["long"]
    d = _dev(make_inputs(w))
    o0, lse0 = nea.nea_attn_fwd(d["q"], d["k"], d["v"], w.rope_base, w.causal)
    g0 = nea.nea_attn_bwd(d["q"], d["k"], d["v"], o0, lse0, d["do"], w.rope_base, w.causal)
    o1, lse1, saved = nea.nea_attn_fwd_save(d["q"], d["k"], d["v"], w.rope_base, w.causal)
    g1 = nea.nea_attn_bwd_saved(d["q"], d["k"], d["v"], o1, lse1, d["do"], saved, w.rope_base, w.causal)
    torch.cuda.synchronize()
    assert nea.nea_device_status() == nea.NEA_OK
    assert torch.equal(o0, o1) and torch.equal(lse0, lse1)
    for x, y in zip(g0, g1):
        assert torch.equal(x, y)


def test_saved_buffer_too_small_is_rejected(cuda_lib):
    import torch

    nea = cuda_lib
    w = CASES[0]
    d = _dev(make_inputs(w))
    need = nea.nea_attn_saved_bytes(w.B, w.T, w.Hq, w.Hkv, w.D, w.torch_dtype, w.rope_base)
    with pytest.raises(ValueError):
        nea.nea_attn_fwd_save(d["q"], d["k"], d["v"], w.rope_base, w.causal,
                              saved=torch.empty(need - 16, dtype=torch.uint8, device="cuda"))
