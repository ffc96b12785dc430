"""The seeded input recipe (no GPU): shapes, storage types and spreads of the
benchmark and parity workloads, and that a seed fixes every value."""
import math

import pytest
import torch

from causal_gqa_attention_sm_b200.workloads import WORKLOADS, custom, make_decode_inputs, make_inputs


def test_configurations_follow_the_model_shapes():
    # GPU model: 12 query heads, 4 kv heads, head dim 64; CPU model: 4 / 2 heads, dim 32
    for name in ("layer", "long", "stack", "sweep512", "sweep1024", "sweep2048", "sweep4096"):
        w = WORKLOADS[name]
        assert (w.Hq, w.Hkv, w.D, w.G) == (12, 4, 64, 3), name
        assert w.causal and w.rope_base == 10000.0
    t = WORKLOADS["tiny"]
    assert (t.B, t.T, t.Hq, t.Hkv, t.D, t.dtype) == (1, 128, 4, 2, 32, "f32")
    assert (WORKLOADS["long"].B, WORKLOADS["long"].T, WORKLOADS["long"].dtype) == (4, 1024, "f32")
    assert WORKLOADS["stack"].layers == 16
    for T in (512, 1024, 2048, 4096):  # the sweep keeps B*T fixed
        w = WORKLOADS[f"sweep{T}"]
        assert w.B * w.T == 16384 and w.dtype == "bf16"
    for name in ("decode1024", "decode4096"):
        assert WORKLOADS[name].decode and WORKLOADS[name].B == 16


@pytest.mark.parametrize("name", ["tiny", "layer"])
def test_inputs_have_the_stated_shapes_and_spreads(name):
    w = WORKLOADS[name]
    x = make_inputs(w)
    assert x["q"].shape == (w.B, w.T, w.Hq, w.D) and x["do"].shape == (w.B, w.T, w.Hq, w.D)
    assert x["k"].shape == (w.B, w.T, w.Hkv, w.D) and x["v"].shape == (w.B, w.T, w.Hkv, w.D)
    assert all(t.dtype == w.torch_dtype and t.is_contiguous() for t in x.values())
    for n, want in (("q", w.qk_std), ("k", w.qk_std), ("v", w.v_std), ("do", w.do_std)):
        t = x[n].double()
        tol = 6.0 / math.sqrt(t.numel())  # several standard errors of the sample moments
        assert abs(t.mean().item()) < want * tol * 2, (n, t.mean().item())
        assert abs(t.std().item() / want - 1.0) < tol * 2, (n, t.std().item(), want)


def test_long_has_peaked_logits_and_layer_a_small_upstream_gradient():
    assert WORKLOADS["long"].qk_std == 3.0
    assert WORKLOADS["layer"].do_std == 0.1


def test_seed_fixes_every_value_and_layers_differ():
    w = custom(B=2, T=5, Hq=4, Hkv=2, D=32, seed=77)
    a, b = make_inputs(w), make_inputs(w)
    assert all(torch.equal(a[n], b[n]) for n in a)
    c = make_inputs(w, layer=1)
    assert not torch.equal(a["q"], c["q"])


def test_bf16_inputs_are_the_rounded_float32_draws():
    w32 = custom(B=1, T=9, Hq=2, Hkv=1, D=32, seed=5)
    w16 = custom(B=1, T=9, Hq=2, Hkv=1, D=32, seed=5, dtype="bf16")
    a, b = make_inputs(w32), make_inputs(w16)
    assert torch.equal(a["q"].to(torch.bfloat16), b["q"])


def test_decode_inputs():
    w = custom(B=3, T=40, Hq=6, Hkv=2, D=64, seed=9, decode=True)
    x = make_decode_inputs(w)
    assert x["q"].shape == (3, 6, 64)
    assert x["kc"].shape == (3, 40, 2, 64) and x["vc"].shape == (3, 40, 2, 64)
    assert x["lens"].dtype == torch.int32 and x["lens"].tolist() == [40, 40, 40]
    assert w.cache_bytes() == 2 * 3 * 40 * 2 * 64 * 4
    assert w.tokens() == 3
