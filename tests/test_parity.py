"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the
same seeded inputs.

Tolerances: float32 storage -- O and LSE max-abs <= 2e-3, dQ/dK/dV relative
Frobenius <= 5e-3; bfloat16 storage -- O and LSE max-abs <= 2e-2, O and
gradients relative Frobenius <= 2e-2.  Small shapes are compared in full;
the full-size workloads run on the GPU exactly as the benchmark launches them
and are compared on sampled (batch, kv-group) slices, which the oracle
computes independently because batches and kv groups do not interact."""
import math
import os

import numpy as np
import pytest

import oracle
from causal_gqa_attention_sm_b200.workloads import WORKLOADS, custom, make_inputs

pytestmark = pytest.mark.gpu

# absolute bound on a gradient whose exact value is zero
ZERO_GRAD_ABS = {"f32": 1e-4, "bf16": 1e-2}

TOL = {
    "f32": dict(o_abs=2e-3, lse_abs=2e-3, grad_rel=5e-3, o_rel=5e-3),
    "bf16": dict(o_abs=2e-2, lse_abs=2e-2, grad_rel=2e-2, o_rel=2e-2),
}


@pytest.fixture(scope="module", autouse=True)
def _oracle_threads():
    oracle.set_threads(len(os.sched_getaffinity(0)))


def rel_fro(a, b):
    return float(np.linalg.norm((a - b).ravel()) / max(np.linalg.norm(b.ravel()), 1e-30))


def to64(t):
    return t.detach().float().cpu().double().numpy()


def run_gpu(nea, w, inp):
    import torch

    dev = {n: t.cuda() for n, t in inp.items()}
    o, lse = nea.nea_attn_fwd(dev["q"], dev["k"], dev["v"], w.rope_base, w.causal)
    dq, dk, dv = nea.nea_attn_bwd(dev["q"], dev["k"], dev["v"], o, lse, dev["do"], w.rope_base, w.causal)
    torch.cuda.synchronize()
    assert nea.nea_device_status() == nea.NEA_OK
    return {"o": to64(o), "lse": to64(lse), "dq": to64(dq), "dk": to64(dk), "dv": to64(dv)}


def compare(w, got, ref, where=""):
    tol = TOL[w.dtype]
    o_abs = float(np.abs(got["o"] - ref["o"]).max()) if ref["o"].size else 0.0
    lse_abs = float(np.abs(got["lse"] - ref["lse"]).max()) if ref["lse"].size else 0.0
    errs = {"o_abs": o_abs, "lse_abs": lse_abs, "o_rel": rel_fro(got["o"], ref["o"])}
    for n in ("dq", "dk", "dv"):
        if np.linalg.norm(ref[n]) == 0.0:
            # identically zero true gradient (T = 1: dS = P (dP - Dv) = 0); the
            # relative error is undefined, so bound the absolute rounding noise
            errs[n] = float(np.abs(got[n]).max()) / (tol["grad_rel"] / ZERO_GRAD_ABS[w.dtype])
        else:
            errs[n] = rel_fro(got[n], ref[n])
    msg = f"{w.name}{where}: {errs}"
    _record(w.name + where, errs)
    assert np.isfinite(got["o"]).all() and np.isfinite(got["dq"]).all(), msg
    assert errs["o_abs"] <= tol["o_abs"], msg
    assert errs["lse_abs"] <= tol["lse_abs"], msg
    assert errs["o_rel"] <= tol["o_rel"], msg
    for n in ("dq", "dk", "dv"):
        assert errs[n] <= tol["grad_rel"], msg
    return errs


def _record(name, errs):
    """Appends the measured errors to $NEA_PARITY_LOG (one JSON line per case)."""
    path = os.environ.get("NEA_PARITY_LOG")
    if path:
        import json

        with open(path, "a") as f:
            f.write(json.dumps({"case": name, **{k: float(v) for k, v in errs.items()}}) + "\n")


def oracle_ref(w, inp, b=None, g=None):
    """Oracle on the whole input, or on batch b / kv group g only."""
    q, k, v, do = (to64(inp[n]) for n in ("q", "k", "v", "do"))
    if b is not None:
        G = w.G
        q, do = q[b:b + 1, :, g * G:(g + 1) * G], do[b:b + 1, :, g * G:(g + 1) * G]
        k, v = k[b:b + 1, :, g:g + 1], v[b:b + 1, :, g:g + 1]
    o, lse = oracle.attn_fwd(q, k, v, w.rope_base, w.causal)
    dq, dk, dv = oracle.attn_bwd(q, k, v, do, w.rope_base, w.causal)
    return {"o": o, "lse": lse, "dq": dq, "dk": dk, "dv": dv}


def slice_got(w, got, b, g):
    G = w.G
    return {
        "o": got["o"][b:b + 1, :, g * G:(g + 1) * G], "dq": got["dq"][b:b + 1, :, g * G:(g + 1) * G],
        "lse": got["lse"][b:b + 1, g * G:(g + 1) * G], "dk": got["dk"][b:b + 1, :, g:g + 1],
        "dv": got["dv"][b:b + 1, :, g:g + 1],
    }


# ------------------------------------------------------------ small shapes, full comparison

EDGE = []
for dtype in ("f32", "bf16"):
    for D in (32, 64):
        for T in (1, 7, 127, 128, 129, 200, 256, 300):
            EDGE.append(custom(f"edge_{dtype}_D{D}_T{T}", B=2, T=T, Hq=6, Hkv=2, D=D, dtype=dtype, seed=T * 7 + D))
    for Hq, Hkv in ((4, 4), (4, 2), (6, 2), (8, 2)):  # G = 1, 2, 3, 4
        for causal in (True, False):
            EDGE.append(custom(f"gqa_{dtype}_{Hq}_{Hkv}_c{int(causal)}", B=1, T=257, Hq=Hq, Hkv=Hkv, D=64,
                               dtype=dtype, causal=causal, seed=11 * Hq + Hkv + causal))
    EDGE.append(custom(f"norope_{dtype}", B=2, T=190, Hq=4, Hkv=1, D=64, dtype=dtype, rope_base=0.0, seed=5))
EDGE.append(custom("peaked_f32", B=1, T=384, Hq=3, Hkv=1, D=64, dtype="f32", qk_std=3.0, seed=6))


@pytest.mark.parametrize("w", EDGE, ids=lambda w: w.name)
def test_small_shapes_full(cuda_lib, w):
    inp = make_inputs(w)
    compare(w, run_gpu(cuda_lib, w, inp), oracle_ref(w, inp))


# head dimension 128, bfloat16 storage: ragged and single-row sequences, GQA
# and MHA, causal and full, rotation off, a longer sequence
D128 = [custom("d128_causal", B=2, T=300, Hq=6, Hkv=2, D=128, dtype="bf16", seed=128),
        custom("d128_full", B=1, T=257, Hq=4, Hkv=4, D=128, dtype="bf16", causal=False, seed=129),
        custom("d128_T1", B=2, T=1, Hq=4, Hkv=2, D=128, dtype="bf16", seed=130),
        custom("d128_T128_norope", B=1, T=128, Hq=8, Hkv=2, D=128, dtype="bf16", rope_base=0.0, seed=131),
        custom("d128_long", B=1, T=1024, Hq=6, Hkv=2, D=128, dtype="bf16", seed=132)]


@pytest.mark.parametrize("w", D128, ids=lambda w: w.name)
def test_d128_full(cuda_lib, w):
    """Head dimension 128 (bfloat16 storage): forward and backward against the
    oracle at the bf16 tolerances."""
    inp = make_inputs(w)
    compare(w, run_gpu(cuda_lib, w, inp), oracle_ref(w, inp))


def test_peaked_bf16_within_rounding_bound(cuda_lib):
    """bf16 storage with peaked logits (Q, K ~ N(0, 9)): the rotated q', k' are
    rounded to bf16 (relative error <= 2^-9 each), so every score carries
    |ds| <= 2^-8 * scale * sum_d |q'_d k'_d| =: eps_s.  Then |dLSE| <= eps_s and
    |dO| <= 2 eps_s max|v| + 2^-8 max|O| (output rounding).  The fixed bf16
    tolerance (2e-2) holds for the N(0, 1) workloads; here the bound is derived
    from the inputs and checked with a factor-2 margin on the rounding model."""
    w = custom("peaked_bf16", B=1, T=384, Hq=3, Hkv=1, D=64, dtype="bf16", qk_std=3.0, seed=6)
    inp = make_inputs(w)
    got = run_gpu(cuda_lib, w, inp)
    ref = oracle_ref(w, inp)
    qa = np.abs(oracle.rope(to64(inp["q"]), w.rope_base))[0].transpose(1, 0, 2)   # [H, T, D]
    ka = np.abs(oracle.rope(to64(inp["k"]), w.rope_base))[0, :, 0]                 # [T, D]
    eps_s = 2.0 ** -8 / math.sqrt(w.D) * float((qa @ ka.T).max())
    vmax = float(np.abs(to64(inp["v"])).max())
    o_bound = 2 * eps_s * vmax + 2.0 ** -8 * float(np.abs(ref["o"]).max())
    lse_err = float(np.abs(got["lse"] - ref["lse"]).max())
    o_err = float(np.abs(got["o"] - ref["o"]).max())
    _record(w.name, {"o_abs": o_err, "lse_abs": lse_err, "eps_s": eps_s, "o_bound": o_bound})
    assert lse_err <= 2 * eps_s, (lse_err, eps_s)
    assert o_err <= 2 * o_bound, (o_err, o_bound)
    for n in ("dq", "dk", "dv"):  # gradients are measured relative to their norm
        assert rel_fro(got[n], ref[n]) <= 2e-2, n


def test_tiny_config_full(cuda_lib):
    w = WORKLOADS["tiny"]
    inp = make_inputs(w)
    compare(w, run_gpu(cuda_lib, w, inp), oracle_ref(w, inp))


# ------------------------------------------------------------ full-size workloads, sampled slices

def _samples(w, n):
    rng = np.random.default_rng(w.seed)
    pairs = {(0, 0), (w.B - 1, w.Hkv - 1)}
    while len(pairs) < min(n, w.B * w.Hkv):
        pairs.add((int(rng.integers(w.B)), int(rng.integers(w.Hkv))))
    return sorted(pairs)


def oracle_slices(w, inp, pairs):
    """Oracle on several (batch, kv group) slices at once: each slice becomes
    one batch element with G query heads and one kv head, so the oracle's
    parallel loop runs over the slices."""
    G = w.G
    q, k, v, do = (to64(inp[n]) for n in ("q", "k", "v", "do"))
    qs = np.concatenate([q[b:b + 1, :, g * G:(g + 1) * G] for b, g in pairs])
    dos = np.concatenate([do[b:b + 1, :, g * G:(g + 1) * G] for b, g in pairs])
    ks = np.concatenate([k[b:b + 1, :, g:g + 1] for b, g in pairs])
    vs = np.concatenate([v[b:b + 1, :, g:g + 1] for b, g in pairs])
    o, lse = oracle.attn_fwd(qs, ks, vs, w.rope_base, w.causal)
    dq, dk, dv = oracle.attn_bwd(qs, ks, vs, dos, w.rope_base, w.causal)
    return [{"o": o[i:i + 1], "lse": lse[i:i + 1], "dq": dq[i:i + 1], "dk": dk[i:i + 1], "dv": dv[i:i + 1]}
            for i in range(len(pairs))]


@pytest.mark.parametrize("name", ["layer", "long", "sweep512", "sweep1024", "sweep2048", "sweep4096", "d128"])
def test_full_size_sampled(cuda_lib, name):
    w = WORKLOADS[name]
    inp = make_inputs(w)
    got = run_gpu(cuda_lib, w, inp)
    pairs = _samples(w, 4 if w.T <= 1024 else 2)
    for (b, g), ref in zip(pairs, oracle_slices(w, inp, pairs)):
        compare(w, slice_got(w, got, b, g), ref, where=f" b={b} g={g}")
    # every softmax row sums to one under the GPU's LSE (checked on slice 0 in fp64)
    check_row_sums(w, inp, got, 0, 0)


def check_row_sums(w, inp, got, b, h):
    q = oracle.rope(to64(inp["q"])[b:b + 1, :, h:h + 1], w.rope_base)[0, :, 0]
    k = oracle.rope(to64(inp["k"])[b:b + 1, :, h // w.G:h // w.G + 1], w.rope_base)[0, :, 0]
    s = q @ k.T / math.sqrt(w.D)
    if w.causal:
        s[np.triu_indices(w.T, 1)] = -np.inf
    lse = got["lse"][b, h]
    sums = np.exp(s - lse[:, None]).sum(1)
    tol = 5e-3 if w.dtype == "f32" else 5e-2
    assert np.abs(sums - 1).max() < tol


def test_stack_sixteen_layers_sampled(cuda_lib):
    w = WORKLOADS["stack"]
    for layer in range(w.layers):
        inp = make_inputs(w, layer)
        got = run_gpu(cuda_lib, w, inp)
        pairs = [(layer % w.B, layer % w.Hkv)]
        compare(w, slice_got(w, got, *pairs[0]), oracle_slices(w, inp, pairs)[0], where=f" layer={layer}")


# ------------------------------------------------------------ boundary behaviour on the GPU

def test_outputs_do_not_spill_past_their_extent(cuda_lib):
    """Ragged T: bytes after each output tensor stay untouched."""
    import torch

    w = custom("canary", B=1, T=131, Hq=3, Hkv=1, D=64, dtype="f32", seed=9)
    inp = {n: t.cuda() for n, t in make_inputs(w).items()}
    pad = 4096
    def canary(shape):
        buf = torch.full((int(np.prod(shape)) + pad,), 1234.5, device="cuda")
        return buf, buf[: int(np.prod(shape))].view(shape)
    ob, o = canary((1, 131, 3, 64))
    lb, lse = canary((1, 3, 131))
    cuda_lib.nea_attn_fwd(inp["q"], inp["k"], inp["v"], w.rope_base, True, o=o, lse=lse)
    qb, dq = canary((1, 131, 3, 64))
    kb, dk = canary((1, 131, 1, 64))
    vb, dv = canary((1, 131, 1, 64))
    cuda_lib.nea_attn_bwd(inp["q"], inp["k"], inp["v"], o, lse, inp["do"], w.rope_base, True, dq=dq, dk=dk, dv=dv)
    torch.cuda.synchronize()
    for buf, n in ((ob, o.numel()), (lb, lse.numel()), (qb, dq.numel()), (kb, dk.numel()), (vb, dv.numel())):
        assert torch.all(buf[n:] == 1234.5)


def test_empty_inputs_are_noops(cuda_lib):
    import torch

    for B, T in ((0, 64), (2, 0)):
        q = torch.zeros((B, T, 4, 64), device="cuda")
        k = torch.zeros((B, T, 2, 64), device="cuda")
        o, lse = cuda_lib.nea_attn_fwd(q, k, k)
        dq, dk, dv = cuda_lib.nea_attn_bwd(q, k, k, o, lse, q)
        assert o.shape == q.shape and dk.shape == k.shape
    assert cuda_lib.nea_device_status() == cuda_lib.NEA_OK


def test_rejects_misaligned_pointer(cuda_lib):
    import torch

    buf = torch.zeros(1 * 8 * 2 * 64 + 1, device="cuda")
    q = buf[1:].view(1, 8, 2, 64)  # 4-byte offset
    k = torch.zeros((1, 8, 1, 64), device="cuda")
    with pytest.raises(cuda_lib.NeaError) as ei:
        cuda_lib.nea_attn_fwd(q, k, k)
    assert ei.value.status == cuda_lib.NEA_ERR_ARG


@pytest.mark.parametrize("D", [64, 128])
def test_repeated_calls_are_deterministic(cuda_lib, D):
    """Bitwise-identical outputs over repeated calls; at D = 128 this also
    guards the gradient kernel's reliance on the issue order of its MMAs (a
    product overwriting P or dS before the previous one read it would show
    as run-to-run differences)."""
    w = custom("det", B=2, T=300 if D == 64 else 1000, Hq=6 if D == 64 else 8, Hkv=2, D=D, dtype="bf16", seed=3)
    inp = make_inputs(w)
    a = run_gpu(cuda_lib, w, inp)
    for _ in range(1 if D == 64 else 8):
        b = run_gpu(cuda_lib, w, inp)
        for n in a:
            assert np.array_equal(a[n], b[n]), n


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_nan_key_reaches_every_later_output_row(cuda_lib, dtype):
    """A NaN in one key makes every output row that sees that key NaN and
    leaves earlier rows finite.  Key 7 sits in a column pair whose bf16
    exponentials are taken by the polynomial on the FMA pipe, so this also
    checks that the polynomial lets NaN through."""
    import torch

    w = custom("nan_key", B=1, T=160, Hq=2, Hkv=1, D=64, dtype=dtype, seed=5)
    inp = {n: t.cuda() for n, t in make_inputs(w).items()}
    inp["k"][0, 7, 0, 3] = float("nan")
    o, lse = cuda_lib.nea_attn_fwd(inp["q"], inp["k"], inp["v"], w.rope_base, True)
    torch.cuda.synchronize()
    assert cuda_lib.nea_device_status() == cuda_lib.NEA_OK
    o = o.float().cpu()
    assert torch.isfinite(o[0, :7]).all()
    assert torch.isnan(o[0, 7:]).all()
