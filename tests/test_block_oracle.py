"""Pins of the fp64 block oracle (oracle/block_ref.py): the RMSNorm pre-norm,
the Q/K/V projections and the output projection with the residual, and the
SwiGLU feed-forward, forward and backward, checked against closed forms,
brute-force sums and central finite differences (no GPU)."""
import numpy as np
import pytest

from oracle import block_ref as br

H = 1e-6  # finite-difference step (float64)


def _fd(f, arrays, grads, rtol=1e-6, atol=1e-7):
    """Central differences of the scalar f() with respect to every element of
    every array, compared with the analytic gradients."""
    for a, ga in zip(arrays, grads):
        assert ga.shape == a.shape
        it = np.nditer(a, flags=["multi_index"])
        for _ in it:
            i = it.multi_index
            old = a[i]
            a[i] = old + H
            fp = f()
            a[i] = old - H
            fm = f()
            a[i] = old
            num = (fp - fm) / (2 * H)
            assert abs(num - ga[i]) <= atol + rtol * max(abs(num), abs(ga[i])), (i, num, ga[i])


def test_rmsnorm_closed_forms():
    g = np.array([1.0, 2.0, -0.5, 3.0])
    # a constant row c: rms = sqrt(c^2 + eps)
    c = 0.3
    y, rstd = br.rmsnorm_fwd(np.full((1, 1, 4), c), g)
    assert np.allclose(y[0, 0], c / np.sqrt(c * c + br.EPS) * g, rtol=0, atol=1e-15)
    assert np.allclose(rstd, 1 / np.sqrt(c * c + br.EPS))
    # no bias: a zero row maps to zero
    y0, _ = br.rmsnorm_fwd(np.zeros((1, 1, 4)), g)
    assert np.all(y0 == 0)
    # eps = 0, unit weights: every row has mean square 1, and scaling a row changes nothing
    x = np.random.default_rng(0).standard_normal((2, 3, 16))
    y1, _ = br.rmsnorm_fwd(x, np.ones(16), eps=0.0)
    assert np.allclose(np.mean(y1 * y1, axis=-1), 1.0, rtol=0, atol=1e-14)
    y2, _ = br.rmsnorm_fwd(7.5 * x, np.ones(16), eps=0.0)
    assert np.allclose(y1, y2, rtol=0, atol=1e-14)


def test_rmsnorm_backward_against_finite_differences():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((2, 3, 8))
    g = rng.standard_normal(8)
    dy = rng.standard_normal((2, 3, 8))
    y, rstd = br.rmsnorm_fwd(x, g)
    dx, dg = br.rmsnorm_bwd(x, g, rstd, dy)
    _fd(lambda: float(np.sum(dy * br.rmsnorm_fwd(x, g)[0])), [x, g], [dx, dg])


def test_projections_match_brute_force_sums():
    rng = np.random.default_rng(2)
    B, T, C, Hq, Hkv, D = 2, 3, 6, 4, 2, 2
    x = rng.standard_normal((B, T, C))
    g = rng.standard_normal(C)
    Wq, Wk, Wv = (rng.standard_normal((C, n * D)) for n in (Hq, Hkv, Hkv))
    q, k, v, y, rstd = br.qkv_fwd(x, g, Wq, Wk, Wv, Hq, Hkv, D)
    for b in range(B):
        for t in range(T):
            rms = np.sqrt(sum(x[b, t, c] ** 2 for c in range(C)) / C + br.EPS)
            yy = [x[b, t, c] / rms * g[c] for c in range(C)]
            for h in range(Hq):
                for d in range(D):
                    assert abs(q[b, t, h, d] - sum(yy[c] * Wq[c, h * D + d] for c in range(C))) < 1e-12
            for h in range(Hkv):
                for d in range(D):
                    assert abs(k[b, t, h, d] - sum(yy[c] * Wk[c, h * D + d] for c in range(C))) < 1e-12
                    assert abs(v[b, t, h, d] - sum(yy[c] * Wv[c, h * D + d] for c in range(C))) < 1e-12
    o = rng.standard_normal((B, T, Hq, D))
    Wo = rng.standard_normal((Hq * D, C))
    hh = br.out_fwd(x, o, Wo)
    for b in range(B):
        for t in range(T):
            for c in range(C):
                want = x[b, t, c] + sum(o[b, t, j // D, j % D] * Wo[j, c] for j in range(Hq * D))
                assert abs(hh[b, t, c] - want) < 1e-12


def test_projection_backwards_against_finite_differences():
    rng = np.random.default_rng(3)
    B, T, C, Hq, Hkv, D = 1, 3, 6, 4, 2, 2
    x = rng.standard_normal((B, T, C))
    g = rng.standard_normal(C)
    Wq, Wk, Wv = (rng.standard_normal((C, n * D)) for n in (Hq, Hkv, Hkv))
    dq, dk, dv = rng.standard_normal((B, T, Hq, D)), rng.standard_normal((B, T, Hkv, D)), rng.standard_normal(
        (B, T, Hkv, D))
    q, k, v, y, rstd = br.qkv_fwd(x, g, Wq, Wk, Wv, Hq, Hkv, D)
    grads = br.qkv_bwd(x, g, Wq, Wk, Wv, y, rstd, dq, dk, dv)

    def loss():
        q, k, v, _, _ = br.qkv_fwd(x, g, Wq, Wk, Wv, Hq, Hkv, D)
        return float(np.sum(dq * q) + np.sum(dk * k) + np.sum(dv * v))

    _fd(loss, [x, g, Wq, Wk, Wv], list(grads))
    o = rng.standard_normal((B, T, Hq, D))
    Wo = rng.standard_normal((Hq * D, C))
    dh = rng.standard_normal((B, T, C))
    dxr, do, dWo = br.out_bwd(o, Wo, dh)
    _fd(lambda: float(np.sum(dh * br.out_fwd(x, o, Wo))), [x, o, Wo], [dxr, do, dWo])


@pytest.mark.parametrize("causal", [True, False])
def test_whole_block_backward_against_finite_differences(causal):
    """Pre-norm, projections, the attention oracle with RoPE and GQA, output
    projection and residual, differentiated end to end."""
    rng = np.random.default_rng(4 + causal)
    B, T, C, Hq, Hkv, D = 1, 4, 8, 4, 2, 4
    x = rng.standard_normal((B, T, C))
    g = 1.0 + 0.1 * rng.standard_normal(C)
    Wq, Wk, Wv = (0.5 * rng.standard_normal((C, n * D)) for n in (Hq, Hkv, Hkv))
    Wo = 0.5 * rng.standard_normal((Hq * D, C))
    dh = rng.standard_normal((B, T, C))
    base = 10000.0
    h, saved = br.block_fwd(x, g, Wq, Wk, Wv, Wo, Hq, Hkv, D, base, causal)
    grads = br.block_bwd(x, g, Wq, Wk, Wv, Wo, saved, dh, base, causal)
    _fd(lambda: float(np.sum(dh * br.block_fwd(x, g, Wq, Wk, Wv, Wo, Hq, Hkv, D, base, causal)[0])),
        [x, g, Wq, Wk, Wv, Wo], list(grads))


# ----------------------------------------------------------------- SwiGLU feed-forward
def test_silu_closed_forms():
    assert br.silu(0.0) == 0.0
    assert abs(br.silu(1.0) - 1.0 / (1.0 + np.exp(-1.0))) < 1e-15
    z = np.linspace(-30, 30, 61)
    assert np.allclose(br.silu(z) - br.silu(-z), z, rtol=0, atol=1e-12)  # silu(z) - silu(-z) = z
    assert np.all(np.abs(br.silu(z[z < -20])) < 1e-6)                    # vanishes for large negative z
    assert np.allclose(br.silu(z[z > 20]), z[z > 20], rtol=0, atol=1e-6)  # tends to z for large positive z


def test_ffn_matches_brute_force_sums():
    rng = np.random.default_rng(7)
    B, T, C, F = 1, 2, 4, 6
    x, g = rng.standard_normal((B, T, C)), rng.standard_normal(C)
    Wg, Wu, Wd = rng.standard_normal((C, F)), rng.standard_normal((C, F)), rng.standard_normal((F, C))
    h, sv = br.ffn_fwd(x, g, Wg, Wu, Wd)
    for t in range(T):
        ms = sum(x[0, t, c] ** 2 for c in range(C)) / C
        y = [x[0, t, c] / (ms + br.EPS) ** 0.5 * g[c] for c in range(C)]
        act = []
        for f in range(F):
            a = sum(y[c] * Wg[c, f] for c in range(C))
            b = sum(y[c] * Wu[c, f] for c in range(C))
            act.append(a / (1.0 + np.exp(-a)) * b)
        for c in range(C):
            ref = x[0, t, c] + sum(act[f] * Wd[f, c] for f in range(F))
            assert abs(h[0, t, c] - ref) < 1e-12


def test_ffn_backward_against_finite_differences():
    rng = np.random.default_rng(8)
    B, T, C, F = 1, 3, 4, 5
    x, g = rng.standard_normal((B, T, C)), rng.standard_normal(C)
    Wg, Wu, Wd = rng.standard_normal((C, F)), rng.standard_normal((C, F)), rng.standard_normal((F, C))
    dh = rng.standard_normal((B, T, C))
    _, sv = br.ffn_fwd(x, g, Wg, Wu, Wd)
    dx, dg, dWg, dWu, dWd = br.ffn_bwd(x, g, Wg, Wu, Wd, sv, dh)
    _fd(lambda: float(np.sum(dh * br.ffn_fwd(x, g, Wg, Wu, Wd)[0])), [x, g, Wg, Wu, Wd], [dx, dg, dWg, dWu, dWd])


def test_ffn_backward_pin_catches_a_dropped_term():
    """A plausible mistake -- d silu(a)/da taken as sigmoid(a) -- fails the
    finite-difference pin."""
    rng = np.random.default_rng(9)
    B, T, C, F = 1, 2, 3, 4
    x, g = rng.standard_normal((B, T, C)), rng.standard_normal(C)
    Wg, Wu, Wd = rng.standard_normal((C, F)), rng.standard_normal((C, F)), rng.standard_normal((F, C))
    dh = rng.standard_normal((B, T, C))
    _, sv = br.ffn_fwd(x, g, Wg, Wu, Wd)
    a, b = sv["a"], sv["b"]
    dact = dh.reshape(B * T, C) @ Wd.T
    wrong = (sv["y"].reshape(B * T, C).T @ (dact * b / (1.0 + np.exp(-a))))
    with pytest.raises(AssertionError):
        _fd(lambda: float(np.sum(dh * br.ffn_fwd(x, g, Wg, Wu, Wd)[0])), [Wg], [wrong])
