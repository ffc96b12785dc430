"""Pins for the fp64 oracle: closed forms, invariants, finite differences and a
library cross-check.  None of these retypes the oracle's formulas; each checks
a consequence of the definition that a plausible slip (a dropped term, a wrong
sign or index, a transposed operand, a wrong pairing of the rotary halves)
would break."""
import json
import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rnd(seed, *shape, std=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * std


# ---------------------------------------------------------------- closed forms


def _eval_tree(x):
    env = {"__builtins__": {}, "log": math.log, "sqrt": math.sqrt, "cos": math.cos, "sin": math.sin}
    if isinstance(x, list):
        return [_eval_tree(e) for e in x]
    return float(eval(x, env))  # fixture strings: rationals and math functions only


def test_golden_two_token_worked_example():
    with open(os.path.join(GOLDEN, "two_token_worked_example.json")) as f:
        fx = json.load(f)
    s = fx["shape"]
    q, k, v, do = (np.array(_eval_tree(fx["inputs"][n])) for n in ("Q", "K", "V", "dO"))
    o, lse = oracle.attn_fwd(q, k, v, s["rope_base"], s["causal"])
    dq, dk, dv = oracle.attn_bwd(q, k, v, do, s["rope_base"], s["causal"])
    exp = {n: np.array(_eval_tree(fx["expected"][n])) for n in fx["expected"]}
    np.testing.assert_allclose(o, exp["O"], atol=1e-13)
    np.testing.assert_allclose(lse, exp["LSE"], atol=1e-13)
    np.testing.assert_allclose(dv, exp["dV"], atol=1e-13)
    np.testing.assert_allclose(dq, exp["dQ"], atol=1e-13)
    np.testing.assert_allclose(dk, exp["dK"], atol=1e-13)


@pytest.mark.parametrize("causal", [True, False])
def test_single_token_output_is_value(causal):
    B, Hq, Hkv, D = 2, 6, 2, 16
    q, k, v = rnd(1, B, 1, Hq, D), rnd(2, B, 1, Hkv, D), rnd(3, B, 1, Hkv, D)
    o, lse = oracle.attn_fwd(q, k, v, 10000.0, causal)
    G = Hq // Hkv
    for h in range(Hq):
        np.testing.assert_allclose(o[:, 0, h], v[:, 0, h // G], atol=1e-14)
        # position 0 turns by angle 0, so the score is the plain scaled dot product
        ref = (q[:, 0, h] * k[:, 0, h // G]).sum(-1) / math.sqrt(D)
        np.testing.assert_allclose(lse[:, h, 0], ref, atol=1e-13)


@pytest.mark.parametrize("which", ["zero_keys", "zero_queries", "identical_keys_no_rope"])
@pytest.mark.parametrize("causal", [True, False])
def test_equal_scores_give_prefix_mean(which, causal):
    B, T, Hq, Hkv, D = 1, 11, 4, 2, 8
    q, k, v = rnd(4, B, T, Hq, D), rnd(5, B, T, Hkv, D), rnd(6, B, T, Hkv, D)
    base = 10000.0
    if which == "zero_keys":
        k[:] = 0.0
    elif which == "zero_queries":
        q[:] = 0.0
    else:
        k[:] = k[:, :1]
        base = 0.0
        q[:] = q[:, :, :1]  # same query per row too, so each row's scores are equal
        q[:] = q[:, :1]
    o, lse = oracle.attn_fwd(q, k, v, base, causal)
    G = Hq // Hkv
    for h in range(Hq):
        for i in range(T):
            n = i + 1 if causal else T
            np.testing.assert_allclose(o[0, i, h], v[0, :n, h // G].mean(0), atol=1e-13)
            if which != "identical_keys_no_rope":
                np.testing.assert_allclose(lse[0, h, i], math.log(n), atol=1e-13)


# ---------------------------------------------------------------- invariants


@pytest.mark.parametrize("causal", [True, False])
def test_probability_rows(causal):
    B, T, Hq, Hkv, D = 2, 37, 3, 1, 16
    q, k = rnd(7, B, T, Hq, D, std=3.0), rnd(8, B, T, Hkv, D, std=3.0)
    for b in range(B):
        for h in range(Hq):
            p = oracle.attn_probs(q, k, b, h, 10000.0, causal)
            assert (p >= 0).all()
            np.testing.assert_allclose(p.sum(1), 1.0, atol=1e-13)
            if causal:
                assert np.all(np.triu(p, 1) == 0.0)
                assert np.all(np.diag(p) > 0)
            else:
                assert np.all(p > 0)


def test_lse_consistent_with_probs():
    """LSE_i = s_ij - ln P_ij for any visible j (pins LSE's log base and scale)."""
    B, T, Hq, Hkv, D = 1, 13, 2, 1, 8
    q, k, v = rnd(9, B, T, Hq, D), rnd(10, B, T, Hkv, D), rnd(11, B, T, Hkv, D)
    _, lse = oracle.attn_fwd(q, k, v, 0.0, True)
    for h in range(Hq):
        p = oracle.attn_probs(q, k, 0, h, 0.0, True)
        s = q[0, :, h] @ k[0, :, 0].T / math.sqrt(D)
        for i in range(T):
            np.testing.assert_allclose(s[i, : i + 1] - np.log(p[i, : i + 1]), lse[0, h, i], atol=1e-12)


@pytest.mark.parametrize("causal", [True, False])
def test_gqa_equals_mha_with_repeated_kv(causal):
    B, T, Hq, Hkv, D = 2, 19, 6, 2, 8
    G = Hq // Hkv
    q, k, v, do = rnd(12, B, T, Hq, D), rnd(13, B, T, Hkv, D), rnd(14, B, T, Hkv, D), rnd(15, B, T, Hq, D)
    kr, vr = np.repeat(k, G, axis=2), np.repeat(v, G, axis=2)
    o1, l1 = oracle.attn_fwd(q, k, v, 10000.0, causal)
    o2, l2 = oracle.attn_fwd(q, kr, vr, 10000.0, causal)
    np.testing.assert_allclose(o1, o2, atol=1e-13)
    np.testing.assert_allclose(l1, l2, atol=1e-13)
    dq1, dk1, dv1 = oracle.attn_bwd(q, k, v, do, 10000.0, causal)
    dq2, dk2, dv2 = oracle.attn_bwd(q, kr, vr, do, 10000.0, causal)
    np.testing.assert_allclose(dq1, dq2, atol=1e-12)
    np.testing.assert_allclose(dk1, dk2.reshape(B, T, Hkv, G, D).sum(3), atol=1e-12)
    np.testing.assert_allclose(dv1, dv2.reshape(B, T, Hkv, G, D).sum(3), atol=1e-12)


def test_bwd_row_term_equals_rowsum_do_o():
    """sum_j P_ij dP_ij = sum_d dO_id O_id (the identity the preprocess uses)."""
    B, T, Hq, Hkv, D = 1, 23, 4, 2, 16
    q, k, v, do = rnd(16, B, T, Hq, D), rnd(17, B, T, Hkv, D), rnd(18, B, T, Hkv, D), rnd(19, B, T, Hq, D)
    _, _, _, o, lse, dvec = oracle.attn_bwd(q, k, v, do, 10000.0, True, extras=True)
    np.testing.assert_allclose(dvec, np.einsum("bthd,bthd->bht", do, o), atol=1e-12)
    o2, lse2 = oracle.attn_fwd(q, k, v, 10000.0, True)
    np.testing.assert_allclose(o, o2, atol=1e-14)
    np.testing.assert_allclose(lse, lse2, atol=1e-14)


# ---------------------------------------------------------------- rotary embedding


def test_rope_unit_vectors_closed_form():
    """Pins the pairing (2i, 2i+1), the frequency base^(-2i/D) and the sign."""
    base, D, T = 10000.0, 4, 6
    for t in range(T):
        x = np.zeros((1, T, 1, D))
        x[0, t, 0, 0] = 1.0
        y = oracle.rope(x, base)[0, t, 0]
        np.testing.assert_allclose(y, [math.cos(t), math.sin(t), 0, 0], atol=1e-15)
        x = np.zeros((1, T, 1, D))
        x[0, t, 0, 3] = 1.0
        y = oracle.rope(x, base)[0, t, 0]
        w = t * base ** (-0.5)
        np.testing.assert_allclose(y, [0, 0, -math.sin(w), math.cos(w)], atol=1e-15)


def test_rope_norm_and_relative_position():
    base, T, D = 10000.0, 40, 16
    x = rnd(20, 1, T, 3, D)
    y = oracle.rope(x, base)
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-14)
    # same q at positions i and i+s, same k at j and j+s: equal rotated dot products
    qv, kv = rnd(21, D), rnd(22, D)
    X = np.zeros((1, T, 2, D))
    X[0, :, 0] = qv
    X[0, :, 1] = kv
    Y = oracle.rope(X, base)
    for i, j, s in [(5, 2, 7), (30, 30, 9), (3, 11, 20)]:
        a = Y[0, i, 0] @ Y[0, j, 1]
        b = Y[0, i + s, 0] @ Y[0, j + s, 1]
        assert abs(a - b) < 1e-12
    assert np.array_equal(oracle.rope(x, 0.0), x)


# ---------------------------------------------------------------- gradients


@pytest.mark.parametrize("T", [1, 5, 9])
@pytest.mark.parametrize("causal", [True, False])
def test_gradients_match_central_differences(T, causal):
    """Every element of dQ, dK, dV against fp64 central differences of
    L = sum(dO * O), the check the pages describe for their own backward."""
    B, Hq, Hkv, D = 1, 4, 2, 8
    base = 10000.0
    q, k, v, do = rnd(30 + T, B, T, Hq, D), rnd(40 + T, B, T, Hkv, D), rnd(50 + T, B, T, Hkv, D), rnd(60 + T, B, T, Hq, D)
    dq, dk, dv = oracle.attn_bwd(q, k, v, do, base, causal)
    h = 1e-6

    def loss(qq, kk, vv):
        return float((oracle.attn_fwd(qq, kk, vv, base, causal)[0] * do).sum())

    for name, x, g in (("dQ", q, dq), ("dK", k, dk), ("dV", v, dv)):
        fd = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp = x.copy()
            xm = x.copy()
            xp[idx] += h
            xm[idx] -= h
            args_p = [q, k, v]
            args_m = [q, k, v]
            pos = {"dQ": 0, "dK": 1, "dV": 2}[name]
            args_p[pos], args_m[pos] = xp, xm
            fd[idx] = (loss(*args_p) - loss(*args_m)) / (2 * h)
        err = np.abs(fd - g).max() / max(1.0, np.abs(g).max())
        assert err < 1e-6, (name, err)


# ---------------------------------------------------------------- library cross-check


@pytest.mark.parametrize("causal", [True, False])
def test_matches_torch_sdpa_without_rotation(causal):
    """With the rotation off, attention is torch's scaled-dot-product attention
    (fp64, CPU, autograd), used here as an independent library routine."""
    torch = pytest.importorskip("torch")
    B, T, Hq, Hkv, D = 2, 33, 6, 3, 16
    G = Hq // Hkv
    q, k, v, do = rnd(70, B, T, Hq, D), rnd(71, B, T, Hkv, D), rnd(72, B, T, Hkv, D), rnd(73, B, T, Hq, D)
    tq = torch.tensor(q).transpose(1, 2).requires_grad_()
    tk = torch.tensor(k).transpose(1, 2).requires_grad_()
    tv = torch.tensor(v).transpose(1, 2).requires_grad_()
    to = torch.nn.functional.scaled_dot_product_attention(
        tq, tk.repeat_interleave(G, 1), tv.repeat_interleave(G, 1), is_causal=causal)
    to.backward(torch.tensor(do).transpose(1, 2))
    o, _ = oracle.attn_fwd(q, k, v, 0.0, causal)
    dq, dk, dv = oracle.attn_bwd(q, k, v, do, 0.0, causal)
    np.testing.assert_allclose(o, to.detach().transpose(1, 2).numpy(), atol=1e-12)
    np.testing.assert_allclose(dq, tq.grad.transpose(1, 2).numpy(), atol=1e-11)
    np.testing.assert_allclose(dk, tk.grad.transpose(1, 2).numpy(), atol=1e-11)
    np.testing.assert_allclose(dv, tv.grad.transpose(1, 2).numpy(), atol=1e-11)


# ---------------------------------------------------------------- edge cases


def test_empty_inputs():
    for B, T in ((0, 5), (2, 0)):
        q, k = np.zeros((B, T, 4, 8)), np.zeros((B, T, 2, 8))
        o, lse = oracle.attn_fwd(q, k, k, 10000.0, True)
        assert o.shape == q.shape and lse.shape == (B, 4, T)
        dq, dk, dv = oracle.attn_bwd(q, k, k, q, 10000.0, True)
        assert dq.shape == q.shape and dk.shape == k.shape


def test_rejects_bad_head_grouping():
    with pytest.raises(ValueError):
        oracle.attn_fwd(np.zeros((1, 2, 5, 8)), np.zeros((1, 2, 2, 8)), np.zeros((1, 2, 2, 8)))


# ----------------------------------------------------------------- decode over a key/value cache
BASE = 10000.0
def _decode_case(B=3, T=11, Hq=6, Hkv=2, D=8, seed=7):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, T, Hq, D))
    k = rng.standard_normal((B, T, Hkv, D))
    v = rng.standard_normal((B, T, Hkv, D))
    return q, k, v


def test_decode_is_last_row_of_causal_attention():
    """Decoding the token at position L-1 over a cache holding the rotated
    keys 0..L-1 reproduces row L-1 of the full causal attention, per batch
    element with ragged lengths."""
    q, k, v = _decode_case()
    o, lse = oracle.attn_fwd(q, k, v, BASE, True)
    kc = oracle.rope(k, BASE)
    lens = np.array([1, 6, 11])
    qd = np.stack([q[b, lens[b] - 1] for b in range(3)])
    od, ld = oracle.attn_decode(qd, kc, v, lens, BASE)
    for b in range(3):
        np.testing.assert_allclose(od[b], o[b, lens[b] - 1], rtol=0, atol=1e-13)
        np.testing.assert_allclose(ld[b], lse[b, :, lens[b] - 1], rtol=0, atol=1e-13)


def test_decode_single_position_closed_form():
    """len = 1: the only key is the query's own position 0 (no rotation):
    O = v_0 and LSE = q . k_0 / sqrt(D)."""
    q, k, v = _decode_case(B=1, T=4, Hq=2, Hkv=1, D=6)
    od, ld = oracle.attn_decode(q[:, 0], k, v, np.array([1]), BASE)
    for h in range(2):
        np.testing.assert_allclose(od[0, h], v[0, 0, 0], rtol=0, atol=1e-14)
        assert abs(ld[0, h] - float(q[0, 0, h] @ k[0, 0, 0]) / math.sqrt(6)) < 1e-13


def test_decode_equal_scores_give_mean_and_log_length():
    """Zero keys make every score 0: O is the mean of the cached values and
    LSE = ln(len)."""
    q, _, v = _decode_case(B=2, T=9, Hq=3, Hkv=1, D=4)
    kc = np.zeros((2, 9, 1, 4))
    lens = np.array([4, 9])
    od, ld = oracle.attn_decode(q[:, 0], kc, v, lens, BASE)
    for b in range(2):
        np.testing.assert_allclose(od[b], np.broadcast_to(v[b, :lens[b], 0].mean(axis=0), (3, 4)), atol=1e-14)
        np.testing.assert_allclose(ld[b], math.log(lens[b]), atol=1e-14)


def test_decode_gqa_equals_mha_and_empty_cache():
    """Query heads of one group read the same cached head (GQA = MHA with the
    cache repeated per group); an empty cache gives O = 0, LSE = -inf."""
    q, k, v = _decode_case(B=2, T=5, Hq=4, Hkv=2, D=8)
    kc = oracle.rope(k, BASE)
    lens = np.array([5, 0])
    od, ld = oracle.attn_decode(q[:, 4], kc, v, lens, BASE)
    om, lm = oracle.attn_decode(q[:, 4], np.repeat(kc, 2, axis=2), np.repeat(v, 2, axis=2), lens, BASE)
    np.testing.assert_allclose(od, om, atol=1e-14)
    np.testing.assert_allclose(ld[0], lm[0], atol=1e-14)
    assert np.all(od[1] == 0.0) and np.all(np.isneginf(ld[1]))
    with pytest.raises(Exception):
        oracle.attn_decode(q[:, 4], kc, v, np.array([6, 1]), BASE)
