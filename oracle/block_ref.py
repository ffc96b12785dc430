"""fp64 CPU oracle for the steps on either side of the attention: the RMSNorm
pre-norm feeding the Q/K/V projections, and the output projection with the
residual add, forward and backward; and the block's other half, the
pre-norm SwiGLU feed-forward with its residual add.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, never by the product
package.  Plain numpy in float64; a matrix product is the only library step.

What the pages fix ("NanoEuler" write-up, aimsg.uk, section 1 "Architecture
design" and section 2 "Model components"): a pre-norm decoder block whose
residual update is x <- x + f(x); RMSNorm as the pre-norm, with no bias; no
bias anywhere in the model; grouped-query attention with RoPE on the queries
and keys.  The smartinfralog.com post ("Hand-written backward", its RMSNorm
backward listing) gives the RMSNorm input gradient this module derives by the
chain rule: dx_i = g_i dy_i / rms - x_i / (C rms^3) * sum_j dy_j g_j x_j.

Readings where the pages are silent:
  * rms = sqrt(mean_j x_j^2 + eps) over the hidden dimension C of each token,
    eps = 1e-5;
  * projections act on the right: q = y @ Wq with Wq of shape [C, Hq*D], and
    the Hq*D outputs of a token are Hq heads of D consecutive values (the
    attention layout [B, T, Hq, D]); likewise K, V with Hkv heads;
  * the block output is h = x + o @ Wo with o in [B, T, Hq*D], Wo [Hq*D, C].
  * SwiGLU feed-forward (the pages: down(silu(gate(x)) * up(x)), silu(z) =
    z * sigmoid(z), inside a residual branch with its own pre-norm):
    h = x + (silu(y @ Wg) * (y @ Wu)) @ Wd with y = RMSNorm(x) * g, Wg and Wu
    of shape [C, F], Wd [F, C]; the pages give no width F: F = 4 C (the
    GPT-2-small MLP width of the configuration they name).

Arrays: x, h, dh [B, T, C]; g [C]; Wq [C, Hq*D]; Wk, Wv [C, Hkv*D];
Wo [Hq*D, C]; q, o [B, T, Hq, D]; k, v [B, T, Hkv, D].
"""
from __future__ import annotations

import numpy as np

EPS = 1e-5


# ----------------------------------------------------------------- RMSNorm
def rmsnorm_fwd(x, g, eps=EPS):
    """y = x / rms(x) * g per token; returns (y, rstd) with rstd = 1 / rms."""
    x = np.asarray(x, np.float64)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    rstd = 1.0 / np.sqrt(ms + eps)
    return x * rstd * np.asarray(g, np.float64), rstd


def rmsnorm_bwd(x, g, rstd, dy):
    """Gradients of y = x * rstd * g, rstd = (mean x^2 + eps)^-1/2:
    dx = rstd (g dy) - x rstd^3 / C * sum_j (g dy)_j x_j;  dg = sum over tokens of dy x rstd."""
    x = np.asarray(x, np.float64)
    dy = np.asarray(dy, np.float64)
    g = np.asarray(g, np.float64)
    C = x.shape[-1]
    gdy = g * dy
    dot = np.sum(gdy * x, axis=-1, keepdims=True)
    dx = rstd * gdy - x * rstd ** 3 * dot / C
    dg = np.sum((dy * x * rstd).reshape(-1, C), axis=0)
    return dx, dg


# ----------------------------------------------------------------- projections
def qkv_fwd(x, g, Wq, Wk, Wv, Hq, Hkv, D, eps=EPS):
    """Pre-norm then the three projections.  Returns (q, k, v, y, rstd) with
    q [B, T, Hq, D], k and v [B, T, Hkv, D] (un-rotated: the attention
    applies RoPE), y the normalised input and rstd its per-token scale."""
    B, T, C = x.shape
    y, rstd = rmsnorm_fwd(x, g, eps)
    q = (y @ Wq).reshape(B, T, Hq, D)
    k = (y @ Wk).reshape(B, T, Hkv, D)
    v = (y @ Wv).reshape(B, T, Hkv, D)
    return q, k, v, y, rstd


def qkv_bwd(x, g, Wq, Wk, Wv, y, rstd, dq, dk, dv):
    """Backward of qkv_fwd: returns (dx, dg, dWq, dWk, dWv)."""
    B, T, C = x.shape
    dq2 = np.asarray(dq, np.float64).reshape(B * T, -1)
    dk2 = np.asarray(dk, np.float64).reshape(B * T, -1)
    dv2 = np.asarray(dv, np.float64).reshape(B * T, -1)
    y2 = y.reshape(B * T, C)
    dWq, dWk, dWv = y2.T @ dq2, y2.T @ dk2, y2.T @ dv2
    dy = (dq2 @ Wq.T + dk2 @ Wk.T + dv2 @ Wv.T).reshape(B, T, C)
    dx, dg = rmsnorm_bwd(x, g, rstd, dy)
    return dx, dg, dWq, dWk, dWv


def out_fwd(x, o, Wo):
    """Block output h = x + o @ Wo (the residual add of the attention)."""
    B, T, C = x.shape
    return np.asarray(x, np.float64) + (np.asarray(o, np.float64).reshape(B, T, -1) @ Wo)


def out_bwd(o, Wo, dh):
    """Backward of out_fwd: returns (dx_residual, do, dWo); do in o's shape."""
    o = np.asarray(o, np.float64)
    B, T = o.shape[0], o.shape[1]
    dh2 = np.asarray(dh, np.float64).reshape(B * T, -1)
    o2 = o.reshape(B * T, -1)
    return np.asarray(dh, np.float64).copy(), (dh2 @ Wo.T).reshape(o.shape), o2.T @ dh2


# ----------------------------------------------------------------- SwiGLU feed-forward
def silu(z):
    z = np.asarray(z, np.float64)
    return z / (1.0 + np.exp(-z))


def ffn_fwd(x, g, Wg, Wu, Wd, eps=EPS):
    """h = x + (silu(y Wg) * (y Wu)) Wd, y = RMSNorm(x) g.  Returns h and the
    saved (y, rstd, a, b) with a = y Wg, b = y Wu."""
    B, T, C = x.shape
    y, rstd = rmsnorm_fwd(x, g, eps)
    y2 = y.reshape(B * T, C)
    a, b = y2 @ Wg, y2 @ Wu
    h = np.asarray(x, np.float64) + ((silu(a) * b) @ Wd).reshape(B, T, C)
    return h, dict(y=y, rstd=rstd, a=a, b=b)


def ffn_bwd(x, g, Wg, Wu, Wd, saved, dh):
    """Backward of ffn_fwd for the upstream gradient dh: returns (dx, dg, dWg,
    dWu, dWd); dx includes the residual branch's dh.  With s = sigmoid(a):
    d silu(a)/da = s (1 + a (1 - s))."""
    B, T, C = x.shape
    y2 = saved["y"].reshape(B * T, C)
    a, b = saved["a"], saved["b"]
    dh2 = np.asarray(dh, np.float64).reshape(B * T, C)
    act = silu(a) * b
    dWd = act.T @ dh2
    dact = dh2 @ Wd.T
    s = 1.0 / (1.0 + np.exp(-a))
    da = dact * b * s * (1.0 + a * (1.0 - s))
    db = dact * silu(a)
    dWg, dWu = y2.T @ da, y2.T @ db
    dy = (da @ Wg.T + db @ Wu.T).reshape(B, T, C)
    dx, dg = rmsnorm_bwd(x, g, saved["rstd"], dy)
    return dx + np.asarray(dh, np.float64), dg, dWg, dWu, dWd


# ----------------------------------------------------------------- whole block
def block_fwd(x, g, Wq, Wk, Wv, Wo, Hq, Hkv, D, rope_base, causal=True, eps=EPS):
    """h = x + Attn(RMSNorm(x) Wq, RMSNorm(x) Wk, RMSNorm(x) Wv) Wo, with the
    attention of ``oracle.attn_fwd`` (RoPE on q and k inside).  Returns h and
    the saved tensors for block_bwd."""
    import oracle

    q, k, v, y, rstd = qkv_fwd(x, g, Wq, Wk, Wv, Hq, Hkv, D, eps)
    o, lse = oracle.attn_fwd(q, k, v, rope_base, causal)
    h = out_fwd(x, o, Wo)
    return h, dict(q=q, k=k, v=v, y=y, rstd=rstd, o=o, lse=lse)


def block_bwd(x, g, Wq, Wk, Wv, Wo, saved, dh, rope_base, causal=True):
    """Backward of block_fwd: returns (dx, dg, dWq, dWk, dWv, dWo)."""
    import oracle

    dx_res, do, dWo = out_bwd(saved["o"], Wo, dh)
    dq, dk, dv = oracle.attn_bwd(saved["q"], saved["k"], saved["v"], do, rope_base, causal)
    dx, dg, dWq, dWk, dWv = qkv_bwd(x, g, Wq, Wk, Wv, saved["y"], saved["rstd"], dq, dk, dv)
    return dx + dx_res, dg, dWq, dWk, dWv, dWo
