"""Seeded synthetic inputs shaped like the source pages' models.

Holds no attention arithmetic: only the workload table and a seeded Gaussian
generator, shared by the tests and the benchmark.  Shapes follow the GPU and
CPU model configurations of the NanoEuler pages (agentlenshq.com summary,
model-configuration table: 768-dim / 12 query and 4 key-value heads / context
512 for the GPU model, 128-dim / 4 and 2 heads / context 128 for the CPU
model; smartinfralog.com post, config listing and benchmark table: batch 4,
sequence 1024).  No corpus or checkpoint is used anywhere; activations are
i.i.d. Gaussians with the stated spreads.
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    T: int
    Hq: int
    Hkv: int
    D: int
    dtype: str          # "f32" (float32 storage) or "bf16"
    qk_std: float = 1.0
    v_std: float = 1.0
    do_std: float = 1.0
    causal: bool = True
    rope_base: float = 10000.0
    layers: int = 1     # independent attention layers per step
    seed: int = 0
    decode: bool = False  # one query per sequence over a cache of T positions
    block: bool = False   # the decoder-block steps beside the attention (model dim C = Hq D)
    ffn: int = 0          # block workloads: the SwiGLU feed-forward of inner width F = ffn instead

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    def flops(self) -> float:
        """Algorithmic FLOPs of one causal fwd+bwd pass: 7 * B * Hq * T^2 * D per
        layer (forward 2, backward 5; half of the 4/10 of a full square)."""
        f = 7.0 * self.B * self.Hq * self.T * self.T * self.D
        if not self.causal:
            f *= 2.0
        return f * self.layers

    def block_flops(self) -> float:
        """Algorithmic FLOPs of the block steps' forward and backward on M = B T
        tokens, C = Hq D: q/k/v projections 2 M C (Hq + 2 Hkv) D forward and
        twice that backward; output projection 2 M (Hq D) C forward, twice that
        backward (the norms' elementwise work is not counted)."""
        M, C = self.B * self.T, self.Hq * self.D
        if self.ffn:  # gate, up and down products: 6 M C F forward, 12 M C F backward
            return 18.0 * M * C * self.ffn
        return 6.0 * M * C * (self.Hq + 2 * self.Hkv) * self.D + 6.0 * M * self.Hq * self.D * C

    def tokens(self) -> int:
        return self.B * (1 if self.decode else self.T) * self.layers

    def cache_bytes(self) -> int:
        """Bytes of the key and value cache a full-length decode step reads."""
        return 2 * self.B * self.T * self.Hkv * self.D * (4 if self.dtype == "f32" else 2)


WORKLOADS = {
    # small CPU model shape: dim 128, 4/2 heads, context 128
    "tiny": Workload("tiny", 1, 128, 4, 2, 32, "f32", seed=1000),
    # GPU model layer: dim 768 = 12 heads x 64, 4 kv heads, context 512; dO ~ N(0, 1e-2)
    "layer": Workload("layer", 8, 512, 12, 4, 64, "f32", do_std=0.1, seed=2000),
    # longer context, peaked softmax: Q, K ~ N(0, 3^2)
    "long": Workload("long", 4, 1024, 12, 4, 64, "f32", qk_std=3.0, seed=3000),
    # full stack: 16 independent layers of the GPU model shape
    "stack": Workload("stack", 8, 512, 12, 4, 64, "f32", do_std=0.1, layers=16, seed=4000),
    # bf16 sweep at B*T = 16384 tokens
    "sweep512": Workload("sweep512", 32, 512, 12, 4, 64, "bf16", seed=5000),
    "sweep1024": Workload("sweep1024", 16, 1024, 12, 4, 64, "bf16", seed=5001),
    "sweep2048": Workload("sweep2048", 8, 2048, 12, 4, 64, "bf16", seed=5002),
    "sweep4096": Workload("sweep4096", 4, 4096, 12, 4, 64, "bf16", seed=5003),
    # head dimension 128 (bf16 storage): 8 query heads over 2 kv heads, context 4096
    "d128": Workload("d128", 4, 4096, 8, 2, 128, "bf16", seed=5004),
    # generation over a key/value cache: 16 sequences, one new token each
    "decode1024": Workload("decode1024", 16, 1024, 12, 4, 64, "f32", seed=6000, decode=True),
    "decode4096": Workload("decode4096", 16, 4096, 12, 4, 64, "bf16", seed=6001, decode=True),
    # the decoder-block steps of the GPU model layer (dim 768 = 12 x 64)
    "block": Workload("block", 8, 512, 12, 4, 64, "f32", seed=7000, block=True),
    # its SwiGLU feed-forward, inner width F = 4 x 768
    "ffn": Workload("ffn", 8, 512, 12, 4, 64, "f32", seed=7100, block=True, ffn=3072),
}


def make_inputs(w: Workload, layer: int = 0, device="cpu"):
    """Returns ``dict(q, k, v, do)`` for one layer: float32 Gaussians drawn from
    a CPU generator seeded with ``w.seed + layer``, scaled, then cast to the
    workload's dtype (the cast values are the exact inputs both sides see)."""
    g = torch.Generator(device="cpu").manual_seed(int(w.seed) + int(layer))
    shp_q = (w.B, w.T, w.Hq, w.D)
    shp_k = (w.B, w.T, w.Hkv, w.D)
    q = torch.randn(shp_q, generator=g, dtype=torch.float32) * w.qk_std
    k = torch.randn(shp_k, generator=g, dtype=torch.float32) * w.qk_std
    v = torch.randn(shp_k, generator=g, dtype=torch.float32) * w.v_std
    do = torch.randn(shp_q, generator=g, dtype=torch.float32) * w.do_std
    out = {"q": q, "k": k, "v": v, "do": do}
    return {n: t.to(w.torch_dtype).to(device).contiguous() for n, t in out.items()}


def make_decode_inputs(w: Workload, device="cpu"):
    """Returns ``dict(q, kc, vc, lens)`` for a decode workload: the new tokens'
    queries ``[B, Hq, D]``, a full cache ``[B, T, Hkv, D]`` of keys (standing
    for keys already rotated at their positions) and values, and the lengths
    (all ``T``), drawn like ``make_inputs``."""
    g = torch.Generator(device="cpu").manual_seed(int(w.seed))
    q = torch.randn((w.B, w.Hq, w.D), generator=g, dtype=torch.float32) * w.qk_std
    kc = torch.randn((w.B, w.T, w.Hkv, w.D), generator=g, dtype=torch.float32) * w.qk_std
    vc = torch.randn((w.B, w.T, w.Hkv, w.D), generator=g, dtype=torch.float32) * w.v_std
    out = {n: t.to(w.torch_dtype).to(device).contiguous() for n, t in {"q": q, "kc": kc, "vc": vc}.items()}
    out["lens"] = torch.full((w.B,), w.T, dtype=torch.int32, device=device)
    return out


def make_block_inputs(w: Workload, device="cpu"):
    """Inputs of the block steps for C = Hq D: x [B, T, C], gain g [C] ~ 1 +
    N(0, 0.01), weights ~ N(0, 1/fan_in) (Wq [C, Hq D], Wk, Wv [C, Hkv D],
    Wo [Hq D, C]), the attention output o and the upstream gradients dh, dq,
    dk, dv ~ N(0, 1); drawn like ``make_inputs``.  Feed-forward workloads:
    x, g, Wg, Wu [C, F], Wd [F, C] and dh, drawn the same way."""
    g = torch.Generator(device="cpu").manual_seed(int(w.seed))
    C = w.Hq * w.D
    r = lambda *shape, std=1.0: torch.randn(shape, generator=g, dtype=torch.float32) * std
    if w.ffn:
        F = w.ffn
        out = dict(x=r(w.B, w.T, C), g=1.0 + r(C, std=0.1), Wg=r(C, F, std=C ** -0.5), Wu=r(C, F, std=C ** -0.5),
                   Wd=r(F, C, std=F ** -0.5), dh=r(w.B, w.T, C))
        return {n: t.to(w.torch_dtype).to(device).contiguous() for n, t in out.items()}
    out = dict(x=r(w.B, w.T, C), g=1.0 + r(C, std=0.1), Wq=r(C, w.Hq * w.D, std=C ** -0.5),
               Wk=r(C, w.Hkv * w.D, std=C ** -0.5), Wv=r(C, w.Hkv * w.D, std=C ** -0.5),
               Wo=r(w.Hq * w.D, C, std=(w.Hq * w.D) ** -0.5), o=r(w.B, w.T, w.Hq, w.D), dh=r(w.B, w.T, C),
               dq=r(w.B, w.T, w.Hq, w.D), dk=r(w.B, w.T, w.Hkv, w.D), dv=r(w.B, w.T, w.Hkv, w.D))
    return {n: t.to(w.torch_dtype).to(device).contiguous() for n, t in out.items()}


def custom(name="custom", **kw) -> Workload:
    """A workload with explicit fields (edge-case tests)."""
    base = Workload(name, 1, 1, 1, 1, 64, "f32")
    return replace(base, **kw)
