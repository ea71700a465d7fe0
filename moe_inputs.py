"""Seeded synthetic inputs for the MoE layer: shapes, weights, activations and
router logits.  This module holds none of the layer's arithmetic; it only
draws random numbers, so both the CUDA path and the CPU oracle can be fed the
same inputs.

Workload shapes follow Table 2 of the "Demystifying the Mixture of Experts
Serving Tax" talk notes (hidden size, expert intermediate size, routed experts,
experts per token, shared experts) plus the tiny fp32 case.  Value recipe:
x ~ N(0, 1); gate/up weights ~ N(0, 1/H); down weights ~ N(0, 1/I); router
weights ~ N(0, 1e-3) (variance) for the bf16 layers, N(0, 1/H) for the tiny
one.  The pages measure on routing datasets and traces that are not available
here; the Zipf/Gumbel logits below stand in for trained-router skew.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch


@dataclass(frozen=True)
class LayerShape:
    name: str
    H: int            # hidden size
    E: int            # routed experts
    K: int            # experts per token
    I: int            # expert intermediate size
    I_sh: int         # total shared-expert width S * I_s (0 = none)
    score_fn: int     # 0 softmax, 1 sigmoid
    renorm: int       # 1: weights normalised over the selected K
    dtype: str        # "bf16" or "fp32"
    tile_B: int       # padding tile
    router_var: float # variance of the router weights
    index: int        # workload index (seed base)
    decode_T: tuple = field(default_factory=tuple)
    prefill_T: tuple = field(default_factory=tuple)

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    @property
    def I_FA(self):
        """DenseFA intermediate: K * I + S * I_s (FLOP-aligned)."""
        return self.K * self.I + self.I_sh

    @property
    def I_PA(self):
        """DensePA intermediate: E * I + S * I_s (parameter-aligned)."""
        return self.E * self.I + self.I_sh


SHAPES = {
    "tiny": LayerShape("tiny", H=256, E=8, K=2, I=512, I_sh=0, score_fn=0, renorm=1, dtype="fp32",
                       tile_B=16, router_var=1.0 / 256, index=0, decode_T=(64,), prefill_T=()),
    "mixtral": LayerShape("mixtral", H=4096, E=8, K=2, I=14336, I_sh=0, score_fn=0, renorm=1,
                          dtype="bf16", tile_B=16, router_var=1e-3, index=1,
                          decode_T=(1, 8, 32, 128), prefill_T=(512, 2048)),
    "qwen2moe": LayerShape("qwen2moe", H=3584, E=64, K=8, I=2560, I_sh=8 * 2560, score_fn=0, renorm=1,
                           dtype="bf16", tile_B=16, router_var=1e-3, index=2,
                           decode_T=(1, 32, 128), prefill_T=(1024, 2048)),
    "deepseekv3": LayerShape("deepseekv3", H=7168, E=256, K=8, I=2048, I_sh=2048, score_fn=1, renorm=1,
                             dtype="bf16", tile_B=16, router_var=1e-3, index=3,
                             decode_T=(32, 128, 256), prefill_T=(1024,)),
}


def seed_for(shape: LayerShape, T: int, extra: int = 0) -> int:
    return shape.index * 1000 + T + extra


def _gen(device, seed):
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def randn(shape, std, dtype, device, gen):
    t = torch.randn(shape, dtype=torch.float32, device=device, generator=gen)
    if std != 1.0:
        t.mul_(std)
    return t.to(dtype)


def make_weights(shape: LayerShape, seed: int, device="cpu", experts=True, shared=True):
    """Routed expert weights w13 [E,2I,H] (gate rows then up rows), w2 [E,H,I],
    router w_r [E,H], and the shared experts as one dense FFN of width I_sh:
    w13_sh [2*I_sh,H], w2_sh [H,I_sh]."""
    dt = shape.torch_dtype
    g = _gen(device, seed)
    H, E, I = shape.H, shape.E, shape.I
    out = {"w_r": randn((E, H), math.sqrt(shape.router_var), dt, device, g)}
    if experts:
        w13 = torch.empty((E, 2 * I, H), dtype=dt, device=device)
        w2 = torch.empty((E, H, I), dtype=dt, device=device)
        for e in range(E):  # per expert keeps the fp32 temporary small
            w13[e] = randn((2 * I, H), 1.0 / math.sqrt(H), dt, device, g)
            w2[e] = randn((H, I), 1.0 / math.sqrt(I), dt, device, g)
        out["w13"], out["w2"] = w13, w2
    if shared and shape.I_sh > 0:
        out["w13_sh"] = randn((2 * shape.I_sh, H), 1.0 / math.sqrt(H), dt, device, g)
        out["w2_sh"] = randn((H, shape.I_sh), 1.0 / math.sqrt(shape.I_sh), dt, device, g)
    return out


def make_dense_weights(H: int, I: int, dtype, seed: int, device="cpu"):
    """A dense SwiGLU FFN of width I (DenseFA / DensePA): w13 [2I,H], w2 [H,I]."""
    g = _gen(device, seed)
    w13 = torch.empty((2 * I, H), dtype=dtype, device=device)
    step = max(1, (1 << 28) // max(H, 1))  # rows per fp32 temporary (~1 GiB)
    for r in range(0, 2 * I, step):
        n = min(step, 2 * I - r)
        w13[r:r + n] = randn((n, H), 1.0 / math.sqrt(H), dtype, device, g)
    w2 = torch.empty((H, I), dtype=dtype, device=device)
    step = max(1, (1 << 28) // max(I, 1))
    for r in range(0, H, step):
        n = min(step, H - r)
        w2[r:r + n] = randn((n, I), 1.0 / math.sqrt(I), dtype, device, g)
    return w13, w2


def make_x(shape: LayerShape, T: int, seed: int, device="cpu"):
    g = _gen(device, seed + 7)
    return randn((T, shape.H), 1.0, shape.torch_dtype, device, g)


def zipf_gumbel_logits(E: int, T: int, s: float, seed: int, device="cpu"):
    """Router logits l[t,e] = ln p_e + G[t,e], G ~ Gumbel(0,1) i.i.d., with
    expert popularity p_{pi(r)} proportional to (r+1)^-s over a seeded random
    expert order pi.  The top-K of such logits is a draw of K distinct experts
    without replacement proportional to p (Gumbel-top-k); s = 0 is uniform."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    perm = torch.randperm(E, generator=g)
    ranks = torch.empty(E, dtype=torch.float64)
    ranks[perm] = torch.arange(E, dtype=torch.float64)
    logp = -s * torch.log(ranks + 1.0)
    logp = logp - torch.logsumexp(logp, 0)
    u = torch.rand((T, E), dtype=torch.float64, generator=g)
    u = u.clamp_(min=1e-300)
    gumbel = -torch.log(-torch.log(u))
    return (logp[None, :] + gumbel).to(torch.float32).to(device)


def tie_heavy_logits(T: int, E: int, seed: int, levels: int = 3):
    """Integer-valued fp32 logits with many exact ties and both signed zeros."""
    rng = np.random.default_rng(seed)
    v = rng.integers(-levels, levels + 1, size=(T, E)).astype(np.float32)
    zero = v == 0
    sign = rng.integers(0, 2, size=(T, E)).astype(bool)
    v[zero & sign] = np.float32(-0.0)
    return v


def to_oracle(t: torch.Tensor) -> np.ndarray:
    """A host numpy view the oracle accepts: bf16 as uint16 bit patterns, fp32 as is."""
    t = t.detach().to("cpu").contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.float32:
        return t.numpy()
    raise TypeError(t.dtype)
