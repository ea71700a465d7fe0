"""Shared helpers for the GPU parity tests: seeded layer construction on the
device, host copies for the oracle, and the output error metric
max|out - ref| / max|ref| (the bound of the layer's outputs)."""
from __future__ import annotations

import math

import numpy as np
import torch

import moe_inputs as mi
import mixture_experts_layer_61_b200 as moe

OUT_TOL = 2e-2


def rel_err(out, ref):
    out = np.asarray(out, np.float64)
    ref = np.asarray(ref, np.float64)
    den = np.abs(ref).max()
    return float(np.abs(out - ref).max() / (den if den > 0 else 1.0))


def host(t):
    return mi.to_oracle(t)


def small_shape(H, E, K, I, I_sh=0, score_fn=0, renorm=1, dtype="bf16", B=16, name="small"):
    return mi.LayerShape(name, H=H, E=E, K=K, I=I, I_sh=I_sh, score_fn=score_fn, renorm=renorm, dtype=dtype,
                         tile_B=B, router_var=1.0 / H, index=9)


def make_layer(shape, T, seed, device="cuda"):
    w = mi.make_weights(shape, seed, device=device)
    x = mi.make_x(shape, T, seed, device=device)
    return x, w


def cfg_for(shape, T, B=None, pad_mode=0):
    n_sh, I_s = (1, shape.I_sh) if shape.I_sh else (0, 0)
    return moe.config(T, shape.H, shape.E, shape.K, shape.I, n_shared=n_sh, I_shared=I_s,
                      tile_B=B or shape.tile_B, score_fn=shape.score_fn, renorm=shape.renorm,
                      dtype=moe.BF16 if shape.dtype == "bf16" else moe.FP32, pad_mode=pad_mode)


def sample_tokens(T, n, seed):
    if T <= n:
        return np.arange(T, dtype=np.int32)
    rng = np.random.default_rng(seed)
    return np.sort(rng.choice(T, size=n, replace=False)).astype(np.int32)
