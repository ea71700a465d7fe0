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


def layer_case(shape, T, w, x, wh=None, override=None, n_sample=None, sample_seed=0, check_stats=True, pad_mode=0,
               k=None):
    """One moe_layer_forward on the GPU against the oracle's layer.

    w / x: device weights and tokens; wh: host copies of the weights (made here
    when None).  The oracle routes on the logits the layer computed (read back
    from the workspace), or on `override`; the layer's logits are checked
    against the oracle's router on the same sampled tokens, spread over all of
    T.  Returns max|out - ref| / max|ref| over the sampled tokens."""
    import oracle

    cfg = cfg_for(shape, T, pad_mode=pad_mode)
    ws = moe.alloc_workspace(moe.workspace_size(cfg))
    stats = torch.zeros(4, dtype=torch.int32, device="cuda")
    kt = None if k is None else torch.from_numpy(np.asarray(k, np.int32)).cuda()
    out = moe.layer_forward(cfg, x, w["w_r"], w["w13"], w["w2"], ws, w.get("w13_sh"), w.get("w2_sh"),
                            logits_override=override, stats=stats, k=kt)
    moe.check_status(ws)
    if wh is None:
        wh = {n: host(t) for n, t in w.items()}
    tok = sample_tokens(T, n_sample or T, sample_seed)
    xh = host(x)
    layer_lg = moe.layer_logits(cfg, ws).cpu().numpy()
    ref_lg = oracle.router_logits(xh[tok], wh["w_r"])
    # fp32 layers that may be routed by the tensor-core router (above 64 tokens,
    # or a router matrix larger than 2^17 elements with more than 256 logits):
    # tf32 router products
    tc = T > 64 or (shape.E * shape.H > 2 ** 17 and T * shape.E > 256)
    tol = 4e-3 if shape.dtype == "fp32" and tc else 1e-5
    assert np.abs(layer_lg[tok] - ref_lg).max() / np.abs(ref_lg).max() < tol
    lg = layer_lg if override is None else override.cpu().numpy()
    if check_stats:
        ids = oracle.topk(lg, shape.K, k)
        r = oracle.align(ids, shape.E, shape.tile_B, mode=pad_mode)
        st = stats.cpu().numpy()
        assert st[0] == r["P"] and st[1] == r["E_active"] and st[2] == 0
    sh = {}
    if shape.I_sh:
        sh = dict(w13_sh=wh["w13_sh"], w2_sh=wh["w2_sh"])
    ref = oracle.moe_layer(xh, None, wh["w13"], wh["w2"], shape.K, shape.score_fn, shape.renorm, logits=lg,
                           tokens=tok, k=k, **sh)
    return rel_err(out.float().cpu().numpy()[tok], ref)
