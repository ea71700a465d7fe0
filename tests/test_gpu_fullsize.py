"""Parity at every configuration the benchmark reports: the full-size layers
(the Mixtral-8x7B-, Qwen2-MoE- and DeepSeek-V3-shaped layers of the talk
notes' Table 2) at every decode and prefill T the benchmark times, the
DeepSeek-V3-shaped routing-skew points, and the dense SwiGLU FFN at the
DenseFA and DensePA widths the tax tau is measured against.

Each full-size case runs in the launch configuration the benchmark times
(the same T, hence the same token-tile caps, fused or two-launch expert FFN,
shared-expert SM share) and is checked on 256 seeded tokens spread over all
of T: the layer is token-wise independent given its logits, so the sample is
exact for the tokens it holds.  Index outputs (P, E_active) are checked over
all T.  The weights of one layer shape are made once and shared by its cases
(the launch configuration depends on T and the routing, not on the values)."""
import numpy as np
import pytest
import torch

import moe_inputs as mi
import mixture_experts_layer_61_b200 as moe
import oracle
from helpers import OUT_TOL, host, layer_case, rel_err, sample_tokens

pytestmark = pytest.mark.gpu

N_SAMPLE = 256
_cache = {}


def _weights(name):
    """Device weights of one layer shape and their host copies (one shape held at a time)."""
    if name not in _cache:
        _cache.clear()
        torch.cuda.empty_cache()
        sh = mi.SHAPES[name]
        w = mi.make_weights(sh, mi.seed_for(sh, 0, 7), device="cuda")
        _cache[name] = (w, {n: host(t) for n, t in w.items()})
    return _cache[name]


@pytest.fixture(scope="module", autouse=True)
def _release():
    yield
    _cache.clear()
    torch.cuda.empty_cache()


BENCHMARKED = [(n, T) for n in ("mixtral", "qwen2moe", "deepseekv3")
               for T in mi.SHAPES[n].decode_T + mi.SHAPES[n].prefill_T]


@pytest.mark.parametrize("name,T", BENCHMARKED)
def test_layer_every_benchmarked_config(name, T):
    sh = mi.SHAPES[name]
    w, wh = _weights(name)
    x = mi.make_x(sh, T, mi.seed_for(sh, T), device="cuda")
    assert layer_case(sh, T, w, x, wh, n_sample=N_SAMPLE, sample_seed=T) < OUT_TOL


@pytest.mark.parametrize("T,s", [(32, 0.5), (32, 1.0), (2048, 0.5), (2048, 1.0), (256, 0.0), (256, 1.5)])
def test_layer_deepseek_skew_sweep_points(T, s):
    # the routing-skew sweep: Zipf(s) Gumbel logits in place of the router's
    sh = mi.SHAPES["deepseekv3"]
    w, wh = _weights("deepseekv3")
    x = mi.make_x(sh, T, mi.seed_for(sh, T, 5), device="cuda")
    lg = mi.zipf_gumbel_logits(sh.E, T, s, seed=4000 + T, device="cuda")
    assert layer_case(sh, T, w, x, wh, override=lg, n_sample=N_SAMPLE, sample_seed=T + 1) < OUT_TOL


# ------------------------------------------------------ DenseFA / DensePA
_dense = {}


def _dense_weights(H, I):
    if (H, I) not in _dense:
        _dense.clear()
        _cache.clear()
        torch.cuda.empty_cache()
        w13, w2 = mi.make_dense_weights(H, I, torch.bfloat16, seed=H + I, device="cuda")
        _dense[(H, I)] = (w13, w2, host(w13), host(w2))
    return _dense[(H, I)]


# T = 1 / 32 / 128: the fused FFN at token-tile caps 32 / 64 / 128; T = 2048:
# the CTA-pair GEMMs (the widths and T the benchmark's tau lines time)
DENSE = ([(n, "FA", T) for n in ("mixtral", "qwen2moe", "deepseekv3") for T in (1, 32, 128, 2048)] +
         [(n, "PA", T) for n in ("mixtral", "qwen2moe", "deepseekv3") for T in (32, 2048)])


@pytest.mark.parametrize("name,kind,T", DENSE)
def test_dense_ffn_at_the_timed_widths(name, kind, T):
    sh = mi.SHAPES[name]
    I = sh.I_FA if kind == "FA" else sh.I_PA
    w13, w2, w13h, w2h = _dense_weights(sh.H, I)
    x = mi.make_x(sh, T, mi.seed_for(sh, T, 50), device="cuda")
    ws = moe.alloc_workspace(moe.dense_workspace_size(T, sh.H, I))
    out = moe.dense_ffn(x, w13, w2, ws)
    moe.check_status(ws)
    tok = sample_tokens(T, 8 if kind == "FA" else 4, seed=I + T)
    ref = oracle.dense_ffn(host(x)[tok], w13h, w2h)
    assert rel_err(out.float().cpu().numpy()[tok], ref) < OUT_TOL
    if kind == "PA" and T == 2048 and name == "deepseekv3":
        _dense.clear()
        torch.cuda.empty_cache()
