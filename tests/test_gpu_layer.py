"""Whole-layer parity: moe_layer_forward on the GPU against the oracle's layer
(router -> top-K -> gate weights -> SwiGLU experts -> weighted sum + shared).
The oracle routes on the logits the layer itself computed (read back from the
workspace), so that a near-tie flipped by fp32 rounding of x.W_r cannot
diverge the two; those logits are checked against the oracle's here.  Small
shapes are checked on every token; the full-size layers of every benchmarked
configuration are in test_gpu_fullsize.py."""
import numpy as np
import pytest
import torch

import moe_inputs as mi
import mixture_experts_layer_61_b200 as moe
from helpers import OUT_TOL, cfg_for, layer_case, small_shape

pytestmark = pytest.mark.gpu


def _run_layer(shape, T, seed, override=None, n_sample=None, check_stats=True, pad_mode=0, k=None):
    w = mi.make_weights(shape, seed, device="cuda")
    x = mi.make_x(shape, T, seed, device="cuda")
    return layer_case(shape, T, w, x, override=override, n_sample=n_sample, sample_seed=seed,
                      check_stats=check_stats, pad_mode=pad_mode, k=k)


def test_layer_tiny_fp32_all_tokens():
    assert _run_layer(mi.SHAPES["tiny"], 64, seed=0) < OUT_TOL


@pytest.mark.parametrize("score_fn,renorm", [(0, 1), (0, 0), (1, 1), (1, 0)])
def test_layer_small_gating_variants(score_fn, renorm):
    shape = small_shape(H=512, E=16, K=4, I=768, I_sh=256, score_fn=score_fn, renorm=renorm)
    assert _run_layer(shape, 96, seed=score_fn * 2 + renorm) < OUT_TOL


@pytest.mark.parametrize("T", [1, 3, 130])
def test_layer_small_shapes_ragged_T(T):
    shape = small_shape(H=256, E=8, K=2, I=512, B=16)
    assert _run_layer(shape, T, seed=T) < OUT_TOL


@pytest.mark.parametrize("B", [1, 8, 128])
def test_layer_padding_tiles(B):
    shape = small_shape(H=256, E=8, K=2, I=512, B=B)
    assert _run_layer(shape, 100, seed=B) < OUT_TOL


def test_layer_skewed_logits_override():
    shape = small_shape(H=1024, E=64, K=8, I=256, I_sh=512, score_fn=1)
    lg = mi.zipf_gumbel_logits(64, 200, 1.5, seed=3, device="cuda")
    assert _run_layer(shape, 200, seed=3, override=lg) < OUT_TOL


@pytest.mark.parametrize("T", [5, 100, 700])
@pytest.mark.parametrize("n_sh", [-1, 16, 0])
def test_layer_shared_experts_beside_routed(T, n_sh):
    # the shared FFN on the library's side stream with a fixed SM share (16),
    # with the cost model's share (0), and serially after the routed experts
    # (-1); T = 5 / 100 run fused FFN kernels, T = 700 the CTA-pair GEMMs
    shape = small_shape(H=512, E=16, K=4, I=384, I_sh=1024)
    moe.set_shared_sms(n_sh)
    try:
        cfg = cfg_for(shape, T)
        if n_sh < 0:
            assert moe.shared_sms(cfg) == 0
        elif n_sh > 0:
            assert moe.shared_sms(cfg) == n_sh
        assert _run_layer(shape, T, seed=T + 7) < OUT_TOL
    finally:
        moe.set_shared_sms(0)


@pytest.mark.parametrize("T", [24, 400])
def test_layer_side_stream_captured_in_cuda_graph(T):
    # the fork/join of the shared experts' stream inside a CUDA graph capture
    # (T = 24: fused shared and routed FFNs; T = 400: the shared GEMM pair
    # beside the routed fused FFN): replays equal an eager call bit for bit
    shape = small_shape(H=512, E=16, K=4, I=384, I_sh=1024)
    w = mi.make_weights(shape, T, device="cuda")
    x = mi.make_x(shape, T, T, device="cuda")
    cfg = cfg_for(shape, T)
    assert moe.shared_sms(cfg) > 0
    ws = moe.alloc_workspace(moe.workspace_size(cfg))
    args = (cfg, x, w["w_r"], w["w13"], w["w2"], ws, w["w13_sh"], w["w2_sh"])
    ref = moe.layer_forward(*args).clone()
    moe.check_status(ws)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        out = moe.layer_forward(*args)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    moe.check_status(ws)
    assert torch.equal(out, ref)
    del g


@pytest.mark.parametrize("T", [1, 20, 64, 200])
def test_layer_max_value_padding(T):
    # every expert padded to the most loaded one's rows: the padding slots are
    # zero rows, so the outputs equal the oracle's (which does not pad); T <= 64
    # runs the fused small-batch routing kernel, larger T the separate launches
    shape = small_shape(H=512, E=16, K=4, I=384, I_sh=256)
    assert _run_layer(shape, T, seed=T + 50, pad_mode=1) < OUT_TOL


def test_layer_max_value_padding_deepseek_decode():
    shape = mi.SHAPES["deepseekv3"]
    assert _run_layer(shape, 32, seed=mi.seed_for(shape, 32), n_sample=64, pad_mode=1) < OUT_TOL


@pytest.mark.parametrize("T,pad_mode", [(7, 0), (48, 0), (300, 0), (48, 1)])
def test_layer_dynamic_k(T, pad_mode):
    # per-token dynamic K (0..K experts per token; 0 = shared experts only)
    shape = small_shape(H=512, E=16, K=4, I=384, I_sh=256)
    k = np.random.default_rng(T).integers(0, shape.K + 1, size=T).astype(np.int32)
    k[0] = 0
    assert _run_layer(shape, T, seed=T + 70, pad_mode=pad_mode, k=k) < OUT_TOL


def test_layer_dynamic_k_qwen_full_size():
    shape = mi.SHAPES["qwen2moe"]
    T = 128
    k = np.random.default_rng(11).integers(1, shape.K + 1, size=T).astype(np.int32)
    assert _run_layer(shape, T, seed=mi.seed_for(shape, T, 9), n_sample=64, k=k) < OUT_TOL
