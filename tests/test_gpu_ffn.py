"""The tcgen05 grouped GEMM path (gate/up + SwiGLU, down) and the dense FFN on
the GPU against the oracle, across token-tile caps (32..256 tokens), data-
parallel and stream-K schedules, ragged feature blocks and skewed groups.
Bound: max|out - ref| / max|ref| <= 2e-2."""
import numpy as np
import pytest
import torch

import moe_inputs as mi
import mixture_experts_layer_61_b200 as moe
import oracle
from helpers import OUT_TOL, cfg_for, host, rel_err, sample_tokens, small_shape

pytestmark = pytest.mark.gpu


def _grouped(shape, T, seed, kind="uniform", n_check=96):
    w = mi.make_weights(shape, seed, device="cuda", shared=False)
    x = mi.make_x(shape, T, seed, device="cuda")
    if kind == "uniform":
        lg = mi.zipf_gumbel_logits(shape.E, T, 0.0, seed).numpy()
    else:
        lg = mi.zipf_gumbel_logits(shape.E, T, 1.5, seed).numpy()
        lg[: T // 2, 0] = 1e30
    cfg = cfg_for(shape, T)
    ids = oracle.topk(lg, shape.K)
    g = moe.align_pad(cfg, torch.from_numpy(ids).cuda())
    xp = moe.permute(cfg, x, g["sorted_ids"], g["scalars"])
    ws = moe.alloc_workspace(moe.gemm_workspace_size())
    y, act = moe.grouped_ffn(cfg, xp, w["w13"], w["w2"], g["offsets"], ws)
    moe.check_status(ws)
    # oracle: each checked row through its expert (rows of one token are independent)
    r = oracle.align(ids, shape.E, shape.tile_B)
    sid = r["sorted_ids"]
    rows = np.nonzero(sid >= 0)[0]
    rng = np.random.default_rng(seed)
    rows = np.sort(rng.choice(rows, size=min(n_check, len(rows)), replace=False))
    xh = host(x)
    w13h, w2h = host(w["w13"]), host(w["w2"])
    yh = y.float().cpu().numpy()
    ref = np.stack([oracle.swiglu_ffn(xh[sid[p] // shape.K], w13h[ids.ravel()[sid[p]]], w2h[ids.ravel()[sid[p]]])
                    for p in rows])
    return rel_err(yh[rows], ref)


@pytest.mark.parametrize("T", [1, 5, 64, 200, 400, 1200])
def test_grouped_bf16_tile_caps(T):
    # rows per expert T*K/E picks the token-tile cap: <=24 -> 32, <=56 -> 64, <=112 -> 128, else 256
    shape = small_shape(H=512, E=8, K=2, I=1024)
    assert _grouped(shape, T, seed=T) < OUT_TOL


def test_grouped_fp32_tiny_config():
    shape = mi.SHAPES["tiny"]
    assert _grouped(shape, 64, seed=0, n_check=128) < OUT_TOL


@pytest.mark.parametrize("kind", ["uniform", "skew"])
def test_grouped_many_experts(kind):
    shape = small_shape(H=1024, E=64, K=8, I=512)
    assert _grouped(shape, 150, seed=11, kind=kind) < OUT_TOL


def test_grouped_ragged_features():
    # I and H not multiples of the 128-row weight block, H not of the 64-element K step
    shape = small_shape(H=264, E=6, K=2, I=200)
    assert _grouped(shape, 77, seed=5) < OUT_TOL


def test_grouped_one_hot_expert_many_chunks():
    # half the tokens on expert 0: several token chunks share one weight block
    shape = small_shape(H=256, E=4, K=1, I=384)
    assert _grouped(shape, 1000, seed=2, kind="skew") < OUT_TOL


@pytest.mark.parametrize("T,H,I", [(1, 512, 1024), (16, 256, 640), (300, 1024, 2048), (700, 512, 14336),
                                   (300, 264, 640), (130, 392, 376)])
def test_dense_ffn(T, H, I):
    # (700, 512, 14336): 3 chunks x 112 feature blocks -> data-parallel waves plus a stream-K tail
    w13, w2 = mi.make_dense_weights(H, I, torch.bfloat16, seed=T + I, device="cuda")
    gen = torch.Generator(device="cuda")
    gen.manual_seed(T)
    x = torch.randn((T, H), generator=gen, device="cuda").to(torch.bfloat16)
    ws = moe.alloc_workspace(moe.dense_workspace_size(T, H, I))
    out = moe.dense_ffn(x, w13, w2, ws)
    moe.check_status(ws)
    tok = sample_tokens(T, 48, seed=T)
    ref = oracle.dense_ffn(host(x)[tok], host(w13), host(w2))
    assert rel_err(out.float().cpu().numpy()[tok], ref) < OUT_TOL


@pytest.mark.parametrize("cap", [32, 64, 128, 256])
def test_grouped_every_token_tile_cap(cap):
    # the same grouped problem through every kernel variant: plain or 256-feature
    # (wide) down tiles, SwiGLU gate/up, token tiles of 32..256
    shape = small_shape(H=520, E=6, K=2, I=392)
    moe.set_token_tile_cap(cap)
    try:
        assert _grouped(shape, 700, seed=cap) < OUT_TOL
    finally:
        moe.set_token_tile_cap(0)


def test_dense_ffn_fp32_tf32():
    T, H, I = 40, 256, 512
    w13, w2 = mi.make_dense_weights(H, I, torch.float32, seed=1, device="cuda")
    x = torch.randn((T, H), device="cuda")
    ws = moe.alloc_workspace(moe.dense_workspace_size(T, H, I, moe.FP32))
    out = moe.dense_ffn(x, w13, w2, ws)
    moe.check_status(ws)
    ref = oracle.dense_ffn(host(x), host(w13), host(w2))
    assert rel_err(out.cpu().numpy(), ref) < OUT_TOL


def test_deterministic_repeat():
    # the stream-K fixup sums partial tiles in a fixed order: bitwise-equal reruns
    shape = small_shape(H=1024, E=8, K=2, I=2048)
    w = mi.make_weights(shape, 4, device="cuda", shared=False)
    x = mi.make_x(shape, 3, 4, device="cuda")
    cfg = cfg_for(shape, 3)
    ws = moe.alloc_workspace(moe.workspace_size(cfg))
    o1 = moe.layer_forward(cfg, x, w["w_r"], w["w13"], w["w2"], ws).clone()
    o2 = moe.layer_forward(cfg, x, w["w_r"], w["w13"], w["w2"], ws).clone()
    moe.check_status(ws)
    assert torch.equal(o1, o2)


@pytest.mark.parametrize("pairs", [True, False])
@pytest.mark.parametrize("T,H,I", [(700, 512, 1024), (300, 1024, 2048), (260, 520, 392)])
def test_dense_ffn_cta_pairs(pairs, T, H, I):
    # 2-SM (CTA pair) tiles at the 256-token cap against the oracle, and
    # against single-SM tiles on the same inputs
    w13, w2 = mi.make_dense_weights(H, I, torch.bfloat16, seed=T, device="cuda")
    gen = torch.Generator(device="cuda")
    gen.manual_seed(H)
    x = torch.randn((T, H), generator=gen, device="cuda").to(torch.bfloat16)
    ws = moe.alloc_workspace(moe.dense_workspace_size(T, H, I))
    moe.set_cta_pairs(pairs)
    try:
        out = moe.dense_ffn(x, w13, w2, ws)
        moe.check_status(ws)
    finally:
        moe.set_cta_pairs(True)
    tok = sample_tokens(T, 40, seed=1)
    ref = oracle.dense_ffn(host(x)[tok], host(w13), host(w2))
    assert rel_err(out.float().cpu().numpy()[tok], ref) < OUT_TOL


@pytest.mark.parametrize("kind", ["uniform", "skew"])
def test_grouped_cta_pairs_match_single(kind):
    shape = small_shape(H=1024, E=4, K=2, I=1536)
    e_pair = _grouped(shape, 900, seed=3, kind=kind)
    moe.set_cta_pairs(False)
    try:
        e_single = _grouped(shape, 900, seed=3, kind=kind)
    finally:
        moe.set_cta_pairs(True)
    assert e_pair < OUT_TOL and e_single < OUT_TOL


@pytest.mark.parametrize("shape_kw,T", [(dict(H=512, E=8, K=2, I=1024), 1), (dict(H=1024, E=64, K=8, I=512), 40),
                                        (dict(H=264, E=6, K=2, I=200), 77), (dict(H=2048, E=16, K=4, I=768), 200)])
def test_fused_decode_ffn_matches_two_launch_path(shape_kw, T):
    # the fused decode kernel (one launch, dynamic work, K-sliced tiles) against
    # the separate gate/up and down GEMM launches on the same permuted rows
    shape = small_shape(**shape_kw)
    cfg = cfg_for(shape, T)
    assert moe.ffn_fused(cfg)
    w = mi.make_weights(shape, T, device="cuda", shared=False)
    x = mi.make_x(shape, T, T, device="cuda")
    ids = oracle.topk(mi.zipf_gumbel_logits(shape.E, T, 0.5, T).numpy(), shape.K)
    g = moe.align_pad(cfg, torch.from_numpy(ids).cuda())
    xp = moe.permute(cfg, x, g["sorted_ids"], g["scalars"])
    ws = moe.alloc_workspace(moe.gemm_workspace_size())
    y1, _ = moe.grouped_ffn(cfg, xp, w["w13"], w["w2"], g["offsets"], ws)
    act = torch.empty_like(_)
    y2 = torch.empty_like(y1)
    moe.grouped_gate_up(cfg, xp, w["w13"], g["offsets"], ws, act)
    moe.grouped_down(cfg, act, w["w2"], g["offsets"], ws, y2)
    moe.check_status(ws)
    P = int(g["scalars"][0].item())
    valid = (g["sorted_ids"][:P] >= 0).cpu().numpy()
    a = y1[:P].float().cpu().numpy()[valid]
    b = y2[:P].float().cpu().numpy()[valid]
    assert rel_err(a, b) < 1e-2


def test_dense_ffn_wide_pair_tiles():
    # 64 token chunks x 4 blocks of 512 output features: enough tiles for the
    # 512-feature (wide) CTA-pair down GEMM; fewer tiles take 256-feature pairs
    T, H, I = 16384, 2048, 1024
    w13, w2 = mi.make_dense_weights(H, I, torch.bfloat16, seed=7, device="cuda")
    gen = torch.Generator(device="cuda")
    gen.manual_seed(7)
    x = torch.randn((T, H), generator=gen, device="cuda").to(torch.bfloat16)
    ws = moe.alloc_workspace(moe.dense_workspace_size(T, H, I))
    out = moe.dense_ffn(x, w13, w2, ws)
    moe.check_status(ws)
    tok = sample_tokens(T, 24, seed=7)
    ref = oracle.dense_ffn(host(x)[tok], host(w13), host(w2))
    assert rel_err(out.float().cpu().numpy()[tok], ref) < OUT_TOL


@pytest.fixture
def split_tail_mode(request):
    moe.set_split_tail(request.param)
    yield request.param
    moe.set_split_tail(1)


# the tiles after the whole waves: contiguous stream-K (0) or aligned k-slices
# taken slice-major (1).  (1200 tokens, 8 experts): 64 gate/up pair tiles, all
# of them a tail of 2 slices, and 16 down tiles of 4 slices; (2048, I = 8192):
# 3 whole waves of 74 pairs and a 34-tile tail; (300, ragged 264 / 640): the
# single-CTA 128-token tiles.
@pytest.mark.parametrize("split_tail_mode", [0, 1], indirect=True)
@pytest.mark.parametrize("T", [1200, 400])
def test_grouped_split_tail_modes(split_tail_mode, T):
    shape = small_shape(H=512, E=8, K=2, I=1024)
    assert _grouped(shape, T, seed=T + 3, n_check=128) < OUT_TOL


@pytest.mark.parametrize("split_tail_mode", [0, 1], indirect=True)
@pytest.mark.parametrize("T,H,I", [(2048, 1024, 8192), (700, 512, 14336), (300, 264, 640)])
def test_dense_ffn_split_tail_modes(split_tail_mode, T, H, I):
    w13, w2 = mi.make_dense_weights(H, I, torch.bfloat16, seed=T + I + 1, device="cuda")
    x = mi.make_x(small_shape(H, 1, 1, I), T, T, device="cuda")
    ws = moe.alloc_workspace(moe.dense_workspace_size(T, H, I))
    out = moe.dense_ffn(x, w13, w2, ws)
    moe.check_status(ws)
    tok = sample_tokens(T, 64, seed=T)
    ref = oracle.dense_ffn(host(x)[tok], host(w13), host(w2))
    assert rel_err(out.float().cpu().numpy()[tok], ref) < OUT_TOL


def test_routed_path_policy_for_large_experts():
    # bf16 layers of large experts whose largest expert is expected past the
    # fused FFN's 128-row chunk take the CTA-pair GEMMs; smaller experts and
    # fewer rows keep the fused kernel; FP8 weights always run fused
    m = mi.SHAPES["mixtral"]
    assert not moe.ffn_fused(cfg_for(m, 512))   # 128 rows per expert on average, ~154 at the largest
    assert moe.ffn_fused(cfg_for(m, 384))       # 96 on average
    assert moe.ffn_fused(cfg_for(mi.SHAPES["qwen2moe"], 1024))  # small experts at 128 rows
    moe.set_token_tile_cap(128)                 # a forced cap is kept
    try:
        assert moe.ffn_fused(cfg_for(m, 512))
    finally:
        moe.set_token_tile_cap(0)
    T = 512
    w = mi.make_weights(m, 5, device="cuda", shared=False)
    x = mi.make_x(m, T, 5, device="cuda")
    cfg = cfg_for(m, T)
    q13, s13 = moe.quantize_fp8(w["w13"])
    q2, s2 = moe.quantize_fp8(w["w2"])
    ws = moe.alloc_workspace(moe.workspace_size(cfg))
    moe.layer_forward_fp8(cfg, x, w["w_r"], q13, s13, q2, s2, ws)
    moe.check_status(ws)
