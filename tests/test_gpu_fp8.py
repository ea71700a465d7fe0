"""FP8 expert weights on the GPU against the oracle: the row quantiser's
codes and scales bit-exact, the token rows' exact E4M3 hi/lo split checked
against the format's definition, and the layer with FP8 routed and shared
weights (the fused decode FFN: E4M3 x E4M3 products throughout, the
activations split into E4M3 terms on chip) within the output bound of the
bf16 layer, against the oracle's layer computed on the same codes and
scales."""
import numpy as np
import pytest
import torch

import moe_inputs as mi
import mixture_experts_layer_61_b200 as moe
import oracle
from helpers import OUT_TOL, cfg_for, host, rel_err, sample_tokens, small_shape

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("rows,cols,dtype", [(300, 512, torch.bfloat16), (7, 4096, torch.bfloat16),
                                             (64, 208, torch.float32), (3, 14336, torch.bfloat16)])
def test_quantize_fp8_bit_exact(rows, cols, dtype):
    g = torch.Generator(device="cuda")
    g.manual_seed(rows + cols)
    w = torch.randn((rows, cols), generator=g, device="cuda") * torch.logspace(-4, 3, rows, device="cuda")[:, None]
    w[1] = 0.0                               # an all-zero row
    w[2, :5] = torch.tensor([448.0, -1e-6, 3e-3, 1e9, -0.0])
    w = w.to(dtype)
    q, s = moe.quantize_fp8(w)
    torch.cuda.synchronize()
    qr, sr = oracle.quantize_fp8(host(w))
    assert np.array_equal(s.cpu().numpy(), sr)
    assert np.array_equal(q.cpu().numpy(), qr)


def _fp8_weights(w):
    out = {}
    for name in ("w13", "w2", "w13_sh", "w2_sh"):
        if name in w:
            out[name] = moe.quantize_fp8(w[name])
    return out


def _run_fp8_layer(shape, T, seed, n_sample=None, k=None):
    w = mi.make_weights(shape, seed, device="cuda")
    x = mi.make_x(shape, T, seed, device="cuda")
    cfg = cfg_for(shape, T)
    q = _fp8_weights(w)
    ws = moe.alloc_workspace(moe.workspace_size(cfg))
    kt = None if k is None else torch.from_numpy(np.asarray(k, np.int32)).cuda()
    sh = {}
    if "w13_sh" in q:
        sh = dict(q13_sh=q["w13_sh"][0], s13_sh=q["w13_sh"][1], q2_sh=q["w2_sh"][0], s2_sh=q["w2_sh"][1])
    out = moe.layer_forward_fp8(cfg, x, w["w_r"], q["w13"][0], q["w13"][1], q["w2"][0], q["w2"][1], ws, k=kt, **sh)
    moe.check_status(ws)
    lg = moe.layer_logits(cfg, ws).cpu().numpy()
    tok = sample_tokens(T, n_sample or T, seed)
    c = lambda t: t.cpu().numpy()
    shr = {}
    if sh:
        shr = dict(q13_sh=c(sh["q13_sh"]), s13_sh=c(sh["s13_sh"]), q2_sh=c(sh["q2_sh"]), s2_sh=c(sh["s2_sh"]))
    ref = oracle.moe_layer_fp8(host(x), None, c(q["w13"][0]), c(q["w13"][1]), c(q["w2"][0]), c(q["w2"][1]),
                               shape.K, shape.score_fn, shape.renorm, logits=lg, tokens=tok, k=k, **shr)
    return rel_err(out.float().cpu().numpy()[tok], ref)


@pytest.mark.parametrize("T", [1, 5, 40, 120])
def test_fp8_layer_small(T):
    # T = 1, 5, 40: fused small-batch routing; T = 120: separate routing
    # launches, 30 rows per expert (64-token tiles), the shared FFN on 128
    shape = small_shape(H=512, E=16, K=4, I=384, I_sh=256)
    assert _run_fp8_layer(shape, T, seed=T + 90) < OUT_TOL


def test_fp8_layer_128_token_tiles_without_shared():
    # 400 tokens x 2 / 8 experts = 100 rows per expert: 128-token tiles
    shape = small_shape(H=512, E=8, K=2, I=512)
    assert _run_fp8_layer(shape, 400, seed=4) < OUT_TOL


def test_fp8_layer_ragged_and_dynamic_k():
    shape = small_shape(H=272, E=8, K=2, I=208, I_sh=144)
    k = np.array([0, 1, 2, 2, 1, 0, 2] * 4, np.int32)
    assert _run_fp8_layer(shape, 28, seed=3, k=k) < OUT_TOL


@pytest.mark.parametrize("name,T", [("mixtral", 32), ("qwen2moe", 32), ("deepseekv3", 32), ("mixtral", 256),
                                    ("qwen2moe", 128), ("deepseekv3", 128), ("mixtral", 1)])
def test_fp8_layer_full_size_sampled(name, T):
    # every token up to 256 (the FP8 path runs decode sizes: at most 128 rows
    # per routed expert, and T <= 128 with shared experts)
    shape = mi.SHAPES[name]
    assert _run_fp8_layer(shape, T, seed=mi.seed_for(shape, T, 3), n_sample=256) < OUT_TOL


def test_fp8_layer_rejects_prefill_sizes():
    shape = small_shape(H=256, E=4, K=2, I=256)
    T = 600  # 300 rows per expert: beyond the fused FFN
    w = mi.make_weights(shape, 1, device="cuda", shared=False)
    x = mi.make_x(shape, T, 1, device="cuda")
    cfg = cfg_for(shape, T)
    ws = moe.alloc_workspace(moe.workspace_size(cfg))
    q13, s13 = moe.quantize_fp8(w["w13"])
    q2, s2 = moe.quantize_fp8(w["w2"])
    with pytest.raises(moe.MoeError) as e:
        moe.layer_forward_fp8(cfg, x, w["w_r"], q13, s13, q2, s2, ws)
    assert e.value.code == -1


def test_fp8_subnormal_codes_are_kept():
    # gate/up rows of one large weight (it sets the scale) and many tiny ones
    # that quantise to E4M3 subnormals; the large weights meet x = 0, so the
    # output comes from the subnormal codes alone and would vanish if the
    # tensor core's E4M3 products dropped them
    T, H, I = 16, 256, 128
    rng = np.random.default_rng(77)
    w13 = rng.uniform(-0.03, 0.03, (2 * I, H)).astype(np.float32)
    w13[:, 0] = 1000.0                       # scale 1000/448: the rest are below 2^-6 x scale
    w2 = (rng.standard_normal((H, I)) / np.sqrt(I)).astype(np.float32)
    x = rng.standard_normal((T, H)).astype(np.float32)
    x[:, 0] = 0.0
    dev = lambda a: torch.from_numpy(a).cuda().to(torch.bfloat16)
    w13_d, w2_d, x_d = dev(w13), dev(w2), dev(x)
    q13, s13 = moe.quantize_fp8(w13_d)
    q2, s2 = moe.quantize_fp8(w2_d)
    codes = q13.cpu().numpy()[:, 1:]
    assert np.mean((codes & 0x78) == 0) > 0.95              # exponent field 0: subnormal (or zero)
    ws = moe.alloc_workspace(moe.dense_fp8_workspace_size(T, H, I))
    out = moe.dense_ffn_fp8(x_d, q13, s13, q2, s2, ws)
    moe.check_status(ws)
    c = lambda t: t.cpu().numpy()
    ref = oracle.moe_layer_fp8(host(x_d), None, c(q13)[None], c(s13)[None], c(q2)[None], c(s2)[None], 1,
                               logits=np.zeros((T, 1), np.float32))
    assert np.abs(ref).max() > 0
    assert rel_err(out.float().cpu().numpy(), ref) < OUT_TOL


# ------------------------------------------------ the token rows' E4M3 split
def _e4m3_values():
    """All 256 E4M3 code values from the format's definition (OCP FP8: sign,
    4-bit exponent with bias 7, 3-bit mantissa, subnormals at exponent 0,
    S.1111.111 NaN, no infinities)."""
    v = np.empty(256)
    for c in range(256):
        e, m = (c >> 3) & 15, c & 7
        mag = m * 2.0 ** -9 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7)
        v[c] = np.nan if (e == 15 and m == 7) else (-mag if c & 0x80 else mag)
    return v


def test_permute_e4m3x2_is_an_exact_split():
    # x[sorted_ids[p] / K] = s_p (hi_p + lo_p): s_p the smallest power of two
    # with max|row| <= 448 s_p, hi the nearest E4M3 value of row / s_p, and the
    # remainder exact wherever |row / s_p| >= 1/4 (its quantum is then on the
    # E4M3 grid), else within half the smallest subnormal
    shape = small_shape(H=272, E=8, K=2, I=208)
    T = 40
    cfg = cfg_for(shape, T)
    Pm = moe.padded_rows_max(cfg)
    rng = np.random.default_rng(5)
    x = rng.standard_normal((T, shape.H)) * np.logspace(-30, 30, T)[:, None]
    x[3] = 0.0                                           # an all-zero row
    x[4, :4] = [448.0, -1e-30, 3e-3, -0.0]
    x_d = torch.from_numpy(x).to(torch.bfloat16).cuda()
    P = Pm - 3                                           # rows past P are left alone
    sid = np.full(Pm, -7, np.int32)
    sid[:P] = rng.permutation(np.concatenate([np.arange(T * shape.K), -np.ones(P, int)]))[:P]
    scalars = torch.tensor([P, 0, 0, 0], dtype=torch.int32, device="cuda")
    codes, scales = moe.permute_e4m3x2(cfg, x_d, torch.from_numpy(sid).cuda(), scalars)
    torch.cuda.synchronize()
    codes, scales = codes.cpu().numpy(), scales.cpu().numpy().astype(np.float64)
    val = _e4m3_values()
    finite = val[~np.isnan(val)]
    xb = x_d.float().cpu().numpy().astype(np.float64)
    for p in range(P):
        hi, lo = val[codes[p]], val[codes[Pm + p]]
        if sid[p] < 0:
            assert not codes[p].any() and not codes[Pm + p].any() and scales[p] == 1.0
            continue
        row, s = xb[sid[p] // shape.K], scales[p]
        assert np.frexp(s)[0] == 0.5                     # a power of two
        amax = np.abs(row).max()
        if amax == 0:
            assert s == 1.0 and not np.any(hi) and not np.any(lo)
            continue
        assert amax <= 448 * s and amax > 224 * s
        y = row / s
        assert not np.isnan(hi).any() and not np.isnan(lo).any()
        nearest = np.abs(finite[None, :] - y[:, None]).min(axis=1)
        assert np.array_equal(np.abs(y - hi), nearest)
        err = np.abs(y - (hi + lo))
        assert np.all(err[np.abs(y) >= 0.25] == 0)
        assert np.all(err <= 2.0 ** -10)


# ------------------------------------------- repeated launches, both entry paths
@pytest.mark.parametrize("name,T", [("mixtral", 128), ("mixtral", 32), ("qwen2moe", 64)])
def test_fp8_repeated_forwards_are_identical(name, T):
    # Each block's phase-B (down) items follow its phase-A (gate/up) items, and
    # the warps that split the activation tiles see only the phase-B stages:
    # a stage handshake that depended on timing would show up here as a
    # reported timeout or as outputs that differ between launches.  The layer
    # call and the per-stage calls (moe_permute_e4m3x2, moe_grouped_ffn_fp8 on a
    # GEMM workspace) both run 12 times on the same inputs.
    shape = mi.SHAPES[name]
    w = mi.make_weights(shape, 11, device="cuda", shared=False)
    x = mi.make_x(shape, T, 11, device="cuda")
    cfg = cfg_for(shape, T)
    cfg.n_shared = 0
    q13, s13 = moe.quantize_fp8(w["w13"])
    q2, s2 = moe.quantize_fp8(w["w2"])
    ws = moe.alloc_workspace(moe.workspace_size(cfg))
    ref = moe.layer_forward_fp8(cfg, x, w["w_r"], q13, s13, q2, s2, ws).clone()
    moe.check_status(ws)
    for _ in range(12):
        out = moe.layer_forward_fp8(cfg, x, w["w_r"], q13, s13, q2, s2, ws)
        moe.check_status(ws)
        assert torch.equal(out, ref)

    gws = moe.alloc_workspace(moe.gemm_workspace_size())
    logits = moe.router_gemm(cfg, x, w["w_r"], gws)
    ids, tw = moe.route(cfg, logits)
    al = moe.align_pad(cfg, ids)
    Pm = moe.padded_rows_max(cfg)
    act = torch.empty((Pm, shape.I), dtype=torch.float16, device="cuda")
    y = torch.empty((Pm, shape.H), dtype=torch.bfloat16, device="cuda")
    first = None
    for _ in range(12):
        codes, scales = moe.permute_e4m3x2(cfg, x, al["sorted_ids"], al["scalars"])
        moe.grouped_ffn_fp8(cfg, codes, scales, q13, s13, q2, s2, al["offsets"], gws, act, y)
        out = moe.combine(cfg, y, al["pos"], tw)
        moe.check_status(gws)
        if first is None:
            first = out.clone()
        assert torch.equal(out, first)
    # the two entry paths may cut the tiles into different K-slices (their own
    # SM counts), so they agree within the output bound, not bit for bit
    assert rel_err(first.float().cpu().numpy(), ref.float().cpu().numpy()) < OUT_TOL


def test_fp8_wait_timeout_is_reported_and_recoverable():
    # the FP8 kernel's abort path: a withheld operand load makes one block's
    # bounded wait run out (20 ms); every role (producer, MMA thread, activation
    # splitters, epilogue) winds down, the status reads MOE_ERR_TIMEOUT, the
    # control words (the per-row activation maxima among them) are zero again
    # and the next call reproduces the reference bit for bit
    shape = small_shape(H=512, E=8, K=2, I=512, I_sh=256)
    T = 40
    w = mi.make_weights(shape, 8, device="cuda")
    x = mi.make_x(shape, T, 8, device="cuda")
    cfg = cfg_for(shape, T)
    q = _fp8_weights(w)
    ws = moe.alloc_workspace(moe.workspace_size(cfg))
    sh = dict(q13_sh=q["w13_sh"][0], s13_sh=q["w13_sh"][1], q2_sh=q["w2_sh"][0], s2_sh=q["w2_sh"][1])
    fwd = lambda: moe.layer_forward_fp8(cfg, x, w["w_r"], q["w13"][0], q["w13"][1], q["w2"][0], q["w2"][1], ws, **sh)
    ref = fwd().clone()
    moe.check_status(ws)
    moe.set_wait_limit_ns(20_000_000)
    try:
        moe.debug_withhold_first_load(True)
        fwd()
        with pytest.raises(moe.MoeError) as e:
            moe.check_status(ws)
        assert e.value.code == -4
    finally:
        moe.debug_withhold_first_load(False)
        moe.set_wait_limit_ns(0)
    out = fwd()
    moe.check_status(ws)
    assert torch.equal(out, ref)
