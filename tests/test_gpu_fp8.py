"""FP8 expert weights on the GPU against the oracle: the row quantiser's
codes and scales bit-exact, and the layer with FP8 routed and shared weights
(the fused decode FFN widening E4M3 codes to f16 in tensor memory, f16 MMAs)
within the output bound of the bf16 layer, against the oracle's layer
computed on the same codes and scales."""
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
                                    ("qwen2moe", 128), ("deepseekv3", 128)])
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
    # widening or the tensor core dropped them
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
