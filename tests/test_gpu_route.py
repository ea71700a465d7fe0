"""Router GEMM and top-K gating on the GPU against the oracle: ids bit-exact on
supplied fp32 logits (ties to the lower index, signed zeros, infinities), gate
weights and router logits within fp32 rounding."""
import numpy as np
import pytest
import torch

import moe_inputs as mi
import mixture_experts_layer_61_b200 as moe
import oracle
from helpers import host, small_shape

pytestmark = pytest.mark.gpu


def _route(T, E, K, logits_np, score_fn=0, renorm=1):
    cfg = moe.config(T, 64, E, K, 64, score_fn=score_fn, renorm=renorm)
    lg = torch.from_numpy(logits_np).cuda()
    ids, w = moe.route(cfg, lg)
    torch.cuda.synchronize()
    return ids.cpu().numpy(), w.cpu().numpy()


@pytest.mark.parametrize("E,K", [(8, 2), (64, 8), (256, 8), (1024, 16), (5, 5), (1, 1), (33, 7)])
@pytest.mark.parametrize("kind", ["gauss", "ties"])
def test_topk_ids_bit_exact(E, K, kind):
    T = 300
    if kind == "gauss":
        lg = np.random.default_rng(E * 31 + K).standard_normal((T, E)).astype(np.float32)
    else:
        lg = mi.tie_heavy_logits(T, E, seed=E + K, levels=2)
    ids, w = _route(T, E, K, lg)
    ref = oracle.topk(lg, K)
    assert np.array_equal(ids, ref)
    for score_fn in (0, 1):
        for renorm in (0, 1):
            ids2, w2 = _route(T, E, K, lg, score_fn, renorm)
            assert np.array_equal(ids2, ref)
            wr = oracle.gate_weights(lg, ref, score_fn, renorm)
            assert np.allclose(w2, wr, rtol=2e-6, atol=1e-7), (score_fn, renorm, np.abs(w2 - wr).max())


def test_topk_special_values():
    E, K, T = 16, 4, 64
    rng = np.random.default_rng(5)
    lg = mi.tie_heavy_logits(T, E, seed=1, levels=1)
    lg[rng.random((T, E)) < 0.2] = np.inf
    lg[rng.random((T, E)) < 0.2] = -np.inf
    lg[0, :] = -np.inf                 # every logit -inf: lowest indices
    lg[1, :] = np.float32(-0.0)
    lg[1, ::3] = np.float32(0.0)       # +0 and -0 tie
    ids, _ = _route(T, E, K, lg)
    assert np.array_equal(ids, oracle.topk(lg, K))
    assert ids[0].tolist() == [0, 1, 2, 3] and ids[1].tolist() == [0, 1, 2, 3]


def test_topk_nan_keeps_ids_in_range():
    E, K, T = 8, 3, 8
    lg = np.full((T, E), np.nan, np.float32)
    lg[1, 2] = 1.0
    ids, _ = _route(T, E, K, lg)
    assert ids.min() >= 0 and ids.max() < E
    for t in range(T):
        assert len(set(ids[t].tolist())) == K
    assert ids[1, 0] == 2


def test_topk_single_token_and_empty():
    lg = np.array([[0.5, 2.0, 2.0, -1.0]], np.float32)
    ids, w = _route(1, 4, 2, lg)
    assert ids.tolist() == [[1, 2]]
    assert np.allclose(w, [[0.5, 0.5]])
    cfg = moe.config(0, 64, 4, 2, 64)
    empty = torch.empty((0, 4), dtype=torch.float32, device="cuda")
    ids, w = moe.route(cfg, empty)
    torch.cuda.synchronize()
    assert ids.shape == (0, 2)


@pytest.mark.parametrize("dtype,H,E,T", [("bf16", 512, 8, 1), ("bf16", 4096, 8, 33), ("bf16", 7168, 256, 70),
                                         ("bf16", 3584, 64, 300), ("fp32", 256, 8, 64), ("bf16", 264, 130, 17)])
def test_router_logits(dtype, H, E, T):
    shape = small_shape(H, E, 2, 64, dtype=dtype)
    w = mi.make_weights(shape, seed=3, device="cuda", experts=False)
    x = mi.make_x(shape, T, seed=4, device="cuda")
    cfg = moe.config(T, H, E, 2, 64, dtype=moe.BF16 if dtype == "bf16" else moe.FP32)
    ws = moe.alloc_workspace(moe.gemm_workspace_size())
    lg = moe.router_gemm(cfg, x, w["w_r"], ws)
    moe.check_status(ws)
    ref = oracle.router_logits(host(x), host(w["w_r"]))
    err = np.abs(lg.cpu().numpy() - ref).max() / np.abs(ref).max()
    # bf16 inputs: exact products, fp32 sums; fp32 inputs run as tf32 products
    assert err < (1e-5 if dtype == "bf16" else 4e-3), err


@pytest.mark.parametrize("E,K", [(8, 2), (64, 8), (256, 8), (1024, 16), (5, 5)])
def test_dynamic_k_topk_bit_exact(E, K):
    # per-token dynamic K: token t takes its k[t] top experts (0..K), empty
    # slots -1 with weight 0, weights renormalised over the selected
    T = 300
    rng = np.random.default_rng(E + K)
    lg = mi.tie_heavy_logits(T, E, seed=E * 3 + K, levels=3)
    k = rng.integers(0, K + 1, size=T).astype(np.int32)
    ref = oracle.topk(lg, K, k)
    kt = torch.from_numpy(k).cuda()
    for score_fn in (0, 1):
        for renorm in (0, 1):
            cfg = moe.config(T, 64, E, K, 64, score_fn=score_fn, renorm=renorm)
            ids, w = moe.route(cfg, torch.from_numpy(lg).cuda(), k=kt)
            torch.cuda.synchronize()
            assert np.array_equal(ids.cpu().numpy(), ref)
            wr = oracle.gate_weights(lg, ref, score_fn, renorm)
            assert np.allclose(w.cpu().numpy(), wr, rtol=2e-6, atol=1e-7)


def test_dynamic_k_is_clamped():
    # counts outside [0, K] act as the nearest bound
    T, E, K = 6, 8, 3
    lg = np.random.default_rng(5).standard_normal((T, E)).astype(np.float32)
    k = np.array([-4, 0, 1, 3, 7, 100], np.int32)
    cfg = moe.config(T, 64, E, K, 64)
    ids, _ = moe.route(cfg, torch.from_numpy(lg).cuda(), k=torch.from_numpy(k).cuda())
    torch.cuda.synchronize()
    assert np.array_equal(ids.cpu().numpy(), oracle.topk(lg, K, np.clip(k, 0, K)))
