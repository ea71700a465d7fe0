"""Alignment with block-wise and max-value padding, permute and combine on the
GPU against the oracle: every index output bit-exact (counts, offsets,
sorted_ids, block_expert, pos, P, E_active), the permute an exact row copy,
the combine within fp32 rounding."""
import numpy as np
import pytest
import torch

import moe_inputs as mi
import mixture_experts_layer_61_b200 as moe
import oracle
from helpers import host

pytestmark = pytest.mark.gpu


def _ids(T, E, K, seed, kind="uniform"):
    if kind == "uniform":
        lg = mi.zipf_gumbel_logits(E, T, 0.0, seed).numpy()
    elif kind == "zipf":
        lg = mi.zipf_gumbel_logits(E, T, 1.5, seed).numpy()
    elif kind == "one":       # every token's first choice is expert 0
        lg = mi.zipf_gumbel_logits(E, T, 0.0, seed).numpy()
        lg[:, 0] = 1e30
    else:
        lg = mi.tie_heavy_logits(T, E, seed, levels=1)
    return oracle.topk(lg, K)


def _check_align(T, E, K, B, ids_np, mode=0):
    cfg = moe.config(T, 64, E, K, 64, tile_B=B, pad_mode=mode)
    ids = torch.from_numpy(ids_np).cuda()
    g = moe.align_pad(cfg, ids)
    torch.cuda.synchronize()
    r = oracle.align(ids_np, E, B, mode=mode)
    assert moe.padded_rows_max(cfg) == oracle.p_max(T, K, E, B, mode)
    for key in ("counts", "offsets", "sorted_ids", "block_expert", "pos"):
        assert np.array_equal(g[key].cpu().numpy(), r[key]), key
    sc = g["scalars"].cpu().numpy()
    assert sc[0] == r["P"] and sc[1] == r["E_active"] and sc[2] == 0
    return g, r


@pytest.mark.parametrize("T,E,K,B", [(1, 8, 2, 16), (64, 8, 2, 16), (128, 64, 8, 16), (1024, 256, 8, 16),
                                     (4096, 256, 8, 16), (2048, 8, 2, 128), (333, 64, 8, 32), (50, 1024, 16, 8),
                                     (7, 5, 5, 1), (129, 8, 2, 256)])
@pytest.mark.parametrize("kind", ["uniform", "zipf", "one", "ties"])
def test_align_bit_exact(T, E, K, B, kind):
    _check_align(T, E, K, B, _ids(T, E, K, seed=T + E + B, kind=kind))


@pytest.mark.parametrize("T,E,K,B", [(1, 8, 2, 16), (64, 8, 2, 16), (128, 64, 8, 16), (32, 256, 8, 16),
                                     (512, 256, 8, 16), (333, 64, 8, 32), (50, 1024, 16, 8), (7, 5, 5, 1),
                                     (129, 8, 2, 256)])
@pytest.mark.parametrize("kind", ["uniform", "zipf", "one", "ties"])
def test_align_max_value_bit_exact(T, E, K, B, kind):
    _check_align(T, E, K, B, _ids(T, E, K, seed=T + E + B + 1, kind=kind), mode=1)


def test_align_max_value_repeated_ids_are_flagged_and_stay_in_bounds():
    # ids repeating within a token (no top-K produces them) would need
    # E * ceil(80 / 16) * 16 = 1280 max-value rows against P_max = 768: the
    # alignment flags bit 2 of scalars[2], aligns nothing and writes nothing at
    # or past P_max (guard words after every buffer stay untouched)
    T, K, E, B = 40, 4, 16, 16
    ids_np = np.zeros((T, K), np.int32)
    ids_np[:, 2], ids_np[:, 3] = 5, 7
    cfg = moe.config(T, 64, E, K, 64, tile_B=B, pad_mode=1)
    Pm = moe.padded_rows_max(cfg)
    assert Pm == 768
    nblk, guard = Pm // B, 4096
    buf = lambda n: torch.full((n + guard,), -7, dtype=torch.int32, device="cuda")
    out = dict(counts=buf(E), offsets=buf(E + 1), sorted_ids=buf(Pm), block_expert=buf(nblk), pos=buf(T * K),
               scalars=torch.zeros(4, dtype=torch.int32, device="cuda"))
    g = moe.align_pad(cfg, torch.from_numpy(ids_np).cuda(), out)
    torch.cuda.synchronize()
    sc = g["scalars"].cpu().numpy()
    assert sc[0] == 0 and sc[1] == 0 and (sc[2] & 2)
    assert np.array_equal(out["counts"][:E].cpu().numpy(), np.bincount(ids_np.ravel(), minlength=E))
    assert np.all(out["offsets"][:E + 1].cpu().numpy() == 0)
    assert np.all(g["pos"].cpu().numpy() == -1)
    assert np.all(g["sorted_ids"].cpu().numpy() == -1)
    assert np.all(g["block_expert"].cpu().numpy() == -1)
    n = {"counts": E, "offsets": E + 1, "sorted_ids": Pm, "block_expert": nblk, "pos": T * K}
    for key, length in n.items():
        assert np.all(out[key][length:].cpu().numpy() == -7), key


@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("T,E,K,B", [(64, 8, 2, 16), (300, 64, 8, 16), (1000, 256, 8, 16), (40, 16, 4, 4)])
def test_align_dynamic_k_empty_slots(mode, T, E, K, B):
    # ids -1 (per-token dynamic K) are empty slots: no row, pos -1, not flagged
    rng = np.random.default_rng(T + E)
    k = rng.integers(0, K + 1, size=T).astype(np.int32)
    ids_np = oracle.topk(mi.zipf_gumbel_logits(E, T, 0.5, T + 1).numpy(), K, k)
    g, r = _check_align(T, E, K, B, ids_np, mode=mode)
    assert np.all(g["pos"].cpu().numpy()[ids_np.ravel() < 0] == -1)


def test_align_empty():
    cfg = moe.config(0, 64, 8, 2, 64)
    ids = torch.empty((0, 2), dtype=torch.int32, device="cuda")
    g = moe.align_pad(cfg, ids)
    torch.cuda.synchronize()
    assert g["counts"].sum().item() == 0 and g["scalars"][0].item() == 0
    assert g["offsets"].cpu().tolist() == [0] * 9


def test_align_flags_bad_ids():
    cfg = moe.config(3, 64, 4, 2, 64, tile_B=4)
    ids = torch.tensor([[0, 1], [2, 9], [-1, 3]], dtype=torch.int32, device="cuda")
    g = moe.align_pad(cfg, ids)
    torch.cuda.synchronize()
    assert g["scalars"][2].item() != 0
    assert g["counts"].cpu().tolist() == [1, 1, 1, 1]


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("T,E,K,B,H", [(64, 8, 2, 16, 256), (300, 64, 8, 16, 520), (1, 8, 2, 16, 4096)])
def test_permute_and_combine(dtype, T, E, K, B, H):
    ids_np = _ids(T, E, K, seed=T * 3 + E)
    g, r = _check_align(T, E, K, B, ids_np)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    cfg = moe.config(T, H, E, K, 64, tile_B=B, dtype=tdt)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(T)
    x = torch.randn((T, H), generator=gen, device="cuda").to(tdt)
    Pm = moe.padded_rows_max(cfg)
    xp = torch.full((Pm, H), 7.0, dtype=tdt, device="cuda")
    moe.permute(cfg, x, g["sorted_ids"], g["scalars"], xp)
    torch.cuda.synchronize()
    P = r["P"]
    ref = oracle.permute(host(x), r["sorted_ids"], K, P)
    assert np.array_equal(xp[:P].float().cpu().numpy().astype(np.float64), ref)
    assert torch.all(xp[P:] == 7.0)          # rows past P untouched
    # combine with random gate weights and a shared term
    y = torch.randn((Pm, H), generator=gen, device="cuda").to(tdt)
    w = torch.rand((T, K), generator=gen, device="cuda")
    sh = torch.randn((T, H), generator=gen, device="cuda").to(tdt)
    for shared in (None, sh):
        out = moe.combine(cfg, y, g["pos"], w, shared)
        torch.cuda.synchronize()
        refc = oracle.combine(host(y), r["pos"], w.cpu().double().numpy(), None if shared is None else host(sh))
        err = np.abs(out.float().cpu().numpy() - refc).max() / np.abs(refc).max()
        assert err < (8e-3 if dtype == "bf16" else 1e-6), err
