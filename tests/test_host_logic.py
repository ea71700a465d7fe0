"""Host-only logic of the library, called through the C-ABI on the CPU (no
device call is made): configuration validation, the padded-row bound that
sizes every permuted buffer, and the status strings."""
import itertools

import numpy as np
import pytest

import mixture_experts_layer_61_b200 as moe
import oracle


@pytest.mark.parametrize("mode", [moe.BLOCKWISE, moe.MAXVALUE])
def test_padded_rows_bound_matches_the_oracle_and_holds(mode):
    rng = np.random.default_rng(mode)
    for T, K, E, B in itertools.product([0, 1, 3, 64, 1000], [1, 2, 8], [8, 64, 256], [1, 16, 128]):
        if K > E:
            continue
        cfg = moe.config(T, 4096, E, K, 1024, tile_B=B, pad_mode=mode)
        bound = moe.padded_rows_max(cfg)
        assert bound == oracle.p_max(T, K, E, B, mode)
        if 0 < T <= 64:
            # any routing's padded rows fit the bound (the library sizes x_perm / act with it)
            ids = np.stack([rng.choice(E, K, replace=False) for _ in range(T)]).astype(np.int32)
            assert oracle.align(ids, E, B, mode=mode)["P"] <= bound


@pytest.mark.parametrize("bad", [
    dict(K=9, E=8), dict(K=17, E=64), dict(E=1025), dict(tile_B=0), dict(tile_B=257), dict(pad_mode=2),
    dict(H=4100), dict(I=1020), dict(dtype=2), dict(score_fn=2), dict(renorm=2), dict(T=-1),
    dict(n_shared=1, I_shared=0), dict(n_shared=1, I_shared=100),
])
def test_invalid_configurations_are_rejected(bad):
    kw = dict(T=32, H=4096, E=8, K=2, I=1024, n_shared=0, I_shared=0, tile_B=16, score_fn=0, renorm=1,
              dtype=moe.BF16, pad_mode=0)
    kw.update(bad)
    cfg = moe.MoeConfig(*(kw[n] for n, _ in moe.MoeConfig._fields_))
    assert moe.padded_rows_max(cfg) == -1


def test_valid_edge_configurations_are_accepted():
    # fp32 rows need 4-element multiples, bf16 rows 8; K = E; T = 0
    assert moe.padded_rows_max(moe.config(5, 260, 8, 8, 12, dtype=moe.FP32)) == oracle.p_max(5, 8, 8, 16)
    assert moe.padded_rows_max(moe.config(0, 4096, 8, 2, 1024)) == 0


def test_status_strings():
    s = moe.lib().moe_status_string
    assert s(0) == b"ok" and s(-1) == b"invalid argument" and s(-2) == b"workspace too small"
    assert s(-3) == b"CUDA error" and s(-4) == b"device wait timed out"
    assert s(-5) == b"unsupported device (needs sm_100)" and s(7) == b"unknown status"
