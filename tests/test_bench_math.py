"""The benchmark's algorithmic work per layer forward, checked against the
counts written out from their definitions: the bytes are the weights that
must be read once (activated experts, shared FFN, router), the flops two per
multiply-add of every token's router row, expert FFNs and shared FFN."""
import pytest

import bench
import moe_inputs as mi


def test_mixtral_prefill_bytes_and_flops():
    sh = mi.SHAPES["mixtral"]
    B, F = bench.algorithmic(sh, 2048, 8)
    # 8 activated experts x (W1, W3, W2) of 4096 x 14336 bf16, plus W_r [8, 4096]
    assert B == 8 * 3 * 4096 * 14336 * 2 + 8 * 4096 * 2 == 2818637824
    # router 2048 x 4096 x 8, and 2048 x 2 assignments x 3 matrices of 4096 x 14336
    assert F == 2 * (2048 * 4096 * 8 + 2048 * 2 * 3 * 4096 * 14336)


def test_shared_experts_and_dynamic_k_counts():
    sh = mi.SHAPES["qwen2moe"]
    B, F = bench.algorithmic(sh, 32, 61, A=100)
    assert B == 61 * 3 * 3584 * 2560 * 2 + 3 * 3584 * 20480 * 2 + 64 * 3584 * 2
    assert F == 2 * (32 * 3584 * 64 + 32 * 3 * 3584 * 20480 + 100 * 3 * 3584 * 2560)


def test_fp8_bytes_count_codes_and_row_scales():
    sh = mi.SHAPES["deepseekv3"]
    B, _ = bench.algorithmic(sh, 32, 163, fp8=True)
    per_expert = 3 * 7168 * 2048 + 4 * (2 * 2048 + 7168)     # 1-byte codes + fp32 scales per output row
    shared = 3 * 7168 * 2048 + 4 * (2 * 2048 + 7168)
    assert B == 163 * per_expert + shared + 256 * 7168 * 2   # the router stays bf16


@pytest.mark.parametrize("world", [1, 2, 8])
def test_tp_rank_work_splits_all_but_the_router(world):
    sh = mi.SHAPES["mixtral"]
    B, F = bench.algorithmic(sh, 32, 8)
    b, f = bench.tp_rank_work(sh, 32, 8, world)
    router_b, router_f = 8 * 4096 * 2, 2 * 32 * 4096 * 8
    assert world * b == pytest.approx(B + (world - 1) * router_b)
    assert world * f == pytest.approx(F + (world - 1) * router_f)


def test_step_percentiles_nearest_rank():
    t = [float(v) for v in range(1, 21)]          # 1 .. 20 ms
    p = bench.step_percentiles(list(reversed(t)))
    assert p == {"ms_median": 10.5, "ms_p10": 2.0, "ms_p90": 18.0}
    assert bench.step_percentiles([3.0]) == {"ms_median": 3.0, "ms_p10": 3.0, "ms_p90": 3.0}


def test_cpu_baseline_timer_reports_all_threads_and_one_core():
    import numpy as np
    import oracle
    shape = mi.SHAPES["tiny"]
    rng = np.random.default_rng(0)
    T, H, E, I = 16, shape.H, shape.E, shape.I
    x = rng.standard_normal((T, H)).astype(np.float32)
    w_r = (rng.standard_normal((E, H)) / np.sqrt(H)).astype(np.float32)
    w13 = (rng.standard_normal((E, 2 * I, H)) / np.sqrt(H)).astype(np.float32)
    w2 = (rng.standard_normal((E, H, I)) / np.sqrt(I)).astype(np.float32)
    lg = oracle.router_logits(x, w_r).astype(np.float32)
    r = bench.time_oracle(shape, x, w13, w2, {}, lg, budget_s=0.2, budget_1core_s=0.1, nthreads=2)
    assert r["kind"] == "oracle" and r["cores"] == 2 and r["unit"] == "tokens/s"
    assert r["value"] > 0 and r["value_1core"] > 0
    assert "one host thread" in r["sample_1core"]
