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


# ------------------------------------------------------------ tax model
# Demystifying the MoE Serving Tax, "Validation of the analytic model
# (Section 5.3)": the pages' parameters for A100-40GB.
A100 = dict(bw_gbs=1500.0, tflops=312.0)


def test_tax_model_single_token_decode_is_eta_decode():
    # T = 1: the K = 2 activated experts are exactly DenseFA's bytes (I_FA = 2 I),
    # both layers memory-bound, so tau = eta_decode x (1 + router bytes / FFN bytes)
    sh = mi.SHAPES["mixtral"]
    r = bench.tax_model(sh, 1, eta=1.05, **A100)
    assert r["E_active"] == pytest.approx(2.0)
    assert r["regime"] == "memory"
    ffn = 3 * 4096 * 28672 * 2
    assert r["t_fa_s"] == pytest.approx(ffn / 1.5e12)
    assert r["tau"] == pytest.approx(1.05 * (ffn + 8 * 4096 * 2) / ffn)


def test_tax_model_large_prefill_is_eta_prefill():
    # both layers compute-bound with the same expert flops; the MoE layer adds
    # the router's 2 T H E flops
    sh = mi.SHAPES["mixtral"]
    r = bench.tax_model(sh, 65536, eta=1.25, **A100)
    assert r["regime"] == "compute"
    assert r["tau"] == pytest.approx(1.25 * (1 + 8 / (3 * 28672)))
    assert r["t_fa_s"] == pytest.approx(2 * 65536 * 3 * 4096 * 28672 / 312e12)


def test_tax_model_transition_regime():
    # T = 512 on A100: the MoE layer still streams all 8 experts (memory-bound),
    # DenseFA is already compute-bound
    sh = mi.SHAPES["mixtral"]
    r = bench.tax_model(sh, 512, eta=1.25, **A100)
    assert r["regime"] == "transition"
    B, _ = bench.algorithmic(sh, 512, bench.expected_active(8, 2, 512))
    F_fa = 2 * 512 * 3 * 4096 * 28672
    assert r["tau"] == pytest.approx(1.25 * (B / 1.5e12) / (F_fa / 312e12))


def test_tax_model_decode_tax_is_bell_shaped():
    # the pages' decode tax rises from one request to a peak at mid batch sizes
    # and falls at large ones
    sh = mi.SHAPES["qwen2moe"]
    Ts = [2 ** k for k in range(0, 14)]
    tau = [bench.tax_model(sh, T, eta=1.0, **A100)["tau"] for T in Ts]
    peak = max(range(len(tau)), key=lambda i: tau[i])
    assert 0 < peak < len(tau) - 1
    assert all(tau[i] <= tau[i + 1] + 1e-12 for i in range(peak))
    assert all(tau[i] >= tau[i + 1] - 1e-12 for i in range(peak, len(tau) - 1))
    assert tau[0] == pytest.approx((8 * 3 * 3584 * 2560 + 3 * 3584 * 20480 + 64 * 3584) / (3 * 3584 * 40960))


def test_expected_active_closed_forms():
    assert bench.expected_active(8, 2, 1) == pytest.approx(2.0)
    assert bench.expected_active(256, 8, 1) == pytest.approx(8.0)
    assert bench.expected_active(8, 2, 10 ** 6) == pytest.approx(8.0)
    assert bench.expected_active(64, 8, 2) == pytest.approx(64 * (1 - (56 / 64) ** 2))


def test_fit_eta_recovers_a_known_factor():
    ratios = [1.0, 2.5, 4.0, 3.2]
    assert bench.fit_eta([1.17 * r for r in ratios], ratios) == pytest.approx(1.17)


def test_tax_model_report_uses_the_phase_of_each_workload():
    rows = [{"layer": "mixtral", "T": 1, "tau_FA": 1.1, "E_active": 2},
            {"layer": "mixtral", "T": 2048, "tau_FA": 1.2, "E_active": 8}]
    rep = bench.tax_model_report(rows, 6554.6, 1591.5)
    ph = {(p["layer"], p["T"]): p for p in rep["points"]}
    assert ph[("mixtral", 1)]["phase"] == "decode" and ph[("mixtral", 2048)]["phase"] == "prefill"
    # one point per phase: the fitted eta reproduces it exactly
    assert ph[("mixtral", 1)]["err_fitted_eta_pct"] == pytest.approx(0.0, abs=0.05)
    assert ph[("mixtral", 2048)]["tau_model_pages_eta"] == pytest.approx(
        1.25 * bench.tax_model(mi.SHAPES["mixtral"], 2048, 6554.6, 1591.5, 1.0)["tau"], rel=1e-3)


# ------------------------------------------------------- latency fits
def test_fit_latency_models_recovers_known_parameters():
    # exact points of t = max(a + b G, c + beta P) spanning both regimes
    a, b, c, beta = -0.013, 0.0134, 0.118, 1.27e-4
    rows = []
    for G in (2, 8, 32, 64, 128, 200, 256):
        for P in (32, 500, 2000, 8000, 20000, 40000, 65000):
            rows.append({"G": G, "P": P, "ffn_ms": max(a + b * G, c + beta * P)})
    fit = bench.fit_latency_models(rows)
    q = fit["max_affine"]
    assert q["a_ms"] == pytest.approx(a, abs=1e-6)
    assert q["b_ms_per_expert"] == pytest.approx(b, rel=1e-5)
    assert q["c_ms"] == pytest.approx(c, rel=1e-5)
    assert q["beta_ms_per_row"] == pytest.approx(beta, rel=1e-5)
    assert q["r2"] > 0.999999
    pm = fit["padding_model_compute_regime"]
    assert pm["c_ms"] == pytest.approx(c, rel=1e-6) and pm["beta_ms_per_row"] == pytest.approx(beta, rel=1e-6)
    assert pm["r2"] == pytest.approx(1.0)
