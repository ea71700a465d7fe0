#!/usr/bin/env python
"""Benchmark of the B200 MoE layer forward (one step = one forward of the whole
layer: router GEMM, top-K gating, alignment + padding, permute, grouped
gate/up + SwiGLU, grouped down, shared FFN, combine) on synthetic inputs.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload mixtral:2048]
                    [--impl ours|reference] [--sweep]

One JSON line on rank 0.  `value` is whole-job tokens/s with inputs resident in
HBM (device time from CUDA events, L2 flushed between steps, max over ranks);
`e2e` is the same through the C-ABI with the input copied from pinned host
memory and the output read back inside the timed region.  Also reported: the
roofline of the dominant kernel (grouped gate/up), the per-stage breakdown, the
tax tau against the same library's DenseFA and DensePA FFNs, the clocks seen
during the timed region, and the CPU oracle timed on a bounded token sample.
Multi-GPU runs are data-parallel replicas (each rank runs its own batch on its
own full copy of the weights; no collective on the data path).
"""
from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import moe_inputs as mi  # noqa: E402

PEAKS_PATH = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
HBM_NOMINAL_GBS = 8000.0
METRIC = "MoE layer tokens/s; % HBM BW (decode) / % tensor peak (prefill); tau vs DenseFA"
N_INPUT_SETS = 4  # seeded token sets rotated through the timed steps (different routings)
# DRAM bytes per launch of the dominant kernel from one ncu capture of the
# current kernels (dram__bytes_read.sum + dram__bytes_write.sum); workloads
# without a capture report None.  Summaries of the captures are in profiles/.
NCU_TRAFFIC = {
    "mixtral:2048": 2.264e9 + 0.137e9,         # moe_gemm_kernel gate/up + SwiGLU, CTA pairs, aligned tail split
    "mixtral:32": 2.824110e9 + 0.006375e9,     # moe_ffn_stream_kernel, fused decode FFN
    "mixtral:32:fp8": 1.415865e9 + 0.005974e9,  # moe_ffn_stream_kernel, FP8 weights (E4M3 x E4M3 MMAs)
}


def peaks():
    try:
        with open(PEAKS_PATH) as f:
            p = json.load(f)
        return p, "measured"
    except Exception:
        return dict(FALLBACK), "fallback"


# ----------------------------------------------------------------- clocks

class ClockSampler:
    """Samples SM clock and throttle reasons of one GPU through NVML (read only)."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, device_index):
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._h = None
        try:
            import pynvml
            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(device_index)
            bus = "%08X:%02X:%02X.0" % (int(props.pci_domain_id), int(props.pci_bus_id), int(props.pci_device_id))
            self._h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            self._nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._h = None

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                get = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                    getattr(nv, "nvmlDeviceGetCurrentClocksThrottleReasons")
                r = get(self._h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            self._stop.wait(0.005)

    def __enter__(self):
        if self._h is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self._h is not None:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# --------------------------------------------------------------- workload

def parse_workload(s):
    name, T = s.split(":")
    return mi.SHAPES[name], int(T)


class Workload:
    def __init__(self, shape, T, rank=0, device="cuda", skew=None, weights=None, pad_mode=0, dyn_k=False,
                 fp8=False):
        import mixture_experts_layer_61_b200 as moe
        self.moe = moe
        self.shape, self.T = shape, T
        seed = mi.seed_for(shape, T)
        self.w = weights if weights is not None else mi.make_weights(shape, seed, device=device)
        # FP8 expert weights (decode sizes): E4M3 codes + row scales, quantised once here (not timed)
        self.fp8 = fp8
        self.q = {n: moe.quantize_fp8(self.w[n]) for n in ("w13", "w2", "w13_sh", "w2_sh") if fp8 and n in self.w}
        self.x = mi.make_x(shape, T, seed + 100 * rank, device=device)
        self.logits = None
        # per-token dynamic K: each token's count drawn uniformly from 1..K (seeded)
        self.k = None
        self.A = T * shape.K
        if dyn_k:
            g = torch.Generator(device="cpu")
            g.manual_seed(seed + 31)
            self.k = torch.randint(1, shape.K + 1, (T,), generator=g, dtype=torch.int32).to(device)
            self.A = int(self.k.sum().item())
        if skew is not None:
            self.logits = mi.zipf_gumbel_logits(shape.E, T, skew, seed=seed + 17 + 100 * rank, device=device)
        n_sh, I_s = (1, shape.I_sh) if shape.I_sh else (0, 0)
        self.cfg = moe.config(T, shape.H, shape.E, shape.K, shape.I, n_shared=n_sh, I_shared=I_s,
                              tile_B=shape.tile_B, score_fn=shape.score_fn, renorm=shape.renorm,
                              dtype=moe.BF16 if shape.dtype == "bf16" else moe.FP32, pad_mode=pad_mode)
        self.ws = moe.alloc_workspace(moe.workspace_size(self.cfg), device)
        self.stats = torch.zeros(4, dtype=torch.int32, device=device)
        self.out = torch.empty((T, shape.H), dtype=shape.torch_dtype, device=device)
        Pm = moe.padded_rows_max(self.cfg)
        self.Pm = Pm
        dt = shape.torch_dtype
        # buffers of the staged run (the same kernels, one ABI call per stage)
        self.gws = moe.alloc_workspace(moe.gemm_workspace_size(), device)
        self.s_logits = torch.empty((T, shape.E), dtype=torch.float32, device=device)
        self.s_ids = torch.empty((T, shape.K), dtype=torch.int32, device=device)
        self.s_w = torch.empty((T, shape.K), dtype=torch.float32, device=device)
        self.s_xp = torch.empty((Pm, shape.H), dtype=dt, device=device)
        self.s_act = torch.empty((Pm, shape.I), dtype=dt, device=device)
        self.s_y = torch.empty((Pm, shape.H), dtype=dt, device=device)
        self.s_sh = torch.empty((T, shape.H), dtype=dt, device=device) if shape.I_sh else None
        # the FP8 path's token operand: E4M3 hi/lo codes (in s_xp's bytes) and row scales
        self.s_xsc = torch.empty((Pm,), dtype=torch.float32, device=device)
        self.s_shws = None
        if shape.I_sh:
            n = (moe.dense_fp8_workspace_size(T, shape.H, shape.I_sh) if fp8
                 else moe.dense_workspace_size(T, shape.H, shape.I_sh, self.cfg.dtype))
            self.s_shws = moe.alloc_workspace(n, device)
        self.s_al = moe.align_buffers(self.cfg, device)
        self.fused = moe.ffn_fused(self.cfg)

    def capture(self):
        """Record one forward into a CUDA graph (the library makes no allocation
        or synchronisation inside a call, so the whole layer is capturable)."""
        self.step()  # first call outside capture: one-time kernel attribute setup
        torch.cuda.synchronize()
        n0 = self.moe.kernel_launch_count()
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            self.step()
        self.launches_per_step = self.moe.kernel_launch_count() - n0
        torch.cuda.synchronize()

    def replay(self):
        self.graph.replay()

    def step(self):
        m = self.moe
        if self.fp8:
            q, sh = self.q, {}
            if "w13_sh" in q:
                sh = dict(q13_sh=q["w13_sh"][0], s13_sh=q["w13_sh"][1], q2_sh=q["w2_sh"][0], s2_sh=q["w2_sh"][1])
            m.layer_forward_fp8(self.cfg, self.x, self.w["w_r"], q["w13"][0], q["w13"][1], q["w2"][0], q["w2"][1],
                                self.ws, logits_override=self.logits, out=self.out, stats=self.stats, k=self.k, **sh)
            return
        m.layer_forward(self.cfg, self.x, self.w["w_r"], self.w["w13"], self.w["w2"], self.ws,
                        self.w.get("w13_sh"), self.w.get("w2_sh"), self.logits, self.out, self.stats, k=self.k)

    def staged_step(self, ev):
        """The same kernels as step(), one ABI call per stage, events in between."""
        m, c = self.moe, self.cfg
        ev[0].record()
        m.router_gemm(c, self.x, self.w["w_r"], self.gws, self.s_logits)
        ev[1].record()
        m.route(c, self.logits if self.logits is not None else self.s_logits, self.s_ids, self.s_w, k=self.k)
        ev[2].record()
        self.al = m.align_pad(c, self.s_ids, self.s_al)
        ev[3].record()
        if self.fp8:
            m.permute_e4m3x2(c, self.x, self.al["sorted_ids"], self.al["scalars"],
                             self.s_xp.view(torch.uint8).view(2 * self.s_xp.shape[0], -1), self.s_xsc)
        else:
            m.permute(c, self.x, self.al["sorted_ids"], self.al["scalars"], self.s_xp)
        ev[4].record()
        if self.fp8:
            q = self.q
            m.grouped_ffn_fp8(c, self.s_xp.view(torch.uint8).view(2 * self.s_xp.shape[0], -1), self.s_xsc,
                              q["w13"][0], q["w13"][1], q["w2"][0], q["w2"][1], self.al["offsets"],
                              self.gws, self.s_act, self.s_y)
            ev[5].record()
        elif self.fused:
            # the layer's expert FFN is one fused launch (gate/up + SwiGLU + down)
            m.grouped_ffn(c, self.s_xp, self.w["w13"], self.w["w2"], self.al["offsets"], self.gws, self.s_act,
                          self.s_y)
            ev[5].record()
        else:
            m.grouped_gate_up(c, self.s_xp, self.w["w13"], self.al["offsets"], self.gws, self.s_act)
            ev[5].record()
            m.grouped_down(c, self.s_act, self.w["w2"], self.al["offsets"], self.gws, self.s_y)
        ev[6].record()
        if self.s_sh is not None and self.fp8:
            q = self.q
            m.dense_ffn_fp8(self.x, q["w13_sh"][0], q["w13_sh"][1], q["w2_sh"][0], q["w2_sh"][1], self.s_shws,
                            self.s_sh)
        elif self.s_sh is not None:
            m.dense_ffn(self.x, self.w["w13_sh"], self.w["w2_sh"], self.s_shws, self.s_sh)
        ev[7].record()
        m.combine(c, self.s_y, self.al["pos"], self.s_w, self.s_sh, self.out)
        ev[8].record()

    def capture_staged(self):
        """The staged step in one CUDA graph with timing events between the
        stages (event record nodes), so that each stage is timed in the same
        launch context as the step: graph replay, no host launch gaps.
        Returns (replay, events); on a torch without graph event nodes, the
        eager staged step and host-launch events."""
        ev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(9)]
        try:
            self.staged_step(ev)  # outside capture first: one-time kernel attribute setup
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                self.staged_step(ev)
            torch.cuda.synchronize()
            self.staged_graph = g
            return g.replay, ev, "CUDA graph replay of the staged calls (event nodes between stages)"
        except Exception:
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(9)]
            return (lambda: self.staged_step(ev)), ev, "host launches of the staged calls"

    STAGES = ("router", "topk", "align", "permute", "gate_up", "down", "shared", "combine")
    # names when the expert FFN is one fused launch ("down" is then empty)
    STAGES_FUSED = ("router", "topk", "align", "permute", "ffn", "down", "shared", "combine")


def staged_breakdown(wl, warmup, steps, flush):
    """Median per-stage device times (ms) of the staged step, L2 flushed
    before each replay, and how the stages were launched."""
    run, ev, how = wl.capture_staged()
    names = Workload.STAGES_FUSED if wl.fused else Workload.STAGES
    stage_ms = {s: [] for s in names}
    for i in range(warmup + steps):
        flush.zero_()
        run()
        ev[8].synchronize()
        if i >= warmup:
            for j, s in enumerate(names):
                stage_ms[s].append(ev[j].elapsed_time(ev[j + 1]))
    wl.moe.check_status(wl.gws)
    wl.staged_graph = None
    return {s: round(statistics.median(v), 4) for s, v in stage_ms.items() if not (wl.fused and s == "down")}, how


def l2_flush_buffer(device):
    """2 GiB (16x the L2): writing it evicts the L2, and it keeps the GPU busy
    long enough for the host to enqueue a whole step behind it."""
    size = max(2 << 30, 16 * torch.cuda.get_device_properties(device).L2_cache_size)
    return torch.empty(size // 4, dtype=torch.float32, device=device)


def time_steps(fn, steps, flush, stream_sync=True, before=None):
    """Per-step CUDA-event durations (ms), L2 flushed before each step (outside
    the events); before(i) (optional) runs after the flush, also outside."""
    times = []
    for i in range(steps):
        flush.zero_()
        if before is not None:
            before(i)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        b.synchronize()
        times.append(a.elapsed_time(b))
    return times


def step_percentiles(times):
    """Median, p10 and p90 of the per-step times (ms), nearest-rank."""
    v = sorted(times)
    n = len(v)

    def pct(q):
        return v[min(n - 1, max(0, math.ceil(q * n) - 1))]

    return {"ms_median": round(statistics.median(v), 4), "ms_p10": round(pct(0.10), 4),
            "ms_p90": round(pct(0.90), 4)}


# ------------------------------------------------------- multi-rank timing

def max_over_ranks(total_ms, dist, device):
    """The slowest rank's device time (ms); replicas run their own batches, so
    whole-job throughput is set by the slowest one."""
    if dist is None:
        return float(total_ms)
    t = torch.tensor([float(total_ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_tokens_per_s(world, T, steps, max_total_ms):
    """Whole-job tokens/s: every rank processes T tokens per step."""
    return world * T * steps / (max_total_ms / 1e3)


# ------------------------------------------------------------ accounting

def algorithmic(shape, T, E_active, A=None, fp8=False):
    """Algorithmic bytes and flops of one layer forward (padding excluded):
    bytes = weights of the activated experts + shared weights + router weights,
    flops = 2 T (H E + 3 H I_sh) + 2 A 3 H I with A = T K assignments (or
    the sum of the per-token counts under dynamic K)."""
    eb = 2 if shape.dtype == "bf16" else 4
    H, I, E, K = shape.H, shape.I, shape.E, shape.K
    A = T * K if A is None else A
    if fp8:  # 1-byte codes + fp32 row scales for the expert weights; the router stays bf16
        B = E_active * (3 * H * I + 4 * (2 * I + H)) + (3 * H * shape.I_sh + 4 * (2 * shape.I_sh + H)) * (
            shape.I_sh > 0) + E * H * eb
    else:
        B = E_active * 3 * H * I * eb + 3 * H * shape.I_sh * eb + E * H * eb
    F = 2.0 * T * (H * E + 3 * H * shape.I_sh) + 2.0 * A * 3 * H * I
    return B, F


def gate_up_work(shape, T, E_active, A=None):
    """Dominant kernel (grouped gate/up + SwiGLU): weight bytes of the activated
    experts' W1/W3, flops 2 * A * H * 2I (A = T K assignments)."""
    eb = 2 if shape.dtype == "bf16" else 4
    A = T * shape.K if A is None else A
    return E_active * 2 * shape.I * shape.H * eb, 2.0 * A * shape.H * 2 * shape.I


def ffn_work(shape, T, E_active, A=None, fp8=False):
    """Fused expert FFN: weight bytes of the activated experts' W1/W3/W2,
    flops 2 * A * 3 * H * I (A = T K assignments)."""
    eb = 2 if shape.dtype == "bf16" else 4
    A = T * shape.K if A is None else A
    B = E_active * (3 * shape.I * shape.H + 4 * (2 * shape.I + shape.H)) if fp8 else E_active * 3 * shape.I * shape.H * eb
    return B, 2.0 * A * 3 * shape.H * shape.I


def dense_times(shape, T, I_d, steps, warmup, flush, device, seed, fp8=False):
    import mixture_experts_layer_61_b200 as moe
    w13, w2 = mi.make_dense_weights(shape.H, I_d, shape.torch_dtype, seed=seed, device=device)
    x = mi.make_x(shape, T, seed, device=device)
    ws = moe.alloc_workspace(moe.dense_fp8_workspace_size(T, shape.H, I_d) if fp8 else
                             moe.dense_workspace_size(T, shape.H, I_d, 0 if shape.dtype == "bf16" else 1), device)
    out = torch.empty_like(x)
    if fp8:
        (q13, s13), (q2, s2) = moe.quantize_fp8(w13), moe.quantize_fp8(w2)
        del w13, w2
        w13 = w2 = None
        run = lambda: moe.dense_ffn_fp8(x, q13, s13, q2, s2, ws, out)
    else:
        run = lambda: moe.dense_ffn(x, w13, w2, ws, out)
    run()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        run()
    for _ in range(warmup):
        g.replay()
    torch.cuda.synchronize()
    t = time_steps(g.replay, steps, flush)
    moe.check_status(ws)
    del w13, w2, ws
    return statistics.median(t)


# ------------------------------------------------------------ CPU oracle

def oracle_tokens_per_s(wl, budget_s=15.0, max_tokens=None, budget_1core_s=5.0):
    """The oracle as it stands on a bounded sample of the workload's tokens,
    all host cores and one core, routing on the GPU path's logits (read back)."""
    shape = wl.shape
    logits = wl.logits
    if logits is None:
        logits = wl.moe.router_gemm(wl.cfg, wl.x, wl.w["w_r"], wl.gws, wl.s_logits)
    lg = logits.float().cpu().numpy()
    sh = {}
    if shape.I_sh:
        sh = dict(w13_sh=mi.to_oracle(wl.w["w13_sh"]), w2_sh=mi.to_oracle(wl.w["w2_sh"]))
    return time_oracle(shape, mi.to_oracle(wl.x), mi.to_oracle(wl.w["w13"]), mi.to_oracle(wl.w["w2"]), sh, lg,
                       budget_s, max_tokens, budget_1core_s)


def time_oracle(shape, xh, w13, w2, sh, lg, budget_s=15.0, max_tokens=None, budget_1core_s=5.0,
                nthreads=None):
    """Oracle tokens/s on the first tokens of host inputs: a sample sized for
    about budget_s of work on all threads, then one sized for budget_1core_s
    on one thread."""
    import numpy as np
    import oracle
    nthreads = nthreads or os.cpu_count() or 1
    T = xh.shape[0]

    def run(n, threads):
        tok = np.arange(n, dtype=np.int32)
        t0 = time.perf_counter()
        oracle.moe_layer(xh, None, w13, w2, shape.K, shape.score_fn, shape.renorm, logits=lg, tokens=tok,
                         nthreads=threads, **sh)
        return time.perf_counter() - t0

    n = min(T, nthreads)
    t1 = run(n, nthreads)
    per_tok = t1 / n
    n2 = int(max(1, min(T if max_tokens is None else max_tokens, budget_s / max(per_tok, 1e-9))))
    n2 = max(n2 - n2 % nthreads, min(T, nthreads)) if n2 >= nthreads else n2
    t2 = run(n2, nthreads)
    # one core: a token costs about nthreads times the all-threads time per token
    n1 = int(max(1, min(T, budget_1core_s / max(t2 / n2 * nthreads, 1e-9))))
    t3 = run(n1, 1)
    return {"value": n2 / t2, "unit": "tokens/s", "cores": nthreads, "kind": "oracle",
            "sample": f"first {n2} of the {T} tokens of the workload (all {nthreads} host threads, "
                      f"{t2:.1f} s), routing on the GPU path's fp32 logits",
            "value_1core": n1 / t3,
            "sample_1core": f"first {n1} tokens on one host thread ({t3:.1f} s)"}


# ------------------------------------------------------------------- main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="mixtral:2048")
    ap.add_argument("--skew", type=float, default=None, help="Zipf exponent of Gumbel router logits")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-tau", action="store_true")
    ap.add_argument("--no-decode", action="store_true",
                    help="skip the decode block (Mixtral-shaped T=32, DeepSeek-V3-shaped T=128) of the default line")
    ap.add_argument("--sweep", action="store_true", help="also time every configured workload")
    ap.add_argument("--sweep-out", default=None)
    ap.add_argument("--quick", action="store_true",
                    help="only the timed region (for profiler captures): no breakdown, e2e, tau or CPU baseline")
    ap.add_argument("--no-graph", action="store_true", help="launch each step from the host instead of a CUDA graph")
    ap.add_argument("--token-tile-cap", type=int, default=0, help="grouped GEMM token-tile cap (0 = automatic)")
    ap.add_argument("--no-pdl", action="store_true", help="plain stream order between kernels")
    ap.add_argument("--split-tail", type=int, default=-1, choices=[-1, 0, 1],
                    help="GEMM tail schedule: 0 contiguous stream-K, 1 aligned k-slices (-1 = library default)")
    ap.add_argument("--pad-mode", type=int, default=0, choices=[0, 1],
                    help="alignment padding: 0 block-wise, 1 max-value")
    ap.add_argument("--fp8", action="store_true",
                    help="FP8 E4M3 expert weights with row scales (decode sizes)")
    ap.add_argument("--dynamic-k", action="store_true",
                    help="per-token dynamic K: each token's expert count uniform in 1..K (seeded)")
    ap.add_argument("--tax-model", action="store_true",
                    help="time every configured workload and its DenseFA, and compare tau with the analytic model")
    ap.add_argument("--padding-model", action="store_true",
                    help="time the expert FFN over routings and fit the padding and max-affine latency models")
    ap.add_argument("--tp", action="store_true",
                    help="tensor parallelism over I across the ranks: every rank holds I/N of every expert and "
                         "runs the same tokens; one NCCL all-reduce of the fp32 partial output per layer")
    ap.add_argument("--tp-chunks", type=int, default=0,
                    help="with --tp: overlap the all-reduce with the down projection in this many blocks of output "
                         "features (0 = one all-reduce after the whole partial layer)")
    ap.add_argument("--shared-sms", type=int, default=0,
                    help="SMs for the shared experts beside the routed ones (0 = cost model, -1 = serial)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist = None
    if world > 1:
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    shape, T = parse_workload(args.workload)

    if args.impl == "reference":
        return reference_arm(args, shape, T, rank, world, local, dist)

    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    pk, pk_kind = peaks()
    import mixture_experts_layer_61_b200 as moe
    if args.token_tile_cap:
        moe.set_token_tile_cap(args.token_tile_cap)
    if args.no_pdl:
        moe.set_programmatic_launch(False)
    if args.split_tail >= 0:
        moe.set_split_tail(args.split_tail)
    if args.shared_sms:
        moe.set_shared_sms(args.shared_sms)
    flush = l2_flush_buffer(device)
    if args.padding_model:
        if rank == 0:
            print(json.dumps(run_padding_model(args, device, flush)), flush=True)
        if dist:
            dist.barrier()
            dist.destroy_process_group()
        return
    if args.tax_model:
        if rank == 0:
            rows = run_sweep(args, device, flush, pk, skew=False)
            print(json.dumps({"tax_model": tax_model_report(rows, pk["hbm_gbs"], pk["bf16_tflops"]),
                              "peak_source": pk_kind, "rows": rows}), flush=True)
        if dist:
            dist.barrier()
            dist.destroy_process_group()
        return
    if args.tp:
        line = run_tp(args, shape, T, rank, world, local, dist, device, flush, pk, pk_kind)
        if rank == 0:
            print(json.dumps(line), flush=True)
        if dist:
            dist.barrier()
            dist.destroy_process_group()
        return
    wl = Workload(shape, T, rank, device, skew=args.skew, pad_mode=args.pad_mode, dyn_k=args.dynamic_k,
                  fp8=args.fp8)
    if args.no_graph:
        run_step, wl.launches_per_step = wl.step, None
    else:
        wl.capture()
        run_step = wl.replay
    for _ in range(args.warmup):
        run_step()
    torch.cuda.synchronize()
    wl.moe.check_status(wl.ws)

    # ---- timed region: K steps of the fused layer call, rotating R seeded token
    # sets (different routings) into the input buffer before each step, outside
    # the events like the L2 flush
    seed = mi.seed_for(shape, T)
    x_sets = [wl.x.clone()] + [mi.make_x(shape, T, seed + 100 * rank + 10 * j, device=device)
                               for j in range(1, N_INPUT_SETS)]

    def rotate(i):
        wl.x.copy_(x_sets[i % N_INPUT_SETS])

    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    n0 = wl.moe.kernel_launch_count()
    with ClockSampler(local) as clk:
        times = time_steps(run_step, args.steps, flush, before=rotate)
    torch.cuda.synchronize()
    launches = wl.moe.kernel_launch_count() - n0
    if not args.no_graph:
        launches = wl.launches_per_step * args.steps  # graph replays launch the captured kernels
    if dist:
        dist.barrier()
    total_ms = max_over_ranks(sum(times), dist, device)
    wl.moe.check_status(wl.ws)
    stats = wl.stats.cpu().tolist()
    P, E_active = stats[0], stats[1]
    ms_step = total_ms / args.steps
    value = replica_tokens_per_s(world, T, args.steps, total_ms)
    # ---- per-stage breakdown (same kernels, one ABI call per stage, replayed
    # from a CUDA graph with event nodes between the stages)
    stages, staged_launch = staged_breakdown(wl, args.warmup, args.steps, flush)

    if args.quick:
        if rank == 0:
            print(json.dumps({"metric": METRIC, "value": round(value, 2), "unit": "tokens/s", "n_gpus": world,
                              "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
                              "quick": True, "config": {"workload": f"{shape.name}:{T}",
                                                        "token_tile_cap": args.token_tile_cap,
                                                        "pdl": not args.no_pdl,
                                                        "shared_sms": moe.shared_sms(wl.cfg),
                                                        "pad_mode": args.pad_mode, "dynamic_k": args.dynamic_k,
                                                        "fp8": args.fp8, "split_tail": args.split_tail},
                              "stages_ms": stages, "E_active": E_active, "P": P}), flush=True)
        if dist:
            dist.barrier()
            dist.destroy_process_group()
        return

    # ---- roofline of the dominant kernel: the grouped gate/up + SwiGLU GEMM,
    # or the fused expert FFN when the layer runs it as one launch
    if wl.fused:
        gu_bytes, gu_flops = ffn_work(shape, T, E_active, wl.A, fp8=args.fp8)
        t_gu = stages["ffn"] * 1e-3
    else:
        gu_bytes, gu_flops = gate_up_work(shape, T, E_active, wl.A)
        t_gu = stages["gate_up"] * 1e-3
    hbm_peak = pk["hbm_gbs"]
    tc_peak = pk["bf16_tflops"] * (0.5 if shape.dtype == "fp32" else 1.0)  # tf32 is half the bf16 rate
    bound = "tensor" if gu_flops / (tc_peak * 1e12) > gu_bytes / (hbm_peak * 1e9) else "hbm"
    if bound == "hbm":
        ach = gu_bytes / t_gu / 1e9
        roof = {"bound": "hbm", "achieved": round(ach, 1), "peak": hbm_peak, "unit": "GB/s",
                "frac": round(ach / hbm_peak, 4), "frac_of_8TBs": round(ach / HBM_NOMINAL_GBS, 4)}
    else:
        ach = gu_flops / t_gu / 1e12
        roof = {"bound": "tensor", "achieved": round(ach, 1), "peak": tc_peak, "unit": "TFLOP/s",
                "frac": round(ach / tc_peak, 4), "frac_of_sustained": round(ach / pk["bf16_tflops_sustained"], 4)}
    roof["kernel"] = ("moe_ffn_stream_kernel (fused expert FFN: gate/up + SwiGLU + down)" if wl.fused
                      else "moe_gemm_kernel (grouped gate/up + SwiGLU)") + (", FP8 weights" if args.fp8 else "")
    roof["peak_source"] = f"{pk_kind} ({'MEASURED_PEAKS.json' if pk_kind == 'measured' else 'fallback'})"
    roof["traffic"] = NCU_TRAFFIC.get(f"{shape.name}:{T}" + (":fp8" if args.fp8 else ""))
    B_alg, F_alg = algorithmic(shape, T, E_active, wl.A, fp8=args.fp8)
    t_layer = ms_step * 1e-3
    layer_roof = max(F_alg / (tc_peak * 1e12), B_alg / (hbm_peak * 1e9)) / t_layer

    # ---- e2e through the C-ABI with host buffers
    x_host = torch.empty(wl.x.shape, dtype=wl.x.dtype, pin_memory=True)
    x_host.copy_(wl.x)
    out_host = torch.empty(wl.out.shape, dtype=wl.out.dtype, pin_memory=True)

    def e2e_step():
        wl.x.copy_(x_host, non_blocking=True)
        run_step()
        out_host.copy_(wl.out, non_blocking=True)

    for _ in range(args.warmup):
        e2e_step()
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    e2e_times = time_steps(e2e_step, args.steps, flush)
    e2e_total = max_over_ranks(sum(e2e_times), dist, device)
    e2e = {"value": replica_tokens_per_s(world, T, args.steps, e2e_total), "unit": "tokens/s",
           "h2d_bytes_per_step": x_host.numel() * x_host.element_size(),
           "d2h_bytes_per_step": out_host.numel() * out_host.element_size()}

    # ---- tau against DenseFA / DensePA (same library, same T)
    tau = None
    if not args.no_tau:
        seed = mi.seed_for(shape, T, 50)
        t_fa = dense_times(shape, T, shape.I_FA, args.steps, args.warmup, flush, device, seed, fp8=args.fp8)
        t_pa = dense_times(shape, T, shape.I_PA, args.steps, args.warmup, flush, device, seed + 1, fp8=args.fp8)
        t_moe = statistics.median(times)
        tau = {"tau_FA": round(t_moe / t_fa, 4), "tau_PA": round(t_moe / t_pa, 4),
               "t_moe_ms": round(t_moe, 4), "t_DenseFA_ms": round(t_fa, 4), "t_DensePA_ms": round(t_pa, 4),
               "I_FA": shape.I_FA, "I_PA": shape.I_PA}

    decode = None
    if not args.no_decode:
        decode = decode_block(device, flush, pk, args.steps, args.warmup, rank)

    sweep = None
    if args.sweep:
        sweep = run_sweep(args, device, flush, pk)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = oracle_tokens_per_s(wl)

    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 4),
        **step_percentiles(times),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if shape.dtype == "bf16" else "f32",
        "data": "synthetic (seeded Gaussian weights/activations of the layer's shape; "
                + ("router logits x.W_r" if args.skew is None else f"Zipf({args.skew}) Gumbel logits") + ")",
        "config": {"workload": f"{shape.name}-shaped MoE layer forward, T={T}", "T": T, "H": shape.H,
                   "E": shape.E, "K": shape.K, "I": shape.I, "I_shared": shape.I_sh, "tile_B": shape.tile_B,
                   "score_fn": "softmax" if shape.score_fn == 0 else "sigmoid", "global_batch": T * world,
                   "parallelism": f"replicas x{world} (data parallel, no collective)",
                   "launch": "host launches" if args.no_graph else "CUDA graph replay of moe_layer_forward",
                   "l2": "flushed between steps (2 GiB write outside the events); weights exceed L2",
                   "inputs": f"{N_INPUT_SETS} seeded token sets rotated step by step (copied in outside the events)",
                   "shared_sms": moe.shared_sms(wl.cfg),
                   "padding": "max-value" if args.pad_mode == 1 else "block-wise",
                   "top_k": (f"per-token dynamic, uniform 1..{shape.K} (sum {wl.A})" if args.dynamic_k
                             else f"{shape.K} for every token"),
                   "expert_weights": ("FP8 E4M3 codes + fp32 row scales (widened to f16 in TMEM, f16 MMAs)"
                                      if args.fp8 else shape.dtype)},
        "roofline": roof,
        "layer": {"P": P, "E_active": E_active, "padded_fraction": round((P - wl.A) / max(P, 1), 4),
                  "bytes_alg": B_alg, "flops_alg": F_alg, "roofline_frac": round(layer_roof, 4),
                  "hbm_GBs_alg": round(B_alg / t_layer / 1e9, 1), "tflops_alg": round(F_alg / t_layer / 1e12, 2)},
        "stages_ms": stages,
        "staged_total_ms": round(sum(stages.values()), 4),
        "staged_launch": staged_launch,
        "tau": tau,
        "decode": decode,
        "e2e": e2e,
        "gpu_launches": launches,
        "clocks": clk.summary(),
        "cpu_baseline": cpu,
    }
    if sweep is not None:
        line["sweep"] = sweep
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


DECODE_POINTS = (("mixtral", 32), ("deepseekv3", 128))


def decode_block(device, flush, pk, steps, warmup, rank=0):
    """The HBM-bound half of the metric on the default line: decode-sized
    layers (the Mixtral-8x7B-shaped layer at T = 32 and the largest
    single-GPU configuration, the DeepSeek-V3-shaped layer at T = 128), each
    timed like the headline (CUDA graph replay, L2 flushed before every step,
    four rotated token sets), with the fused expert FFN's stage time, the
    fractions of the measured copy bandwidth and of 8 TB/s, and tau against
    DenseFA at the same T."""
    out = []
    for name, T in DECODE_POINTS:
        sh = mi.SHAPES[name]
        wl = Workload(sh, T, rank, device)
        wl.capture()
        for _ in range(warmup):
            wl.replay()
        torch.cuda.synchronize()
        seed = mi.seed_for(sh, T)
        xs = [wl.x.clone()] + [mi.make_x(sh, T, seed + 100 * rank + 10 * j, device=device)
                               for j in range(1, N_INPUT_SETS)]
        times = time_steps(wl.replay, steps, flush, before=lambda i: wl.x.copy_(xs[i % N_INPUT_SETS]))
        wl.moe.check_status(wl.ws)
        st = wl.stats.cpu().tolist()
        stages, _ = staged_breakdown(wl, 3, max(5, steps // 2), flush)
        t = statistics.median(times)
        B, F = algorithmic(sh, T, st[1])
        fb, _ = ffn_work(sh, T, st[1])
        t_ffn = stages.get("ffn") or (stages["gate_up"] + stages["down"])
        del wl, xs
        torch.cuda.empty_cache()
        t_fa = dense_times(sh, T, sh.I_FA, max(5, steps // 2), 3, flush, device, mi.seed_for(sh, T, 50))
        out.append({"workload": f"{name}:{T}", "ms_median": round(t, 4), "tokens_per_s": round(T / t * 1e3, 1),
                    "E_active": st[1], "P": st[0], "bytes_alg": B,
                    "hbm_GBs_alg": round(B / t / 1e6, 1),
                    "hbm_frac_measured": round(B / (t * 1e-3) / (pk["hbm_gbs"] * 1e9), 4),
                    "hbm_frac_8TBs": round(B / (t * 1e-3) / (HBM_NOMINAL_GBS * 1e9), 4),
                    "ffn_ms": round(t_ffn, 4),
                    "ffn_hbm_frac_measured": round(fb / (t_ffn * 1e-3) / (pk["hbm_gbs"] * 1e9), 4),
                    "tau_FA": round(t / t_fa, 4), "t_DenseFA_ms": round(t_fa, 4)})
        torch.cuda.empty_cache()
    return out


def tp_rank_work(shape, T, E_active, world):
    """Algorithmic bytes and flops of one rank under TP over I: its 1/world
    share of the experts' and the shared FFN's, plus the whole router (every
    rank routes all tokens)."""
    B_alg, F_alg = algorithmic(shape, T, E_active)
    eb = 2 if shape.dtype == "bf16" else 4
    B_r, F_r = shape.E * shape.H * eb, 2.0 * T * shape.H * shape.E
    return (B_alg - B_r) / world + B_r, (F_alg - F_r) / world + F_r


def tp_tokens_per_s(T, steps, max_total_ms):
    """TP: every rank works on the same T tokens, so the job's throughput is
    T per step over the slowest rank's device time."""
    return T * steps / (max_total_ms * 1e-3)


def run_tp(args, shape, T, rank, world, local, dist, device, flush, pk, pk_kind):
    """The layer under tensor parallelism over I on `world` ranks (strong
    scaling): each rank slices every expert and the shared FFN, computes its
    fp32 partial output (one CUDA graph of the layer's kernels), NCCL sums the
    partials across the ranks, and one kernel rounds the sum."""
    import mixture_experts_layer_61_b200 as moe
    seed = mi.seed_for(shape, T)
    w = mi.make_weights(shape, seed, device=device)
    x = mi.make_x(shape, T, seed, device=device)           # the same tokens on every rank
    n_sh, I_s = (1, shape.I_sh) if shape.I_sh else (0, 0)
    cfg = moe.config(T, shape.H, shape.E, shape.K, shape.I, n_shared=n_sh, I_shared=I_s, tile_B=shape.tile_B,
                     score_fn=shape.score_fn, renorm=shape.renorm,
                     dtype=moe.BF16 if shape.dtype == "bf16" else moe.FP32, pad_mode=args.pad_mode)
    cl = moe.tp_config(cfg, world)
    w13, w2 = moe.tp_shard(w["w13"], w["w2"], rank, world)
    sh = moe.tp_shard(w["w13_sh"], w["w2_sh"], rank, world) if shape.I_sh else (None, None)
    w_r = w["w_r"]
    del w
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    ws = moe.alloc_workspace(moe.workspace_size(cl), device)
    stats = torch.zeros(4, dtype=torch.int32, device=device)
    partial = torch.empty((T, shape.H), dtype=torch.float32, device=device)
    out = torch.empty((T, shape.H), dtype=x.dtype, device=device)

    overlap = args.tp_chunks > 0 and not moe.ffn_fused(cl)
    n_chunks = args.tp_chunks if overlap else 0
    parts = [torch.empty((T, shape.H // n_chunks), dtype=torch.float32, device=device)
             for _ in range(n_chunks)]

    def layer():
        if overlap:   # routing, permute, gate/up and the shared FFN; the down blocks follow per step
            moe.layer_forward_partial_front(cl, x, w_r, w13, ws, sh[0], sh[1], stats=stats)
        else:
            moe.layer_forward_partial(cl, x, w_r, w13, w2, ws, sh[0], sh[1], out=partial, stats=stats)

    layer()
    torch.cuda.synchronize()
    n0 = moe.kernel_launch_count()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        layer()
    per_graph = moe.kernel_launch_count() - n0 + (2 * n_chunks + 1 if overlap else 1)
    torch.cuda.synchronize()

    def step():
        graph.replay()
        if overlap:
            # each block's down projection + combine, its all-reduce started
            # beside the next block's kernels; then the blocks side by side, rounded
            moe.tp_overlapped_allreduce(
                parts, lambda c: moe.layer_forward_partial_down(cl, w2, c, n_chunks, ws, parts[c]))
            moe.tp_gather(parts, out)
        else:
            moe.tp_allreduce(partial)             # NCCL all-reduce (no-op on one rank)
            moe.tp_reduce([partial], out)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    moe.check_status(ws)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        times = time_steps(step, args.steps, flush)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    total_ms = max_over_ranks(sum(times), dist, device)
    moe.check_status(ws)
    P, E_active = stats.cpu().tolist()[:2]
    ms_step = total_ms / args.steps
    # per-rank algorithmic work: this rank's slice of the layer's weights and flops
    B_rank, F_rank = tp_rank_work(shape, T, E_active, world)
    hbm_peak = pk["hbm_gbs"]
    tc_peak = pk["bf16_tflops"] * (0.5 if shape.dtype == "fp32" else 1.0)
    t = ms_step * 1e-3
    if F_rank / (tc_peak * 1e12) > B_rank / (hbm_peak * 1e9):
        ach = F_rank / t / 1e12
        roof = {"bound": "tensor", "achieved": round(ach, 1), "peak": tc_peak, "unit": "TFLOP/s",
                "frac": round(ach / tc_peak, 4)}
    else:
        ach = B_rank / t / 1e9
        roof = {"bound": "hbm", "achieved": round(ach, 1), "peak": hbm_peak, "unit": "GB/s",
                "frac": round(ach / hbm_peak, 4)}
    roof.update({"kernel": "whole TP step per rank (slice of the layer + all-reduce + rounding)",
                 "peak_source": f"{pk_kind} ({'MEASURED_PEAKS.json' if pk_kind == 'measured' else 'fallback'})",
                 "traffic": None})
    # e2e: tokens from pinned host memory, the rounded output back
    x_host = torch.empty(x.shape, dtype=x.dtype, pin_memory=True)
    x_host.copy_(x)
    out_host = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)

    def e2e_step():
        x.copy_(x_host, non_blocking=True)
        step()
        out_host.copy_(out, non_blocking=True)

    for _ in range(args.warmup):
        e2e_step()
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    e2e_total = max_over_ranks(sum(time_steps(e2e_step, args.steps, flush)), dist, device)
    del graph
    return {
        "metric": METRIC, "value": round(tp_tokens_per_s(T, args.steps, total_ms), 2), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
        "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
        "dtype": "bf16" if shape.dtype == "bf16" else "f32",
        "data": "synthetic (seeded Gaussian weights/activations of the layer's shape; router logits x.W_r)",
        "config": {"workload": f"{shape.name}-shaped MoE layer forward, T={T}", "T": T, "H": shape.H,
                   "E": shape.E, "K": shape.K, "I": shape.I, "I_per_rank": cl.I, "I_shared": shape.I_sh,
                   "tile_B": shape.tile_B, "global_batch": T,
                   "parallelism": (f"TP over I x{world} (all-reduce of the fp32 partial output in {n_chunks} blocks "
                                   "of output features, each beside the next block's down projection)" if overlap else
                                   f"TP over I x{world} (one all-reduce of the fp32 partial output per layer)"),
                   "launch": ("CUDA graph of the front part (routing, gate/up, shared FFN), then per block the down "
                              "projection + combine and an async all-reduce, then the gather kernel" if overlap else
                              "CUDA graph of the partial layer, then the all-reduce and the rounding kernel"),
                   "l2": "flushed between steps (2 GiB write outside the events)"},
        "roofline": roof,
        "layer": {"P": P, "E_active": E_active, "bytes_alg_per_rank": B_rank, "flops_alg_per_rank": F_rank},
        "e2e": {"value": tp_tokens_per_s(T, args.steps, e2e_total), "unit": "tokens/s",
                "h2d_bytes_per_step": x_host.numel() * x_host.element_size(),
                "d2h_bytes_per_step": out_host.numel() * out_host.element_size()},
        "gpu_launches": per_graph * args.steps,
        "clocks": clk.summary(),
        "cpu_baseline": None,
    }


# ---------------------------------------------------- analytic tax model
# Demystifying the MoE Serving Tax, "Validation of the analytic model
# (Section 5.3)": the pages give the model's parameters for A100-40GB
# (HBM 1500 GB/s, 312 TFLOP/s bf16, padding overhead eta = 1.05 in decode and
# 1.25 in prefill), its three regimes (memory-bound, compute-bound and the
# transition between them) and its accuracy (within 10-30 % of measured), not
# its formula.  Reading taken here, the plainest one the printed endpoints
# support: each layer takes the roofline time of its algorithmic bytes and
# flops, the MoE layer's multiplied by the phase's eta,
#   t_MoE = eta * max(B_MoE / BW, F_MoE / FLOPS),  t_FA = max(B_FA / BW, F_FA / FLOPS),
#   tau = t_MoE / t_FA,
# with B_MoE counting the expected activated experts E (1 - (1 - K/E)^T)
# ("Balls-Bins-Buckets").  At T = 1 both layers read the same expert bytes and
# tau = eta_decode (the pages: 1.05x for Mixtral at one request); at large T
# both are compute-bound with equal flops and tau = eta_prefill (the pages:
# about 1.28x at 1024-2048 tokens).
PAGES_TAX_MODEL = {"hardware": "A100-40GB (the pages' validation)", "bw_gbs": 1500.0, "tflops": 312.0,
                   "eta_decode": 1.05, "eta_prefill": 1.25}


def expected_active(E, K, T):
    """E[E_active] = E (1 - (1 - K/E)^T) under uniform routing (talk notes,
    "Balls-Bins-Buckets" model construction)."""
    return E * (1.0 - (1.0 - K / E) ** T)


def dense_fa_work(shape, T):
    """DenseFA's algorithmic bytes (its weights, read once) and flops: a dense
    SwiGLU FFN of width I_FA = K I + S I_s, no router."""
    eb = 2 if shape.dtype == "bf16" else 4
    return 3.0 * shape.H * shape.I_FA * eb, 2.0 * T * 3 * shape.H * shape.I_FA


def tax_model(shape, T, bw_gbs, tflops, eta, E_active=None):
    """Predicted MoE and DenseFA layer times (s), tau and the regime."""
    if E_active is None:
        E_active = expected_active(shape.E, shape.K, T)
    B_m, F_m = algorithmic(shape, T, E_active)
    B_d, F_d = dense_fa_work(shape, T)
    bw, fl = bw_gbs * 1e9, tflops * 1e12
    mem_m, cmp_m = B_m / bw, F_m / fl
    mem_d, cmp_d = B_d / bw, F_d / fl
    t_m, t_d = eta * max(mem_m, cmp_m), max(mem_d, cmp_d)
    if mem_m >= cmp_m and mem_d >= cmp_d:
        regime = "memory"
    elif mem_m < cmp_m and mem_d < cmp_d:
        regime = "compute"
    else:
        regime = "transition"
    return {"t_moe_s": t_m, "t_fa_s": t_d, "tau": t_m / t_d, "regime": regime, "E_active": E_active}


def phase_of(shape, T):
    return "prefill" if T in shape.prefill_T else "decode"


def fit_eta(taus, ratios):
    """Least-squares eta of tau = eta * ratio (ratio: the roofline tau with
    eta = 1) over a phase's points."""
    num = sum(t * r for t, r in zip(taus, ratios))
    den = sum(r * r for r in ratios)
    return num / den if den > 0 else float("nan")


def tax_model_report(rows, bw_gbs, tflops):
    """Predicted against measured tau_FA for every measured configuration
    (rows: layer, T, tau_FA), with the pages' eta constants on this GPU's
    peaks and with eta fitted per phase to the measurements."""
    pts = []
    for r in rows:
        sh = mi.SHAPES[r["layer"]]
        ph = phase_of(sh, r["T"])
        base = tax_model(sh, r["T"], bw_gbs, tflops, 1.0)
        pts.append((r, sh, ph, base))
    eta_fit = {}
    for ph in ("decode", "prefill"):
        sel = [(r["tau_FA"], b["tau"]) for r, sh, p, b in pts if p == ph]
        eta_fit[ph] = fit_eta([a for a, _ in sel], [b for _, b in sel]) if sel else None
    table = []
    for r, sh, ph, b in pts:
        e_pages = PAGES_TAX_MODEL["eta_" + ph]
        tp, tf = e_pages * b["tau"], eta_fit[ph] * b["tau"]
        table.append({"layer": r["layer"], "T": r["T"], "phase": ph, "regime": b["regime"],
                      "tau_measured": r["tau_FA"], "tau_model_pages_eta": round(tp, 4),
                      "err_pages_eta_pct": round(100.0 * (tp - r["tau_FA"]) / r["tau_FA"], 1),
                      "tau_model_fitted_eta": round(tf, 4),
                      "err_fitted_eta_pct": round(100.0 * (tf - r["tau_FA"]) / r["tau_FA"], 1),
                      "E_active_model": round(b["E_active"], 2), "E_active_measured": r.get("E_active")})
    return {"bw_gbs": bw_gbs, "tflops": tflops, "eta_pages": {"decode": PAGES_TAX_MODEL["eta_decode"],
                                                               "prefill": PAGES_TAX_MODEL["eta_prefill"]},
            "eta_fitted": eta_fit, "points": table}


def run_sweep(args, device, flush, pk, skew=True):
    """Every configured workload (decode and prefill T of each layer shape) and
    the DeepSeek-V3-shaped routing-skew sweep (Zipf s in {0, 0.5, 1, 1.5},
    T = 1 .. 4096 in powers of two): tokens/s, activated experts, padded
    fraction, roofline fractions and tau against DenseFA (same T, same
    library).  Weights are generated once per layer shape."""
    import mixture_experts_layer_61_b200 as moe
    rows = []
    steps = max(5, args.steps // 2)
    for name in ("mixtral", "qwen2moe", "deepseekv3"):
        sh = mi.SHAPES[name]
        weights = mi.make_weights(sh, mi.seed_for(sh, 0), device=device)
        plan = [(T, None) for T in sh.decode_T + sh.prefill_T]
        if name == "deepseekv3" and skew:
            plan += [(2 ** k, s) for s in (0.0, 0.5, 1.0, 1.5) for k in range(13)]
        fa_cache = {}
        for T, s in plan:
            wl = Workload(sh, T, 0, device, skew=s, weights=weights)
            wl.capture()
            for _ in range(3):
                wl.replay()
            torch.cuda.synchronize()
            t = statistics.median(time_steps(wl.replay, steps, flush))
            moe.check_status(wl.ws)
            st = wl.stats.cpu().tolist()
            B, F = algorithmic(sh, T, st[1])
            if T not in fa_cache:
                fa_cache[T] = dense_times(sh, T, sh.I_FA, steps, 3, flush, device, mi.seed_for(sh, T, 50))
            row = {"layer": sh.name, "T": T, "skew": s, "ms": round(t, 4), "tokens_per_s": round(T / t * 1e3, 1),
                   "E_active": st[1], "P": st[0],
                   "padded_fraction": round((st[0] - T * sh.K) / max(st[0], 1), 4),
                   "hbm_frac_8TBs": round(B / (t * 1e-3) / 8e12, 4),
                   "hbm_frac_measured": round(B / (t * 1e-3) / (pk["hbm_gbs"] * 1e9), 4),
                   "tensor_frac": round(F / (t * 1e-3) / (pk["bf16_tflops"] * 1e12), 4),
                   "roofline_frac": round(max(F / (pk["bf16_tflops"] * 1e12), B / (pk["hbm_gbs"] * 1e9)) /
                                          (t * 1e-3), 4),
                   "tau_FA": round(t / fa_cache[T], 4), "fused_ffn": bool(wl.fused),
                   "shared_sms": moe.shared_sms(wl.cfg)}
            rows.append(row)
            if args.sweep_out:
                with open(args.sweep_out, "a") as f:
                    f.write(json.dumps(row) + "\n")
            del wl
            torch.cuda.empty_cache()
        del weights
        torch.cuda.empty_cache()
    return rows


def ffn_time(wl, steps, flush):
    """Median device time (ms) of the routed expert FFN alone (the fused
    launch, or gate/up + down), from the per-stage events of staged steps."""
    run, ev, _ = wl.capture_staged()
    names = Workload.STAGES_FUSED if wl.fused else Workload.STAGES
    out = []
    for i in range(3 + steps):
        flush.zero_()
        run()
        ev[8].synchronize()
        if i >= 3:
            st = {s: ev[j].elapsed_time(ev[j + 1]) for j, s in enumerate(names)}
            out.append(st["ffn"] if wl.fused else st["gate_up"] + st["down"])
    wl.moe.check_status(wl.gws)
    return statistics.median(out)


def fit_latency_models(rows):
    """Least-squares fits of the expert-FFN time t (ms) over the sweep points:
    the padding model t = c + beta * P on the points in the compute regime
    (Demystifying the MoE Serving Tax, "Padding model (Section 5.1)": latency
    from the padded rows P), and the max-affine profile
    t = max(a + b * G, c + beta * N) of the TEMPO write-up (G activated
    experts, N rows the kernel computes = P) on all points.  G counts the
    experts whose weights the kernel streams: the activated ones under
    block-wise padding, all E under max-value padding."""
    import numpy as np
    from scipy.optimize import least_squares
    G = np.array([r["G"] for r in rows], float)
    P = np.array([r["P"] for r in rows], float)
    t = np.array([r["ffn_ms"] for r in rows], float)

    def r2(pred):
        return float(1.0 - ((t - pred) ** 2).sum() / max(((t - t.mean()) ** 2).sum(), 1e-30))

    mem = np.polyfit(G, t, 1)      # t ~ a + b G
    comp = np.polyfit(P, t, 1)     # t ~ c + beta P
    x0 = [mem[1], mem[0], comp[1], comp[0]]
    f = lambda q: np.maximum(q[0] + q[1] * G, q[2] + q[3] * P) - t
    q = least_squares(f, x0).x
    pred = np.maximum(q[0] + q[1] * G, q[2] + q[3] * P)
    compute = (q[2] + q[3] * P) > (q[0] + q[1] * G)
    out = {"max_affine": {"a_ms": q[0], "b_ms_per_expert": q[1], "c_ms": q[2], "beta_ms_per_row": q[3],
                          "r2": r2(pred), "points": int(len(t)), "compute_regime_points": int(compute.sum())},
           "linear_in_P_all_points": {"r2": r2(np.polyval(comp, P))}}
    if compute.sum() >= 3:
        pc = np.polyfit(P[compute], t[compute], 1)
        tc = t[compute]
        out["padding_model_compute_regime"] = {
            "c_ms": pc[1], "beta_ms_per_row": pc[0],
            "r2": float(1.0 - ((tc - np.polyval(pc, P[compute])) ** 2).sum() / max(((tc - tc.mean()) ** 2).sum(), 1e-30))}
    return out


def run_padding_model(args, device, flush):
    """Expert-FFN time over routings of the DeepSeek-V3-shaped layer: T = 1..4096
    with Zipf(s) Gumbel logits, s in {0, 0.5, 1, 1.5}, block-wise padding; and
    T = 1..128 with max-value padding.  Each point records E_active, P and the
    FFN time; the fits follow (fit_latency_models)."""
    import mixture_experts_layer_61_b200 as moe
    sh = mi.SHAPES["deepseekv3"]
    weights = mi.make_weights(sh, mi.seed_for(sh, 0), device=device)
    plan = [(0, 2 ** k, s) for s in (0.0, 0.5, 1.0, 1.5) for k in range(13)]
    plan += [(1, 2 ** k, s) for s in (0.0, 1.5) for k in range(8)]
    rows = []
    for mode, T, s in plan:
        wl = Workload(sh, T, 0, device, skew=s, weights=weights, pad_mode=mode)
        t = ffn_time(wl, max(3, args.steps // 4), flush)
        st = wl.al["scalars"].cpu().tolist()
        G = int((torch.diff(wl.al["offsets"]) > 0).sum().item())  # segments with rows: experts streamed
        row = {"layer": sh.name, "pad_mode": mode, "T": T, "skew": s, "E_active": st[1], "G": G, "P": st[0],
               "A": T * sh.K, "ffn_ms": round(t, 4), "fused_ffn": bool(wl.fused)}
        rows.append(row)
        if args.sweep_out:
            with open(args.sweep_out, "a") as f:
                f.write(json.dumps(row) + "\n")
        del wl
        torch.cuda.empty_cache()
    fits = {"block-wise": fit_latency_models([r for r in rows if r["pad_mode"] == 0]),
            "all": fit_latency_models(rows)}
    mv = [r for r in rows if r["pad_mode"] == 1]
    bw = {(r["T"], r["skew"]): r for r in rows if r["pad_mode"] == 0}
    compare = [{"T": r["T"], "skew": r["skew"], "P_block": bw[(r["T"], r["skew"])]["P"], "P_max_value": r["P"],
                "ms_block": bw[(r["T"], r["skew"])]["ffn_ms"], "ms_max_value": r["ffn_ms"]} for r in mv]
    return {"padding_model": fits, "max_value_vs_block": compare, "layer": sh.name, "points": len(rows)}


def reference_arm(args, shape, T, rank, world, local, dist):
    """The CPU oracle as the reference implementation, on rank 0 only: each step
    runs the oracle over a bounded sample of the workload's tokens."""
    if rank != 0:
        if dist:
            dist.destroy_process_group()
        return
    import numpy as np
    import oracle
    seed = mi.seed_for(shape, T)
    w = mi.make_weights(shape, seed, device="cuda" if torch.cuda.is_available() else "cpu")
    x = mi.make_x(shape, T, seed, device=w["w_r"].device)
    xh, wr = mi.to_oracle(x), mi.to_oracle(w["w_r"])
    w13, w2 = mi.to_oracle(w["w13"]), mi.to_oracle(w["w2"])
    sh = {}
    if shape.I_sh:
        sh = dict(w13_sh=mi.to_oracle(w["w13_sh"]), w2_sh=mi.to_oracle(w["w2_sh"]))
    nthreads = os.cpu_count() or 1
    # size the per-step sample so that warmup + steps stay within ~2 minutes
    t0 = time.perf_counter()
    oracle.moe_layer(xh, wr, w13, w2, shape.K, shape.score_fn, shape.renorm,
                     tokens=np.arange(min(T, nthreads), dtype=np.int32), nthreads=nthreads, **sh)
    per_tok = (time.perf_counter() - t0) / min(T, nthreads)
    n = int(max(1, min(T, 120.0 / (args.steps + args.warmup) / per_tok)))
    tok = np.arange(n, dtype=np.int32)
    for _ in range(args.warmup):
        oracle.moe_layer(xh, wr, w13, w2, shape.K, shape.score_fn, shape.renorm, tokens=tok, nthreads=nthreads, **sh)
    ts = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle.moe_layer(xh, wr, w13, w2, shape.K, shape.score_fn, shape.renorm, tokens=tok, nthreads=nthreads, **sh)
        ts.append(time.perf_counter() - t0)
    total = sum(ts)
    value = n * args.steps / total
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "tokens/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(total / args.steps * 1e3, 2),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic",
            "config": {"workload": f"{shape.name}-shaped MoE layer forward, T={T}", "T": T, "H": shape.H,
                       "E": shape.E, "K": shape.K, "I": shape.I, "I_shared": shape.I_sh},
            "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": nthreads, "kind": "oracle",
                             "sample": f"first {n} of the {T} tokens per step, router GEMM included"},
            "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    if dist:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
