"""The allocation-free router GEMM (moe_router_gemm_noalloc), called through
the C-ABI.  It exists for callers that cannot allocate device memory while
they enqueue work (a plugin whose enqueue hook must not allocate, a runtime
that plans all device memory up front): its scratch is a fixed array inside
the library instead of a caller workspace.  Its logits must match the
workspace entry point's and the oracle's, call after call, since every call
reuses the same array; a device wait that runs out is reported by
moe_router_gemm_noalloc_status.  This file is collected last so that a
failure here comes after every other test has run."""
import ctypes

import numpy as np
import pytest
import torch

import moe_inputs as mi
import mixture_experts_layer_61_b200 as moe
import oracle
from helpers import host, small_shape

pytestmark = pytest.mark.gpu


def _entry():
    f = moe.lib().moe_router_gemm_noalloc
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.POINTER(moe.MoeConfig), ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    return f


def _status():
    f = moe.lib().moe_router_gemm_noalloc_status
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p]
    return f(ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _call(cfg, x, w_r):
    out = torch.full((cfg.T, cfg.E), float("nan"), dtype=torch.float32, device="cuda")
    rc = _entry()(ctypes.byref(cfg), ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(w_r.data_ptr()),
                  ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0
    return out


@pytest.mark.parametrize("T,H,E,dtype", [(1, 4096, 8, "bf16"), (32, 7168, 256, "bf16"), (17, 3584, 64, "bf16"),
                                         (8, 256, 8, "fp32"), (5, 264, 130, "bf16")])
def test_noalloc_router_matches_workspace_router_twice(T, H, E, dtype):
    shape = small_shape(H, E, 2, 64, dtype=dtype)
    w = mi.make_weights(shape, seed=T + E, device="cuda", experts=False)
    x = mi.make_x(shape, T, seed=T, device="cuda")
    cfg = moe.config(T, H, E, 2, 64, dtype=moe.BF16 if dtype == "bf16" else moe.FP32)
    ws = moe.alloc_workspace(moe.gemm_workspace_size())
    ref = moe.router_gemm(cfg, x, w["w_r"], ws)
    moe.check_status(ws)
    ref = ref.cpu().numpy().astype(np.float64)
    f = _entry()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    tol = 1e-5 if dtype == "bf16" else 4e-3   # the router tests' bounds
    for _ in range(2):
        out = torch.full((T, E), float("nan"), dtype=torch.float32, device="cuda")
        rc = f(ctypes.byref(cfg), ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(w["w_r"].data_ptr()),
               ctypes.c_void_p(out.data_ptr()), stream)
        assert rc == 0
        torch.cuda.synchronize()
        got = out.cpu().numpy().astype(np.float64)
        assert np.isfinite(got).all()
        assert np.abs(got - ref).max() / np.abs(ref).max() <= tol


def test_noalloc_router_rejects_more_tokens_than_its_scratch_holds():
    cfg = moe.config(33, 256, 8, 2, 64)
    x = torch.zeros((33, 256), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((8, 256), dtype=torch.bfloat16, device="cuda")
    out = torch.empty((33, 8), dtype=torch.float32, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = _entry()(ctypes.byref(cfg), ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(w.data_ptr()),
                  ctypes.c_void_p(out.data_ptr()), stream)
    assert rc == -1


def _router_case(T, H, E, seed):
    shape = small_shape(H, E, 2, 64)
    w = mi.make_weights(shape, seed=seed, device="cuda", experts=False)
    x = mi.make_x(shape, T, seed=seed + 1, device="cuda")
    cfg = moe.config(T, H, E, 2, 64)
    return cfg, x, w["w_r"], oracle.router_logits(host(x), host(w["w_r"]))


def test_noalloc_router_matches_the_oracle_across_shapes_on_one_stream():
    # a large router (two stream-K split feature tiles) then a small one on the
    # same stream: the second call sees the shared array's counters cleared
    for T, H, E in [(32, 7168, 256), (1, 4096, 8), (17, 3584, 64)]:
        cfg, x, w_r, ref = _router_case(T, H, E, seed=T + E)
        got = _call(cfg, x, w_r)
        assert _status() == 0
        g = got.cpu().numpy().astype(np.float64)
        assert np.isfinite(g).all()
        assert np.abs(g - ref).max() / np.abs(ref).max() <= 1e-5


def test_noalloc_router_timeout_is_reported_and_cleared():
    # one withheld operand load makes block 0's waits run out (20 ms limit):
    # the status call reports it once, clears the array's control words, and
    # the next call is exact again
    cfg, x, w_r, ref = _router_case(8, 7168, 256, seed=5)
    moe.set_wait_limit_ns(20_000_000)
    try:
        moe.debug_withhold_first_load(True)
        _call(cfg, x, w_r)
        assert _status() == -4
        assert _status() == 0
    finally:
        moe.debug_withhold_first_load(False)
        moe.set_wait_limit_ns(0)
    got = _call(cfg, x, w_r).cpu().numpy().astype(np.float64)
    assert _status() == 0
    assert np.abs(got - ref).max() / np.abs(ref).max() <= 1e-5
