"""C-ABI behaviour on the GPU: argument errors, workspace checks, T = 0,
bounded device waits (a withheld operand load makes one block's wait run out;
the status is reported and the workspace stays usable), and the launch
counter."""
import ctypes

import numpy as np
import pytest
import torch

import moe_inputs as mi
import mixture_experts_layer_61_b200 as moe
from helpers import cfg_for, small_shape

pytestmark = pytest.mark.gpu


def _setup(T=40):
    shape = small_shape(H=256, E=8, K=2, I=512)
    w = mi.make_weights(shape, 1, device="cuda")
    x = mi.make_x(shape, T, 1, device="cuda")
    cfg = cfg_for(shape, T)
    return shape, w, x, cfg


def test_bad_arguments():
    shape, w, x, cfg = _setup()
    L = moe.lib()
    ws = moe.alloc_workspace(moe.workspace_size(cfg))
    out = torch.empty_like(x)
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    P = lambda t: ctypes.c_void_p(t.data_ptr())
    for field, bad in [("K", 0), ("K", 17), ("E", 0), ("E", 1025), ("tile_B", 0), ("tile_B", 257),
                       ("dtype", 2), ("score_fn", 2), ("H", 250), ("T", -1)]:
        c = cfg_for(shape, 40)
        setattr(c, field, bad)
        rc = L.moe_layer_forward(ctypes.byref(c), P(x), P(w["w_r"]), P(w["w13"]), P(w["w2"]), None, None, None,
                                 P(out), P(ws), ws.numel(), None, s)
        assert rc == -1, (field, bad, rc)
    rc = L.moe_layer_forward(ctypes.byref(cfg), None, P(w["w_r"]), P(w["w13"]), P(w["w2"]), None, None, None,
                             P(out), P(ws), ws.numel(), None, s)
    assert rc == -1
    rc = L.moe_layer_forward(ctypes.byref(cfg), P(x), P(w["w_r"]), P(w["w13"]), P(w["w2"]), None, None, None,
                             P(out), P(ws), ws.numel() - 1024, None, s)
    assert rc == -2
    assert L.moe_workspace_size(None) == 0
    assert torch.cuda.synchronize() is None


def test_zero_tokens_is_noop():
    shape, w, x, cfg = _setup(T=0)
    ws = moe.alloc_workspace(moe.workspace_size(cfg))
    before = moe.kernel_launch_count()
    out = moe.layer_forward(cfg, x, w["w_r"], w["w13"], w["w2"], ws)
    moe.check_status(ws)
    assert out.shape == (0, 256)
    assert moe.kernel_launch_count() == before


def test_launch_count_of_a_forward():
    shape, w, x, cfg = _setup()
    ws = moe.alloc_workspace(moe.workspace_size(cfg))
    before = moe.kernel_launch_count()
    moe.layer_forward(cfg, x, w["w_r"], w["w13"], w["w2"], ws)
    moe.check_status(ws)
    # decode size: routing (router + top-K + alignment), permute, expert FFN, combine
    assert moe.ffn_fused(cfg)
    assert moe.kernel_launch_count() - before == 4


def test_launch_count_of_a_prefill_forward():
    shape = small_shape(H=256, E=8, K=2, I=512)
    T = 1500
    w = mi.make_weights(shape, 2, device="cuda")
    x = mi.make_x(shape, T, 2, device="cuda")
    cfg = cfg_for(shape, T)
    ws = moe.alloc_workspace(moe.workspace_size(cfg))
    before = moe.kernel_launch_count()
    moe.layer_forward(cfg, x, w["w_r"], w["w13"], w["w2"], ws)
    moe.check_status(ws)
    # routing (router logits on the CUDA cores for this 8 x 256 router matrix,
    # top-K and alignment in one launch), permute, gate/up, down, combine
    assert not moe.ffn_fused(cfg)
    assert moe.kernel_launch_count() - before == 5


def test_launch_count_of_a_prefill_forward_with_a_tensor_core_router():
    shape = small_shape(H=256, E=64, K=4, I=512)
    T = 4000  # 250 rows per expert: the two-launch expert FFN
    w = mi.make_weights(shape, 2, device="cuda")
    x = mi.make_x(shape, T, 2, device="cuda")
    cfg = cfg_for(shape, T)
    ws = moe.alloc_workspace(moe.workspace_size(cfg))
    before = moe.kernel_launch_count()
    moe.layer_forward(cfg, x, w["w_r"], w["w13"], w["w2"], ws)
    moe.check_status(ws)
    # router GEMM, top-K, align, permute, gate/up, down, combine
    assert not moe.ffn_fused(cfg)
    assert moe.kernel_launch_count() - before == 7


def test_wait_timeout_is_reported_and_recoverable():
    shape, w, x, cfg = _setup()
    ws = moe.alloc_workspace(moe.workspace_size(cfg))
    ref = moe.layer_forward(cfg, x, w["w_r"], w["w13"], w["w2"], ws).clone()
    moe.check_status(ws)
    moe.set_wait_limit_ns(20_000_000)  # 20 ms
    try:
        moe.debug_withhold_first_load(True)
        moe.layer_forward(cfg, x, w["w_r"], w["w13"], w["w2"], ws)
        with pytest.raises(moe.MoeError) as e:
            moe.check_status(ws)
        assert e.value.code == -4
    finally:
        moe.debug_withhold_first_load(False)
        moe.set_wait_limit_ns(0)
    out = moe.layer_forward(cfg, x, w["w_r"], w["w13"], w["w2"], ws)
    moe.check_status(ws)
    assert torch.equal(out, ref)


def test_wait_timeout_in_shared_experts_is_reported_and_recoverable():
    # the withheld load lands in the shared FFN, launched first on the side
    # stream: its status word (the header's second) reports the timeout and
    # its own control block is re-zeroed
    shape = small_shape(H=256, E=8, K=2, I=512, I_sh=768)
    T = 40
    w = mi.make_weights(shape, 3, device="cuda")
    x = mi.make_x(shape, T, 3, device="cuda")
    cfg = cfg_for(shape, T)
    ws = moe.alloc_workspace(moe.workspace_size(cfg))
    fwd = lambda: moe.layer_forward(cfg, x, w["w_r"], w["w13"], w["w2"], ws, w["w13_sh"], w["w2_sh"])
    moe.set_shared_sms(16)
    try:
        ref = fwd().clone()
        moe.check_status(ws)
        moe.set_wait_limit_ns(20_000_000)  # 20 ms
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
    finally:
        moe.set_shared_sms(0)
