"""TP over the expert intermediate dimension I: the host side (per-rank
configuration, the collective step) checked with gloo ranks on the CPU.

Every rank routes the same tokens identically and holds a slice of every
expert; the oracle stands in for the kernels (it computes each rank's partial
output from its slice), the package's tp_allreduce sums them across the ranks,
and the sum must equal the oracle's unsplit layer."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import mixture_experts_layer_61_b200 as moe
import oracle


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _layer(seed):
    rng = np.random.default_rng(seed)
    T, H, E, K, I, I_sh = 7, 32, 6, 2, 48, 24
    x = rng.standard_normal((T, H)).astype(np.float32)
    w_r = (rng.standard_normal((E, H)) / np.sqrt(H)).astype(np.float32)
    w13 = (rng.standard_normal((E, 2 * I, H)) / np.sqrt(H)).astype(np.float32)
    w2 = (rng.standard_normal((E, H, I)) / np.sqrt(I)).astype(np.float32)
    w13_sh = (rng.standard_normal((2 * I_sh, H)) / np.sqrt(H)).astype(np.float32)
    w2_sh = (rng.standard_normal((H, I_sh)) / np.sqrt(I_sh)).astype(np.float32)
    return x, w_r, w13, w2, w13_sh, w2_sh, K


def _rank(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        x, w_r, w13, w2, w13_sh, w2_sh, K = _layer(5)  # the same seed on every rank: replicated inputs
        a13, a2 = oracle.tp_shard(w13, w2, rank, world)
        s13, s2 = oracle.tp_shard(w13_sh, w2_sh, rank, world)
        mine = oracle.moe_layer(x, w_r, a13, a2, K, w13_sh=s13, w2_sh=s2, nthreads=1)
        part = torch.from_numpy(mine.copy())
        moe.tp_allreduce(part)
        out[rank] = (mine, part.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_tp_allreduce_of_rank_partials_is_the_whole_layer_gloo(world):
    mgr = mp.get_context("spawn").Manager()  # no fork of this multi-threaded process
    out = mgr.dict()
    mp.spawn(_rank, args=(world, _free_port(), out), nprocs=world, join=True)
    x, w_r, w13, w2, w13_sh, w2_sh, K = _layer(5)
    full = oracle.moe_layer(x, w_r, w13, w2, K, w13_sh=w13_sh, w2_sh=w2_sh)
    tol = 1e-12 * np.abs(full).max()
    for r in range(world):
        mine, summed = out[r]
        assert np.abs(mine - full).max() > 1e-3 * np.abs(full).max()  # one slice is not the layer
        assert np.allclose(summed, full, rtol=1e-12, atol=tol)        # every rank holds the sum
    assert all(np.array_equal(out[0][1], out[r][1]) for r in range(world))


def test_tp_allreduce_without_a_group_is_identity():
    p = torch.arange(8, dtype=torch.float32)
    assert moe.tp_allreduce(p.clone()).equal(p)


def test_tp_config_splits_I_and_the_shared_width():
    c = moe.config(32, 3584, 64, 8, 2560, n_shared=8, I_shared=2560)
    t = moe.tp_config(c, 8)
    assert (t.T, t.H, t.E, t.K, t.I) == (32, 3584, 64, 8, 320)
    assert t.n_shared * t.I_shared == 8 * 2560 // 8
    d = moe.tp_config(moe.config(4, 7168, 256, 8, 2048, n_shared=1, I_shared=2048), 4)
    assert (d.I, d.n_shared, d.I_shared) == (512, 1, 512)
    assert moe.tp_config(moe.config(4, 4096, 8, 2, 14336), 8).n_shared == 0
    with pytest.raises(ValueError):
        moe.tp_config(moe.config(4, 4096, 8, 2, 14336), 5)


def _rank_overlapped(rank, world, port, n_chunks, out):
    # the overlap protocol: each block of H / n_chunks output features is
    # produced, its all-reduce started asynchronously, the next block produced
    # beside it; the blocks side by side after all waits are the whole layer
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        x, w_r, w13, w2, w13_sh, w2_sh, K = _layer(5)
        a13, a2 = oracle.tp_shard(w13, w2, rank, world)
        s13, s2 = oracle.tp_shard(w13_sh, w2_sh, rank, world)
        mine = oracle.moe_layer(x, w_r, a13, a2, K, w13_sh=s13, w2_sh=s2, nthreads=1)
        Hc = mine.shape[1] // n_chunks
        parts = [torch.empty((mine.shape[0], Hc), dtype=torch.float64) for _ in range(n_chunks)]
        order = []

        def produce(c):
            order.append(c)
            parts[c].copy_(torch.from_numpy(np.ascontiguousarray(mine[:, c * Hc:(c + 1) * Hc])))

        moe.tp_overlapped_allreduce(parts, produce)
        out[rank] = (order, torch.cat(parts, dim=1).numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,n_chunks", [(2, 2), (2, 4), (4, 4)])
def test_tp_overlapped_allreduce_protocol_gloo(world, n_chunks):
    mgr = mp.get_context("spawn").Manager()  # no fork of this multi-threaded process
    out = mgr.dict()
    mp.spawn(_rank_overlapped, args=(world, _free_port(), n_chunks, out), nprocs=world, join=True)
    x, w_r, w13, w2, w13_sh, w2_sh, K = _layer(5)
    full = oracle.moe_layer(x, w_r, w13, w2, K, w13_sh=w13_sh, w2_sh=w2_sh)
    for r in range(world):
        order, got = out[r]
        assert order == list(range(n_chunks))
        assert np.allclose(got, full, rtol=1e-10, atol=1e-10)
