"""The multi-GPU path of bench.py is data-parallel replicas with no collective
on the data path; its only cross-rank steps are the barrier and the MAX
reduction of the device-timed totals.  Checked here with world-size-2 gloo
ranks on the CPU."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, totals, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        dist.barrier()
        m = bench.max_over_ranks(totals[rank], dist, torch.device("cpu"))
        out[rank] = (m, bench.replica_tokens_per_s(world, 2048, 20, m))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_throughput_gloo():
    world = 2
    totals = [25.0, 31.5]   # ms of K = 20 steps on each rank
    mgr = mp.get_context("spawn").Manager()  # no fork of this multi-threaded process
    out = mgr.dict()
    mp.spawn(_rank, args=(world, _free_port(), totals, out), nprocs=world, join=True)
    for r in range(world):
        m, v = out[r]
        assert m == 31.5                         # every rank sees the slowest rank's time
        assert v == pytest.approx(2 * 2048 * 20 / 0.0315)


def test_single_rank_is_identity():
    assert bench.max_over_ranks(12.5, None, torch.device("cpu")) == 12.5
    assert bench.replica_tokens_per_s(1, 100, 10, 1000.0) == pytest.approx(1000.0)


def test_tp_throughput_counts_the_shared_tokens_once():
    # under TP every rank works on the same T tokens: the job's rate is T per
    # step over the slowest rank's time, whatever the number of ranks
    assert bench.tp_tokens_per_s(32, 10, 5.0) == pytest.approx(32 * 10 / 0.005)
