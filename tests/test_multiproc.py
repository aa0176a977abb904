"""The multi-rank host path of bench.py on CPU: two gloo ranks.

Each rank runs its own replica of the workload (channels are independent, so
no collective touches the data); the only collectives are barriers and the
max-over-ranks of the measured time, which these tests exercise with gloo.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from selective_state_space_mss_b200 import inputs as gen


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, times, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        dist.barrier()
        ms_max = bench.max_over_ranks(times[rank], world, torch.device("cpu"))
        rate = bench.whole_job_rate(1000, world, 10, ms_max)
        seed = bench.rank_seed(1003, rank)
        # the replica's inputs: generated from the rank's own seed
        inp = gen.scan_inputs(1, 4, 16, 8, "bf16", seed, "normal")
        digest = int(inp["u"].stored.astype("int64").sum())
        out[rank] = (ms_max, rate, seed, digest)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_time_and_replicas():
    world, port = 2, _free_port()
    times = [12.5, 20.0]
    manager = mp.get_context("spawn").Manager()
    out = manager.dict()
    mp.start_processes(_worker, args=(world, port, times, out), nprocs=world, start_method="spawn", join=True)
    res = [out[r] for r in range(world)]
    # every rank sees the slowest rank's time
    assert all(r[0] == max(times) for r in res)
    # whole-job throughput: all ranks' units over the slowest time
    assert all(r[1] == pytest.approx(world * 1000 * 10 / (max(times) * 1e-3)) for r in res)
    # distinct replicas
    assert res[0][2] != res[1][2] and res[0][3] != res[1][3]


def test_single_rank_helpers():
    assert bench.max_over_ranks(3.5, 1, torch.device("cpu")) == 3.5
    assert bench.whole_job_rate(10, 1, 2, 1000.0) == pytest.approx(20.0)
