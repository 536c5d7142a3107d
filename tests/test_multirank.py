"""The benchmark's multi-rank host path on CPU: two gloo ranks, each timing
its own batch (weak scaling, no data exchange); the job's time is the
slowest rank's and the job's bytes are every rank's."""

import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import workloads as W


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, times, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        m = bench.max_over_ranks(times[rank], world, torch.device("cpu"))
        value = bench.weak_scaling_gbs(1_000_000_000, world, m)
        # every rank routes its own seeded batch
        idx = W.make_inputs("tiny", seed=rank)["topk_idx"]
        gathered = [None] * world
        dist.all_gather_object(gathered, idx.tobytes())
        out[rank] = (m, value, len(set(gathered)))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time_and_sum_the_bytes():
    world, times = 2, [3.0, 5.0]
    manager = mp.get_context("spawn").Manager()
    out = manager.dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), times, out), nprocs=world,
                       join=True, start_method="spawn")
    for rank in range(world):
        m, value, distinct = out[rank]
        assert m == 5.0
        assert np.isclose(value, 2 * 1.0 / 5e-3)   # 2 ranks x 1 GB per 5 ms step
        assert distinct == world                    # different batches per rank


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(4.5, 1, torch.device("cpu")) == 4.5
    assert np.isclose(bench.weak_scaling_gbs(2_000_000_000, 1, 1.0), 2000.0)
