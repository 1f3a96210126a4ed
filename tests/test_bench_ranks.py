"""The multi-rank logic of bench.py on CPU: two gloo ranks (world size 2), each a replica with its
own step time; the job's time is the slowest rank's and its throughput counts both replicas."""
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


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = 3.0 + 2.0 * rank  # rank 1 is the slow replica
        slowest = bench.max_over_ranks(ms, True, "cpu")
        out[rank] = (slowest, bench.job_tflops(world, 1e12, slowest))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time_and_sum_the_work():
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    for r in range(2):
        slowest, tflops = out[r]
        assert slowest == pytest.approx(5.0)
        assert tflops == pytest.approx(2 * 1e12 / 5e-3 / 1e12)


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(4.5, False, "cpu") == 4.5
    assert bench.job_tflops(1, 2e12, 2.0) == pytest.approx(1000.0)
