"""The multi-rank host logic of bench.py, on CPU with gloo and two ranks:
timings are reduced to the slowest rank, the job value sums all ranks' work,
and the reference arm runs on rank 0 only."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        mine = [1.0 + rank, 5.0 - rank, 0.25 * (rank + 1)]
        got = bench.max_over_ranks(mine, torch.device("cpu"), world)
        assert bench.dist_env() == (rank, world, rank)
        class A:  # the reference arm's arguments
            workload, keep, heads, cpu_rows, warmup, steps, gpus = "tiny", None, None, 64, 0, 1, world
        ref = bench.run_reference(A, rank, world)
        dist.barrier()
        out[rank] = (got, ref is None)
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_reference_on_rank0_only():
    port = _free_port()
    manager = mp.get_context("spawn").Manager()  # no fork of this multi-threaded process
    out = manager.dict()
    mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
    for rank in (0, 1):
        got, ref_none = out[rank]
        assert got == [2.0, 5.0, 0.5]
        assert ref_none == (rank == 1)


def test_job_throughput_sums_ranks_over_slowest():
    import bench
    assert bench.job_throughput(2e12, 4, 1000.0) == pytest.approx(8.0)
    assert bench.job_throughput(3e12, 1, 500.0) == pytest.approx(6.0)
