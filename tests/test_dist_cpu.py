"""bench.py's multi-process plumbing on CPU: two ranks over gloo (127.0.0.1).

Every rank runs its own problem (weak scaling, no data-path collective); the job
time is the slowest rank's, taken with an all-reduce(max), and only rank 0 runs
the CPU reference arm and prints."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    r, w, local = bench.dist_setup(world)
    try:
        assert (r, w, local) == (rank, world, rank)
        bench.barrier(w)
        slowest = bench.max_over_ranks(10.0 + 5.0 * rank, w)
        ref = bench.run_reference(type("A", (), {"workload": "dense31b_m8192", "seed": 0, "warmup": 0,
                                                 "steps": 0})(), r, w) if r != 0 else "rank0-skipped"
        results[rank] = (slowest, ref)
    finally:
        torch.distributed.destroy_process_group()


@pytest.mark.timeout(300)
def test_two_ranks_max_time_and_rank0_reference():
    world = 2
    port = _free_port()
    manager = mp.Manager()
    results = manager.dict()
    mp.start_processes(_worker, args=(world, port, results), nprocs=world, start_method="spawn", join=True)
    assert results[0][0] == 15.0 and results[1][0] == 15.0   # both ranks see the slowest time
    assert results[1][1] is None                              # the reference arm runs on rank 0 only


def test_weak_scaling_throughput():
    import bench
    flops = 2.0 * 8192 * 21504 * 5376 * 2
    one = bench.job_throughput(1, 20, flops, 40.0)
    two = bench.job_throughput(2, 20, flops, 40.0)
    assert two == pytest.approx(2 * one)                       # units of all ranks / max time
    assert bench.job_throughput(1, 10, flops, 10.0) == pytest.approx(flops * 1000 / 1e12)
