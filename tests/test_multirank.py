"""The benchmark's multi-rank logic on two CPU processes (gloo): every rank runs its own
problem (weak scaling, no data-path collective), the job time is the largest rank time,
and the job throughput counts every rank's work over that time."""
import datetime
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        spec = bench.rank_spec("tiny_t2k_g1_k8", rank)
        local_ms = 10.0 + 5.0 * rank            # rank 1 is the slow one
        job_ms = bench.max_over_ranks(local_ms, dist, torch.device("cpu"))
        tflops = bench.job_tflops(world, 2.0e12, 4, job_ms)
        out[rank] = (spec["seed"], spec["hq"], job_ms, tflops)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_weak_scaling_gloo():
    world, port = 2, _free_port()
    # the manager process is spawned, not forked: the test process already runs threads
    with mp.get_context("spawn").Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        r = dict(out)
    assert sorted(r) == [0, 1]
    assert r[0][0] != r[1][0] and r[0][1] == r[1][1]      # own seed, same shapes
    assert r[0][2] == r[1][2] == 15.0                      # the slowest rank's time
    assert r[0][3] == r[1][3] == pytest.approx(world * 2.0e12 * 4 / 15.0e-3 / 1e12)


def test_single_process_passes_through():
    import bench
    assert bench.max_over_ranks(7.5, None, torch.device("cpu")) == 7.5
    assert bench.job_tflops(1, 1.0e12, 10, 1000.0) == pytest.approx(10.0)
