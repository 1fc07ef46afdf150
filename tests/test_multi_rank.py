"""The N > 1 bench path on CPU: two gloo ranks, each an independent replica.

Checks the pieces that make the multi-GPU number: the max-over-ranks
reduction of the step time (every rank gets the slowest rank's time) and the
whole-job throughput (all ranks' bytes over that time), plus the barrier
the timed region is bracketed by.  No GPU is used."""
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
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        dist.barrier()
        step_ms = 1.5 + rank          # rank 1 is the slow one
        slowest = bench.max_over_ranks(step_ms)
        gbs = bench.job_gbs(world, 10_485_760 * 16, slowest)
        out[rank] = (slowest, gbs)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_replicas_reduce_max_and_aggregate():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
    assert set(out.keys()) == {0, 1}
    for r in range(world):
        slowest, gbs = out[r]
        assert slowest == pytest.approx(2.5)
        assert gbs == pytest.approx(world * 10_485_760 * 16 / 2.5e-3 / 1e9)


def test_single_process_is_identity():
    import bench
    assert not dist.is_initialized()
    assert bench.max_over_ranks(3.25) == 3.25
