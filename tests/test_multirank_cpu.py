"""The multi-GPU path of bench.py is replicas only: every rank runs its own
cache on its own GPU, and the only collectives are the barrier and the
max-over-ranks timing.  These run that plumbing with world size 2 on the
gloo backend (CPU, no GPU), as separate processes."""
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    import bench
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world,
                                         timeout=datetime.timedelta(seconds=60))
    try:
        torch.distributed.barrier()
        elapsed = 10.0 + 5.0 * rank            # the ranks' own device times (ms)
        slowest = bench.max_over_ranks(elapsed, world, torch, "cpu")
        value = bench.replica_throughput(64, 100, world, slowest)
        # the reference arm under torchrun: rank 0 alone works, others return
        class A:
            gpus, steps, warmup = world, 1, 0
        ref = bench.run_reference(A(), bench.WORKLOADS["cr88"], rank, world) if rank != 0 else None
        out[rank] = (slowest, value, ref)
        torch.distributed.barrier()
    finally:
        torch.distributed.destroy_process_group()


def test_replicas_take_the_slowest_rank_time_world2():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
    for r in range(world):
        slowest, value, ref = out[r]
        assert slowest == 15.0
        assert value == pytest.approx(64 * 100 * world / 0.015)
        assert ref is None


def test_single_rank_needs_no_collective():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(12.5, 1, torch, "cpu") == 12.5
    assert bench.replica_throughput(64, 10, 1, 2.0) == pytest.approx(320000.0)
