"""Multi-process host logic of bench.py on CPU (gloo, world_size 2).

The forward has no cross-GPU exchange; bench.py only synchronises ranks and
takes the max of their timed regions.  These tests run that logic as two
spawned processes over the gloo backend (no GPU).
"""
import multiprocessing as mp
import os
import socket

import pytest


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        t = bench._max_over_ranks(1.5 + rank, world, torch.device("cpu"))
        bench._barrier(world)
        ref = bench.run_reference(None, rank, world) if rank != 0 else "rank0"
        q.put((rank, t, ref))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_max_over_ranks_and_barrier_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=90) for _ in procs)
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    # both ranks see the slowest rank's time
    assert [o[1] for o in out] == [2.5, 2.5]
    # the reference (oracle) arm runs on rank 0 only; other ranks return nothing
    assert out[1][2] is None


def test_weak_scaling_throughput():
    import bench
    one = bench._throughput(1, 10, 1.0)
    assert one == 10 * bench.TOKENS_PER_STEP
    assert bench._throughput(8, 10, 1.0) == 8 * one
