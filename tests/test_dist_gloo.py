"""Host logic of the multi-GPU bench path, run as 2 gloo ranks on CPU.

Each rank runs its own replica of the workload (weak scaling, no data-path
collective).  Checked here: the barrier, the max-over-ranks of the step time
and the whole-job throughput formula, with ranks that report different times.
"""
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


def _worker(rank, world, port, q):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.barrier(world, device="cpu")
        my_ms = 10.0 + 5.0 * rank            # rank 1 is the slower one
        m = bench.max_over_ranks(my_ms, world, device="cpu")
        v = bench.weak_scaling_value(65536, world, m)
        q.put((rank, m, v))
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_reduction():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, m, v in res:
        assert m == 15.0                      # max over ranks, seen by every rank
        assert v == pytest.approx(2 * 65536 / 0.015)


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.weak_scaling_value(100, 1, 1000.0) == pytest.approx(100.0)
