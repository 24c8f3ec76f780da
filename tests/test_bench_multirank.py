"""The multi-rank plumbing of bench.py on CPU: two gloo ranks, timing
aggregated as the max over ranks, whole-job weak-scaling value."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import torch.distributed as dist

    import bench

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = 10.0 + 5.0 * rank  # rank 1 is the slow one
        out[rank] = bench.max_over_ranks(mine)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert out[0] == out[1] == 15.0


def test_max_over_ranks_without_group():
    import bench

    assert bench.max_over_ranks(3.25) == 3.25


def test_weak_scaling_value():
    import bench

    # 2 ranks, 1e12 FLOP each per step, slowest step 2 ms -> 1000 TFLOP/s whole job.
    assert bench.weak_scaling_value(2, 1e12, 2.0) == pytest.approx(1000.0)
    assert bench.weak_scaling_value(1, 3.5e11, 1.0) == pytest.approx(350.0)
