"""The N > 1 bench path on the CPU: two gloo ranks, each with its own
device-time measurement; every rank must end with the max over ranks and
the whole-job throughput computed from it (weak scaling: the units of all
ranks over the slowest rank's time)."""
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
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        mine = [10.0, 12.5][rank]
        max_ms, tflops = bench.aggregate(mine, steps=100, flops_per_step=1e12, world=world)
        out[rank] = (max_ms, tflops)
    finally:
        dist.destroy_process_group()


def test_two_rank_aggregation_takes_the_max():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    for r in range(2):
        max_ms, tflops = out[r]
        assert max_ms == 12.5
        # 2 ranks x 100 steps x 1 TFLOP in 12.5 ms
        assert tflops == pytest.approx(2 * 100 * 1.0 / 12.5e-3)


def test_single_rank_aggregation_is_identity():
    import bench
    assert bench.aggregate(4.0, 10, 2e12, 1) == (4.0, pytest.approx(2e12 * 10 / 4e-3 / 1e12))
