"""The bench's multi-rank host logic on CPU: two gloo ranks check the
max-over-ranks timing reduction and the whole-job aggregate (every rank's
work over the slowest rank's time), as bench.py uses them under torchrun."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r, w, local = bench.dist_env()
        assert (r, w, local) == (rank, world, rank)
        ms = 10.0 + 5.0 * rank                     # rank 1 is the slowest
        worst = bench.max_over_ranks(ms, world)
        value = bench.aggregate_value(1e12, 4, world, worst / 1e3)
        dist.barrier()
        out[rank] = (worst, value)
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_gloo_ranks_max_and_aggregate():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(90)
        assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
        res = dict(out)
    for r in range(world):
        worst, value = res[r]
        assert worst == 15.0
        # 2 ranks x 4 steps x 1 TFLOP over the slowest rank's 15 ms
        assert abs(value - 2 * 4 * 1.0 / 0.015) < 1e-9


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.aggregate_value(2e12, 10, 1, 2.0) == 10.0
