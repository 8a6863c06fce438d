"""Host logic of bench.py's multi-rank (replica) path, run as two gloo ranks
on CPU: the job time is the max over ranks and the metric divides it by all
ranks' block forwards."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local = [1200.0, 1500.0][rank]          # per-rank device ms of the timed steps
        job = bench.max_over_ranks(local, world)
        out[rank] = (job, bench.per_block_ms(job, 4, 40, world))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_metric():
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_rank, args=(2, port, out), nprocs=2, join=True)
        res = dict(out)
    assert res[0] == res[1]
    job, value = res[0]
    assert job == 1500.0
    assert value == pytest.approx(1500.0 / (4 * 40 * 2 * 2))


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(123.5, 1) == 123.5
    assert bench.per_block_ms(3200.0, 4, 40, 1) == pytest.approx(10.0)
