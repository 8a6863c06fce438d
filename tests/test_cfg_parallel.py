"""The CFG-parallel denoising step (step.CFGParallelStep): the conditional and
unconditional branches of one step on two ranks, their block outputs
exchanged within the pair, each rank updating its own copy of x.

CPU tests (gloo, two ranks): the rank pairing and the order of the exchange.
GPU test: two processes on one GPU exchanging over gloo (no kernel of one
rank waits on the other's; the exchange is a host collective) run whole
steps through the library; both copies of x must equal the batched step's
(DenoiseStep, both branches as B = 2) bit for bit, since no kernel mixes
sequences of a batch.
"""
import dataclasses
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from video_diffusion_transformer_fwd_b200.configs import BlockConfig, get
from video_diffusion_transformer_fwd_b200.step import cfg_exchange, cfg_pairs


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_cfg_pairs():
    assert cfg_pairs(2) == [[0, 1]]
    assert cfg_pairs(8) == [[0, 1], [2, 3], [4, 5], [6, 7]]
    for bad in (0, 1, 3, 5):
        with pytest.raises(ValueError):
            cfg_pairs(bad)


def _exchange_rank(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        groups = [dist.new_group(pr) for pr in cfg_pairs(world)]
        L, D = 5, 3
        local = torch.full((1, L, D), 10.0 * rank) + torch.arange(L * D, dtype=torch.float32).view(1, L, D)
        gathered = torch.empty((2, L, D))
        cfg_exchange(local, gathered, groups[rank // 2])
        out[rank] = gathered.numpy().copy()
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_cfg_exchange_order_four_ranks():
    """Ranks 2p / 2p+1 receive [conditional, unconditional] of their own pair."""
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_exchange_rank, args=(4, port, out), nprocs=4, join=True)
        res = dict(out)
    base = np.arange(15, dtype=np.float32).reshape(5, 3)
    for r in range(4):
        p = r // 2
        np.testing.assert_array_equal(res[r][0], base + 10.0 * (2 * p))
        np.testing.assert_array_equal(res[r][1], base + 10.0 * (2 * p + 1))


SMALL_BF16 = BlockConfig("cfg-parallel-bf16", 2, 8, 8, 256, 2, 512, 64, "bf16", batch=2, blocks=2)


def _gpu_rank(rank, world, port, cfg, steps, out):
    from video_diffusion_transformer_fwd_b200 import wan
    from video_diffusion_transformer_fwd_b200.step import CFGParallelStep
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        groups = [dist.new_group(pr) for pr in cfg_pairs(world)]
        st = CFGParallelStep(cfg, rank % 2, groups[rank // 2], seed=0, device="cuda:0")
        for _ in range(steps):
            st.step()
        torch.cuda.synchronize()
        assert wan.device_status() == wan.WAN_OK, wan.last_error()
        out[rank] = st.x.cpu().numpy()
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.gpu
@pytest.mark.parametrize("cfg", [dataclasses.replace(get("tiny"), batch=2, blocks=3), SMALL_BF16],
                         ids=["tiny-f32", "small-bf16"])
def test_cfg_parallel_step_equals_batched_step(cfg):
    from video_diffusion_transformer_fwd_b200.step import DenoiseStep
    steps = 2
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_gpu_rank, args=(2, port, cfg, steps, out), nprocs=2, join=True)
        res = dict(out)
    ref = DenoiseStep(cfg, seed=0, device="cuda:0")
    for _ in range(steps):
        ref.step()
    torch.cuda.synchronize()
    x_ref = ref.x.cpu().numpy()
    assert np.isfinite(x_ref).all()
    np.testing.assert_array_equal(res[0], res[1])
    np.testing.assert_array_equal(res[0], x_ref)
