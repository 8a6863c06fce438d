"""Head-parallel (Ulysses) block on the GPU, through the C ABI.

- wan_permute_chunks against the host permutation, for the four layout
  changes of the exchange and ragged chunk sizes.
- The phases with one shard (N = 1: wan_block_sp_qkv, wan_attention on all
  heads, wan_block_sp_finish) against the fp64 oracle: fp32 max-abs <= 1e-4,
  bf16 relative L2 <= 2e-2 on the output and on the block delta.
- N = 2 and 4 ranks emulated in one process (each rank's phases in turn; the
  all-to-all as copies between the ranks' buffers; no kernel of one rank
  waits on another's): the union of the ranks' x equals the N = 1 run bit
  for bit, over whole denoising steps.
- Two processes on one GPU, exchanging over gloo (staged through host
  memory): the same equality through torch.distributed.
"""
import dataclasses
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import wan_oracle as O
from video_diffusion_transformer_fwd_b200 import configs, synth, wan
from video_diffusion_transformer_fwd_b200.configs import BlockConfig
from video_diffusion_transformer_fwd_b200.step import UlyssesStep, permute_chunks_device

from parity_util import BF16_REL_L2, F32_MAX_ABS, Guarded, np64, rel_l2, weights64
from test_ulysses import permute_chunks_host

pytestmark = pytest.mark.gpu

TINY = dataclasses.replace(configs.get("tiny"), batch=2, blocks=2)
SMALL_BF16 = BlockConfig("ulysses-bf16", 2, 4, 8, 512, 4, 1024, 24, "bf16", batch=2, blocks=2)


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    wan.load()


@pytest.mark.parametrize("dims,perm,chunk", [
    ((2, 7, 3, 4), (3, 0, 1, 2), 256),         # pack q|k|v
    ((4, 2, 7, 3), (3, 1, 0, 2), 256),         # unpack q|k|v
    ((2, 4, 7), (1, 0, 2), 2560),              # pack o
    ((4, 2, 7), (1, 2, 0), 16),                # unpack o
    ((3, 5, 2, 2, 3), (4, 2, 0, 3, 1), 48),
    ((1000,), (0,), 64),
])
def test_permute_chunks_matches_host(dims, perm, chunk):
    n = int(np.prod(dims)) * chunk // 2
    src = torch.randn(n, device="cuda").to(torch.bfloat16)
    gdst = Guarded((n,), torch.bfloat16)
    permute_chunks_device(src, gdst.t, dims, perm, chunk)
    torch.cuda.synchronize()
    gdst.check("permute dst")
    ref = torch.empty_like(src)
    permute_chunks_host(src, ref, dims, perm, chunk)
    assert torch.equal(gdst.t, ref)


def _no_exchange(send, recv, group):
    recv.copy_(send)


def _oracle_step(cfg, st_ref):
    """The fp64 oracle's denoising step on the same inputs and weights."""
    w = [weights64(w) for w in st_ref.weights]
    acts = synth.block_activations(2, cfg.L, cfg.dim, cfg.text_len, cfg.dtype, "cuda", 100, same_e0=True)
    x0 = np64(acts["x"][0])
    ctx = np64(acts["ctx"])
    return x0, O.denoise_step(x0, ctx[0], ctx[1], None, np64(acts["e0"][0]), w, cfg.heads, (cfg.F, cfg.H, cfg.W),
                              cfg.eps, cfg.guide_scale, cfg.sigma, cfg.sigma_next, cfg.theta)


@pytest.mark.parametrize("cfg", [TINY, SMALL_BF16], ids=["tiny-f32", "small-bf16"])
def test_one_shard_phases_match_oracle(cfg):
    st = UlyssesStep(cfg, 0, 1, seed=0, device="cuda", exchange=_no_exchange)
    st.step()
    torch.cuda.synchronize()
    assert wan.device_status() == wan.WAN_OK
    x0, ref = _oracle_step(cfg, st)
    got = np64(st.x)
    if cfg.dtype == "f32":
        assert np.abs(got - ref).max() <= F32_MAX_ABS
    else:
        assert rel_l2(got, ref) <= BF16_REL_L2
        assert rel_l2(got - x0, ref - x0) <= BF16_REL_L2


def _emulated_step(ranks):
    """One denoising step of N ranks in this process: the phases of each
    rank in turn, the all-to-alls as copies between the ranks' buffers."""
    N = len(ranks)
    for r in ranks:
        r.xb[0].copy_(r.x)
        r.xb[1].copy_(r.x)
    for i in range(len(ranks[0].cweights)):
        for r in ranks:
            r.block_qkv(i)
            r.ex.pack_qkv()
        for r in range(N):
            for j in range(N):
                ranks[r].ex.recv_qkv[j].copy_(ranks[j].ex.send_qkv[r])
        for r in ranks:
            r.ex.unpack_qkv()
            r.block_attention()
            r.ex.pack_o()
        for r in range(N):
            for j in range(N):
                ranks[r].ex.recv_o[j].copy_(ranks[j].ex.send_o[r])
        for r in ranks:
            r.ex.unpack_o()
            r.block_finish(i)
    for r in ranks:
        r.euler()


@pytest.mark.parametrize("cfg", [TINY, SMALL_BF16], ids=["tiny-f32", "small-bf16"])
@pytest.mark.parametrize("N", [2, 4])
def test_sharded_step_equals_one_shard(cfg, N):
    ref = UlyssesStep(cfg, 0, 1, seed=0, device="cuda", exchange=_no_exchange)
    ranks = [UlyssesStep(cfg, r, N, seed=0, device="cuda", exchange=_no_exchange) for r in range(N)]
    for _ in range(2):
        ref.step()
        _emulated_step(ranks)
    torch.cuda.synchronize()
    assert wan.device_status() == wan.WAN_OK
    got = torch.cat([r.x for r in ranks])
    assert torch.isfinite(ref.x).all()
    assert torch.equal(got, ref.x)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _gpu_rank(rank, world, port, cfg, steps, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        st = UlyssesStep(cfg, rank, world, group=dist.group.WORLD, seed=0, device="cuda:0")
        for _ in range(steps):
            st.step()
        torch.cuda.synchronize()
        assert wan.device_status() == wan.WAN_OK, wan.last_error()
        out[rank] = st.x.cpu().numpy()
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("cfg", [TINY, SMALL_BF16], ids=["tiny-f32", "small-bf16"])
def test_two_processes_equal_one_shard(cfg):
    steps = 2
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_gpu_rank, args=(2, port, cfg, steps, out), nprocs=2, join=True)
        res = dict(out)
    ref = UlyssesStep(cfg, 0, 1, seed=0, device="cuda:0", exchange=_no_exchange)
    for _ in range(steps):
        ref.step()
    torch.cuda.synchronize()
    np.testing.assert_array_equal(np.concatenate([res[0], res[1]]), ref.x.cpu().numpy())
