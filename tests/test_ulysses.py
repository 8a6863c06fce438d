"""Head-parallel (Ulysses) attention: the layout contract of the all-to-alls
(step.UlyssesExchange) and the argument checks of its C entry points.

The exchange-order tests run on CPU with gloo ranks (2 and 4): every rank
starts from its token shard of a full q|k|v tensor whose values encode
(sequence, token, q/k/v, head, channel); after the first all-to-all rank r
must hold exactly heads [r n/N, (r + 1) n/N) of every token in order, and
after the second one all heads of its own tokens. The pack / unpack layout
changes run here as a host permutation with the same (dims, perm) arguments
that the device path passes to wan_permute_chunks (whose kernel the GPU
tests check against that permutation)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from video_diffusion_transformer_fwd_b200 import build_lib, wan
from video_diffusion_transformer_fwd_b200.step import UlyssesExchange


def permute_chunks_host(src, dst, dims, perm, chunk_bytes, stream=None):
    """Host reference of wan_permute_chunks: chunk axes of src permuted."""
    es = src.element_size()
    c = chunk_bytes // es
    v = src.reshape(*dims, c).permute(*perm, len(dims))
    dst.copy_(v.reshape(dst.shape))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _full_qkv(B, L, heads, d):
    """Value = b * 1e6 + token * 1e3 + s * 100 + head * 10 + channel % 10 (exact in fp32)."""
    b = torch.arange(B).view(B, 1, 1, 1, 1)
    t = torch.arange(L).view(1, L, 1, 1, 1)
    s = torch.arange(3).view(1, 1, 3, 1, 1)
    h = torch.arange(heads).view(1, 1, 1, heads, 1)
    c = torch.arange(d).view(1, 1, 1, 1, d) % 10
    return (b * 1e6 + t * 1e3 + s * 100 + h * 10 + c).float()


def _rank(rank, world, port, B, L, heads, d, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        N = world
        ex = UlyssesExchange(B, L, N, heads, d, torch.float32, group=dist.group.WORLD, device="cpu",
                             permute=permute_chunks_host)
        rows, hl = L // N, heads // N
        full = _full_qkv(B, L, heads, d)                              # [B, L, 3, heads, d]
        ex.qkv_rows.copy_(full[:, rank * rows:(rank + 1) * rows].reshape(B, rows, -1))
        ex.to_heads()
        want = full[:, :, :, rank * hl:(rank + 1) * hl, :].permute(2, 0, 1, 3, 4).reshape(3, B, L, hl * d)
        ok_heads = torch.equal(ex.qkv_heads, want)
        # outputs: o_heads = q of this rank's heads plus 0.5 (any function of
        # (b, token, head, channel) will do); back to token shards
        ex.o_heads.copy_(ex.qkv_heads[0] + 0.5)
        ex.to_rows()
        want_o = (full[:, rank * rows:(rank + 1) * rows, 0] + 0.5).reshape(B, rows, heads * d)
        ok_rows = torch.equal(ex.o_rows, want_o)
        out[rank] = (ok_heads, ok_rows)
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,B,L,heads,d", [(2, 2, 12, 4, 16), (4, 2, 20, 8, 8), (4, 1, 8, 4, 4)])
def test_exchange_order(world, B, L, heads, d):
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_rank, args=(world, port, B, L, heads, d, out), nprocs=world, join=True)
        res = dict(out)
    for r in range(world):
        assert res[r] == (True, True), (r, res[r])


def test_exchange_rejects_uneven_split():
    with pytest.raises(ValueError):
        UlyssesExchange(1, 10, 4, 8, 4, torch.float32, device="cpu")
    with pytest.raises(ValueError):
        UlyssesExchange(1, 8, 4, 6, 4, torch.float32, device="cpu")


def test_host_permutation_is_the_documented_one():
    """dst axis k runs over src axis perm[k]: checked element by element."""
    src = torch.arange(2 * 3 * 4 * 5 * 8, dtype=torch.float32)
    dims, perm = (2, 3, 4, 5), (3, 0, 1, 2)
    dst = torch.empty_like(src)
    permute_chunks_host(src, dst, dims, perm, 8 * 4)
    s = src.view(2, 3, 4, 5, 8)
    d = dst.view(5, 2, 3, 4, 8)
    for i0 in range(2):
        for i1 in range(3):
            for i2 in range(4):
                for i3 in range(5):
                    assert torch.equal(d[i3, i0, i1, i2], s[i0, i1, i2, i3])


# ------------------------------------------------------------------ C entry points (no launch)

@pytest.fixture(scope="module")
def lib():
    build_lib.build(verbose=False)
    return wan.load()


def test_permute_chunks_rejects_bad_arguments(lib):
    P = wan.wan_permute_chunks
    assert P(16, 1 << 20, 0, [], [], 16, None) == wan.WAN_EINVAL              # ndim 0
    assert P(16, 1 << 20, 6, [1] * 6, list(range(6)), 16, None) == wan.WAN_EINVAL
    assert P(16, 1 << 20, 2, [2, 3], [0, 0], 16, None) == wan.WAN_EINVAL      # not a permutation
    assert P(16, 1 << 20, 2, [2, 3], [1, 0], 8, None) == wan.WAN_EINVAL       # chunk not a multiple of 16
    assert P(16, 32, 2, [2, 3], [1, 0], 16, None) == wan.WAN_EINVAL           # overlap
    assert P(24, 1 << 20, 2, [2, 3], [1, 0], 16, None) == wan.WAN_EALIGN
    assert P(16, 1 << 20, 2, [0, 3], [1, 0], 16, None) == wan.WAN_OK          # empty


def _dims(**kw):
    base = dict(F=2, H=4, W=4, dim=128, heads=4, ffn_dim=512, text_len=8, eps=1e-6, dtype="f32")
    base.update(kw)
    return wan.make_dims(**base)


def test_sp_phases_reject_bad_shards(lib):
    w = wan.wan_block_weights(*([4096] * len(wan.WEIGHT_FIELDS)))
    d = _dims()
    n = wan.wan_block_sp_workspace_bytes(d, 2, 16)
    assert n > 0 and n < wan.wan_block_workspace_bytes(d, 2)
    Q = lambda dd, rows, tok0, qkv=4096: wan.wan_block_sp_qkv(dd, 2, rows, tok0, 4096, 4096, w, 4096, 1024, qkv,
                                                             4096, 1 << 30, None)
    assert Q(d, 16, 17) == wan.WAN_EINVAL                 # past the 32-token grid
    assert Q(d, 0, 0) == wan.WAN_EINVAL
    assert Q(d, 16, -1) == wan.WAN_EINVAL
    assert Q(d, 16, 0, qkv=None) == wan.WAN_EINVAL
    assert Q(d, 16, 0, qkv=4104) == wan.WAN_EALIGN
    assert Q(_dims(dtype="fp8", dim=256, heads=2), 16, 0) == wan.WAN_EUNSUPPORTED
    F = lambda dd, rows, o=4096: wan.wan_block_sp_finish(dd, 2, rows, 4096, 4096, None, 4096, w, o, 4096, 1 << 30,
                                                         None)
    assert F(d, 33) == wan.WAN_EINVAL
    assert F(d, 16, o=None) == wan.WAN_EINVAL
    assert F(d, 16, o=4100) == wan.WAN_EALIGN
    assert wan.wan_block_sp_finish(d, 2, 16, 4096, 4096, None, 4096, w, 4096, 4096, 100, None) == wan.WAN_EINVAL
