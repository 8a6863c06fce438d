"""wan_block_forward_noalloc: the block forward for callers that cannot
allocate device memory (for example a plug-in whose host framework owns the
GPU memory pool, or a loop where allocating is not allowed), using the
library's built-in workspace array instead of a caller-supplied one.

Each case first runs the no-allocation entry point on a different problem,
so the shared array holds unrelated contents, then runs the block through the
existing entry point (wan_block_forward with a torch-allocated workspace) and
through wan_block_forward_noalloc twice in a row on the same inputs -- the
second call finds the previous call's contents in the array. Both paths run
the same kernels and the block is bit-deterministic, so the outputs must be
identical: a stale byte read from the array would show. This file is
collected last so that a run stopping at the first failure has run every
other test; it also passes alone.
"""
import pytest
import torch

from video_diffusion_transformer_fwd_b200 import configs, synth, wan
from video_diffusion_transformer_fwd_b200.configs import BlockConfig



def _setup(cfg, B, seed):
    dev = "cuda"
    dims = wan.dims_of(cfg)
    w = synth.block_weights(cfg.dim, cfg.ffn_dim, cfg.dtype, dev, seed)
    acts = synth.block_activations(B, cfg.L, cfg.dim, cfg.text_len, cfg.dtype, dev, seed + 100)
    rope = wan.rope_freqs(cfg.head_dim, 1024, cfg.theta, device=dev)
    return dims, wan.make_weights(w), w, acts, rope


def _noalloc(dims, B, x, acts, cw, rope, ctx_lens=None):
    s = torch.cuda.current_stream().cuda_stream
    return wan.wan_block_forward_noalloc(dims, B, x.data_ptr(), acts["ctx"].data_ptr(),
                                         None if ctx_lens is None else ctx_lens.data_ptr(),
                                         acts["e0"].data_ptr(), cw, rope.data_ptr(), rope.shape[0], s)


@pytest.mark.gpu
@pytest.mark.parametrize("cfg,B", [
    (configs.get("tiny"), 2),
    (BlockConfig("bf16-small", 3, 5, 7, 256, 2, 512, 24, "bf16"), 2),
])
def test_noalloc_matches_workspace_entry_point(cfg, B):
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    # an unrelated problem first: other dtype, grid and text length, so the
    # shared array is left holding values that are wrong for the cases below
    other = (BlockConfig("bf16-other", 2, 4, 6, 256, 2, 256, 11, "bf16") if cfg.dtype == "f32"
             else BlockConfig("f32-other", 3, 4, 5, 128, 2, 256, 7, "f32"))
    od, ocw, _, oacts, orope = _setup(other, 1, seed=29)
    wan.check(_noalloc(od, 1, oacts["x"], oacts, ocw, orope))
    torch.cuda.synchronize()

    dims, cw, w, acts, rope = _setup(cfg, B, seed=17)
    assert wan.wan_block_workspace_bytes(dims, B) <= wan.WAN_NOALLOC_WORKSPACE_BYTES
    x0 = acts["x"].clone()
    ref = x0.clone()
    ws = wan.alloc_workspace(dims, B)
    wan.block_forward(dims, ref, acts["ctx"], acts["e0"], cw, rope, ws)
    torch.cuda.synchronize()
    for call in range(2):
        x = x0.clone()
        wan.check(_noalloc(dims, B, x, acts, cw, rope))
        torch.cuda.synchronize()
        assert wan.device_status() == wan.WAN_OK
        assert torch.equal(x, ref), (call, float((x - ref).abs().max()))
    # and the block did change x (the comparison is not between two no-ops)
    assert not torch.equal(ref, x0)


def test_noalloc_rejects_problems_larger_than_its_array():
    """A problem whose workspace exceeds the built-in array is refused on the
    host, before anything is launched, with a message naming both sizes."""
    cfg = configs.get("1.3b-short")
    dims = wan.dims_of(cfg)
    need = wan.wan_block_workspace_bytes(dims, 1)
    assert need > wan.WAN_NOALLOC_WORKSPACE_BYTES
    cw = wan.wan_block_weights(*([4096] * len(wan.WEIGHT_FIELDS)))
    rc = wan.wan_block_forward_noalloc(dims, 1, 4096, 4096, None, 4096, cw, 4096, 1024, None)
    assert rc == wan.WAN_EINVAL
    msg = wan.last_error()
    assert str(need) in msg and str(wan.WAN_NOALLOC_WORKSPACE_BYTES) in msg
