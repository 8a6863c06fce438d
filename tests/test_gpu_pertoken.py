"""Per-token timestep modulation ("Wan2.2 code walkthrough", time-projection
snippet: e0 unflattened to (batch, seq_len), as the TI2V model uses it):
blocks with e0 [B, L, 6, dim] and the model with t [B, L], through the C ABI,
against the fp64 oracle."""
import numpy as np
import pytest
import torch

from oracle import wan_oracle as O
from video_diffusion_transformer_fwd_b200 import synth, wan
from video_diffusion_transformer_fwd_b200.configs import BlockConfig

from parity_util import BF16_REL_L2, F32_MAX_ABS, np64, rel_l2, weights64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    wan.load()


def _ti2v_e0(B, grid, D, seed, distinct=True):
    """e0 per token: the first frame's tokens get one value, the rest another
    (the image-conditioned first frame at t = 0), or every token its own."""
    F, H, W = grid
    L = F * H * W
    g = torch.Generator(device="cuda").manual_seed(seed)
    if distinct:
        return torch.randn(B, L, 6, D, device="cuda", generator=g) * 0.1
    a = torch.randn(B, 1, 6, D, device="cuda", generator=g) * 0.1
    b = torch.randn(B, 1, 6, D, device="cuda", generator=g) * 0.1
    first = torch.zeros(1, L, 1, 1, device="cuda")
    first[:, :H * W] = 1.0
    return (a * first + b * (1 - first)).contiguous()


def _run_block(cfg, dtype, e0, ctx_lens=None, seed=0):
    dev = "cuda"
    B, L = e0.shape[0], cfg.L
    w = synth.block_weights(cfg.dim, cfg.ffn_dim, "bf16" if dtype in ("fp8", "fp8attn") else dtype, dev, seed)
    wk = wan.quantize_block_weights(w) if dtype in ("fp8", "fp8attn") else w
    acts = synth.block_activations(B, L, cfg.dim, cfg.text_len, "f32" if dtype == "f32" else "bf16", dev, seed + 100)
    dims = wan.make_dims(cfg.F, cfg.H, cfg.W, cfg.dim, cfg.heads, cfg.ffn_dim, cfg.text_len, cfg.eps, dtype,
                         e0_per_token=e0.dim() == 4)
    rope = wan.rope_freqs(cfg.head_dim, 1024, cfg.theta)
    ws = wan.alloc_workspace(dims, B)
    x = acts["x"].clone()
    kl = None if ctx_lens is None else torch.tensor(ctx_lens, dtype=torch.int32, device=dev)
    wan.block_forward(dims, x, acts["ctx"], e0.contiguous(), wk, rope, ws, ctx_lens=kl)
    torch.cuda.synchronize()
    assert wan.device_status() == wan.WAN_OK
    return x, acts, w


@pytest.mark.parametrize("distinct", [True, False])
def test_block_per_token_f32(distinct):
    cfg = BlockConfig("pt-tiny", 2, 4, 4, 128, 4, 512, 8, "f32")
    e0 = _ti2v_e0(2, (2, 4, 4), 128, 3, distinct)
    out, acts, w = _run_block(cfg, "f32", e0, ctx_lens=[8, 3])
    ref = O.block_forward(np64(acts["x"]), np64(acts["ctx"]), np.array([8, 3]), np64(e0), weights64(w),
                          cfg.heads, (cfg.F, cfg.H, cfg.W), cfg.eps)
    assert np.abs(np64(out) - ref).max() <= F32_MAX_ABS


def test_block_per_token_bf16():
    cfg = BlockConfig("pt-bf16", 3, 8, 8, 256, 2, 512, 16, "bf16")
    e0 = _ti2v_e0(2, (3, 8, 8), 256, 4, distinct=False)
    out, acts, w = _run_block(cfg, "bf16", e0)
    x = np64(acts["x"])
    ref = O.block_forward(x, np64(acts["ctx"]), None, np64(e0), weights64(w), cfg.heads, (cfg.F, cfg.H, cfg.W),
                          cfg.eps)
    got = np64(out)
    assert rel_l2(got, ref) <= BF16_REL_L2
    assert rel_l2(got - x, ref - x) <= BF16_REL_L2


def test_block_per_token_fp8():
    cfg = BlockConfig("pt-fp8", 2, 8, 8, 256, 2, 512, 16, "bf16")
    e0 = _ti2v_e0(2, (2, 8, 8), 256, 5, distinct=True)
    out, acts, w = _run_block(cfg, "fp8", e0)
    x = np64(acts["x"])
    ref = O.block_forward(x, np64(acts["ctx"]), None, np64(e0), weights64(w), cfg.heads, (cfg.F, cfg.H, cfg.W),
                          cfg.eps, fp8=True)
    got = np64(out)
    assert rel_l2(got, ref) <= BF16_REL_L2
    assert rel_l2(got - x, ref - x) <= 5e-2


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_equal_per_token_e0_is_bit_identical(dtype):
    cfg = BlockConfig("pt-eq", 2, 8, 8, 256, 2, 512, 16, dtype)
    g = torch.Generator(device="cuda").manual_seed(6)
    e0 = torch.randn(2, 6, 256, device="cuda", generator=g) * 0.1
    a, _, _ = _run_block(cfg, dtype, e0)
    b, _, _ = _run_block(cfg, dtype, e0[:, None].expand(2, cfg.L, 6, 256).contiguous())
    assert torch.equal(a, b)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_model_per_token_t(dtype):
    """TI2V-style timesteps: the first latent frame at t = 0, the rest at 900."""
    from test_gpu_model import ModelCase
    if dtype == "f32":
        c = ModelCase(16, 16, 3, 8, 10, 128, 4, 256, 9, 64, 2, "f32")
    else:
        c = ModelCase(48, 48, 2, 16, 32, 256, 2, 512, 16, 256, 1, "bf16")
    dims = c.dims
    dims.t_per_token = 1
    c.ws = wan.alloc_model_workspace(dims, 2)
    Lg = dims.F * (dims.H // 2) * (dims.W // 2)
    hw = (dims.H // 2) * (dims.W // 2)
    t = np.full((2, Lg), 900.0, np.float32)
    t[:, :hw] = 0.0
    t[1, hw:] = 312.5
    got = c.run(t)
    ref = c.oracle(t)
    if dtype == "f32":
        assert np.abs(got - ref).max() <= F32_MAX_ABS
    else:
        assert rel_l2(got, ref) <= BF16_REL_L2
