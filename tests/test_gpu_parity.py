"""Parity of the CUDA path (through the C ABI) against the fp64 oracle on the
same seeded inputs. fp32: max-abs <= 1e-4; bf16: relative L2 <= 2e-2 on
sampled token rows, also on the block delta and on each branch output."""
import math

import numpy as np
import pytest
import torch

from oracle import wan_oracle as O
from video_diffusion_transformer_fwd_b200 import configs, synth, wan
from video_diffusion_transformer_fwd_b200.configs import BlockConfig

from parity_util import BF16_REL_L2, F32_MAX_ABS, GpuBlockRun, Guarded, np64, rel_l2, weights64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    wan.load()


# ------------------------------------------------------------------ RoPE table

@pytest.mark.parametrize("d", [32, 128])
def test_rope_table(d):
    t = np64(wan.rope_freqs(d, 1024, 1e4))
    ref = O.rope_table(d, 1024, 1e4)
    assert np.abs(t - ref).max() <= 1.2e-7          # fp32 rounding of an fp64 angle


# ------------------------------------------------------------------ CFG + Euler

@pytest.mark.parametrize("vdt", ["f32", "bf16"])
@pytest.mark.parametrize("n", [1, 3, 1003, 1 << 20])
@pytest.mark.parametrize("cfg", [True, False])
def test_euler_cfg(vdt, n, cfg):
    g = torch.Generator(device="cuda").manual_seed(7)
    gx = Guarded((n,), torch.float32, init=torch.randn(n, device="cuda", generator=g))
    x = gx.t
    vc = torch.randn(n, device="cuda", generator=g).to(synth.TORCH_DTYPES[vdt])
    vu = torch.randn(n, device="cuda", generator=g).to(synth.TORCH_DTYPES[vdt]) if cfg else None
    x0 = np64(x)
    wan.euler_cfg_step(x, vc, vu, 5.0, 0.9, 0.875)
    torch.cuda.synchronize()
    gx.check("euler x")
    dt = float(np.float32(0.875) - np.float32(0.9))
    ref = O.euler_cfg_step(x0, np64(vc), None if vu is None else np64(vu), 5.0, 0.9, 0.9 + dt)
    assert np.abs(np64(x) - ref).max() <= 1e-5


def test_euler_cfg_empty():
    x = torch.zeros(4, device="cuda")
    wan.check(wan.wan_euler_cfg_step(x.data_ptr(), x.data_ptr(), None, wan.WAN_F32, 0, 5.0, 0.9,
                                     0.875, torch.cuda.current_stream().cuda_stream))


# ------------------------------------------------------------------ attention

def _attn_case(B, Lq, Lk, n, d, dtype, k_lens=None, std=1.0, seed=500):
    q, k, v = synth.attention_inputs(B, Lq, Lk, n, d, dtype, "cuda", seed, std)
    kl = None if k_lens is None else torch.tensor(k_lens, dtype=torch.int32, device="cuda")
    go = Guarded(tuple(q.shape), q.dtype)
    o = wan.attention(q, k, v, k_lens=kl, out=go.t)
    torch.cuda.synchronize()
    go.check("attention output")
    got = np64(o)
    ref = np.stack([O.attention(np64(q[b]), np64(k[b]), np64(v[b]),
                                None if k_lens is None else k_lens[b]) for b in range(B)])
    return got, ref


@pytest.mark.parametrize("d", [32, 64, 128])
def test_attention_f32(d):
    got, ref = _attn_case(2, 77, 200, 3, d, "f32", k_lens=[200, 57])
    assert np.abs(got - ref).max() <= F32_MAX_ABS


def test_attention_f32_zero_keys_and_sharp():
    got, ref = _attn_case(2, 40, 33, 2, 128, "f32", k_lens=[0, 1])
    assert np.abs(got - ref).max() <= F32_MAX_ABS
    assert np.all(got[0] == 0.0)
    got, ref = _attn_case(1, 65, 300, 2, 64, "f32", std=4.0)    # logits std ~ 16
    assert np.abs(got - ref).max() <= F32_MAX_ABS


@pytest.mark.parametrize("Lq,Lk", [(128, 128), (200, 333), (1, 7), (300, 512)])
def test_attention_bf16(Lq, Lk):
    got, ref = _attn_case(2, Lq, Lk, 3, 128, "bf16", k_lens=[Lk, max(1, Lk // 3)])
    assert rel_l2(got, ref) <= BF16_REL_L2
    got, ref = _attn_case(1, Lq, Lk, 2, 128, "bf16", std=2.5)   # sharp softmax
    assert rel_l2(got, ref) <= BF16_REL_L2


def test_attention_rope_in_place_f32():
    grid = (3, 4, 5)
    L = 60
    q, k, v = synth.attention_inputs(2, L, L, 2, 64, "f32", "cuda", 900)
    q0, k0 = np64(q), np64(k)
    rope = wan.rope_freqs(64, 1024)
    o = wan.attention(q, k, v, grid=grid, rope=rope)
    torch.cuda.synchronize()
    for b in range(2):
        qr = O.rope_apply(q0[b], grid)
        kr = O.rope_apply(k0[b], grid)
        assert np.abs(np64(q[b]) - qr).max() <= 1e-5
        ref = O.attention(qr, kr, np64(v[b]))
        assert np.abs(np64(o[b]) - ref).max() <= F32_MAX_ABS


# ------------------------------------------------------------------ block, fp32

TINY = configs.get("tiny")


def test_block_tiny_f32_full():
    run = GpuBlockRun(TINY, B=2, seed=0).run()
    inter = {}
    rows = np.arange(TINY.L)
    ref = run.oracle_rows(rows, intermediates=inter)
    assert np.abs(np64(run.x) - ref).max() <= F32_MAX_ABS
    assert np.abs(run.ws_rows(wan.WAN_WS_O, TINY.dim, rows) - inter["o_self"]).max() <= F32_MAX_ABS
    assert np.abs(run.ws_rows(wan.WAN_WS_OC, TINY.dim, rows) - inter["o_cross"]).max() <= F32_MAX_ABS
    assert np.abs(run.ws_rows(wan.WAN_WS_H, TINY.ffn_dim, rows) - inter["h"]).max() <= F32_MAX_ABS


def test_block_tiny_f32_against_scalar_oracle():
    """The tiny fp32 block against the scalar-loop form of the oracle."""
    from oracle import wan_oracle_scalar as S
    run = GpuBlockRun(TINY, B=2, seed=0, ctx_lens=[8, 3]).run()
    grid = (TINY.F, TINY.H, TINY.W)
    w = weights64(run.w)
    for b, kl in enumerate((8, 3)):
        ref = np.array(S.block_forward(np64(run.x0[b]), np64(run.ctx[b]), kl, np64(run.e0[b]), w,
                                       TINY.heads, grid, TINY.eps, TINY.theta))
        assert np.abs(np64(run.x[b]) - ref).max() <= F32_MAX_ABS


def test_block_tiny_f32_ctx_lens_and_sharp():
    run = GpuBlockRun(TINY, B=2, seed=3, ctx_lens=[5, 1], gain_scale=4.0).run()
    ref = run.oracle_rows(np.arange(TINY.L))
    assert np.abs(np64(run.x) - ref).max() <= F32_MAX_ABS


def test_block_tiny_f32_zero_text_len():
    cfg = BlockConfig("tiny-t0", 2, 4, 4, 128, 4, 512, 0, "f32")
    run = GpuBlockRun(cfg, B=1, seed=5).run()
    ref = run.oracle_rows(np.arange(cfg.L))
    assert np.abs(np64(run.x) - ref).max() <= F32_MAX_ABS


def test_block_f32_ragged_grid_head64():
    # L = 3*5*7 = 105 (not a multiple of any tile), head_dim 64
    cfg = BlockConfig("ragged", 3, 5, 7, 256, 4, 512, 13, "f32")
    run = GpuBlockRun(cfg, B=2, seed=11, ctx_lens=[13, 4]).run()
    ref = run.oracle_rows(np.arange(cfg.L))
    assert np.abs(np64(run.x) - ref).max() <= F32_MAX_ABS


def test_block_gates_zero_and_cross_out_zero_is_identity():
    run = GpuBlockRun(TINY, B=2, seed=4, zero_gates=True)
    run.w["cwo"].zero_()
    run.w["cbo"].zero_()
    run.run()
    assert torch.equal(run.x, run.x0)


def test_block_is_deterministic():
    a = GpuBlockRun(TINY, B=2, seed=9).run()
    b = GpuBlockRun(TINY, B=2, seed=9).run()
    assert torch.equal(a.x, b.x)


def test_block_bf16_is_deterministic():
    """The tensor-core path (including the TMA reduce-add residual) gives
    bit-identical results run to run."""
    cfg = BlockConfig("bf16-det", 3, 5, 7, 512, 4, 1024, 24, "bf16")
    a = GpuBlockRun(cfg, B=2, seed=13).run()
    b = GpuBlockRun(cfg, B=2, seed=13).run()
    assert torch.equal(a.x, b.x)


def test_tiny_stack_of_40_blocks_and_step():
    """The denoising-step launch sequence (40 blocks on the CFG pair, then
    CFG-Euler) on the tiny config, against the full fp64 chain."""
    from video_diffusion_transformer_fwd_b200.step import DenoiseStep
    cfg = BlockConfig("tiny-step", 2, 4, 4, 128, 4, 512, 8, "f32", batch=2, blocks=40)
    st = DenoiseStep(cfg, seed=0)
    x0 = np64(st.x)
    st.step()
    torch.cuda.synchronize()
    ref = O.denoise_step(x0, np64(st.ctx[0]), np64(st.ctx[1]), None, np64(st.e0[0]),
                         [weights64(w) for w in st.weights], cfg.heads, (cfg.F, cfg.H, cfg.W),
                         cfg.eps, cfg.guide_scale, cfg.sigma, cfg.sigma_next)
    assert np.abs(np64(st.x) - ref).max() <= F32_MAX_ABS


def test_bf16_stack_of_40_blocks_and_step():
    """The denoising-step launch sequence at a bf16 size where the whole fp64
    chain is affordable (40 blocks, dim 512, 4 heads of 128, ffn 1024, grid
    4 x 8 x 16 = 512 tokens, text 64, CFG pair): the two block-stack outputs
    (their accumulated change over the 40 blocks) and the CFG-Euler update,
    every row, against the oracle run block by block on its own outputs."""
    from video_diffusion_transformer_fwd_b200.step import DenoiseStep
    cfg = BlockConfig("bf16-chain", 4, 8, 16, 512, 4, 1024, 64, "bf16", batch=2, blocks=40)
    st = DenoiseStep(cfg, seed=0)
    x0 = np64(st.x)
    st.step()
    torch.cuda.synchronize()
    assert wan.device_status() == wan.WAN_OK
    grid = (cfg.F, cfg.H, cfg.W)
    ctx = np.stack([np64(st.ctx[0]), np64(st.ctx[1])])
    e0 = np.stack([np64(st.e0[0])] * 2)
    xb = np.stack([x0, x0])
    for w in st.weights:
        xb = O.block_forward(xb, ctx, None, e0, weights64(w), cfg.heads, grid, cfg.eps, cfg.theta)
    ref = O.euler_cfg_step(x0, xb[0], xb[1], cfg.guide_scale, cfg.sigma, cfg.sigma_next)
    got_v = np64(st.xb)
    errs = {"stack_delta_cond": rel_l2(got_v[0] - x0, xb[0] - x0),
            "stack_delta_uncond": rel_l2(got_v[1] - x0, xb[1] - x0),
            "cfg_direction": rel_l2(got_v[0] - got_v[1], xb[0] - xb[1]),
            "step_update": rel_l2(np64(st.x) - x0, ref - x0)}
    print({k: f"{v:.2e}" for k, v in errs.items()})
    for k, v in errs.items():
        assert v <= BF16_REL_L2, (k, v)


# ------------------------------------------------------------------ block, bf16 (sampled rows)

def _bf16_block_check(cfg, B=1, same=False, seed=0, gain_scale=1.0, ctx_lens=None):
    run = GpuBlockRun(cfg, B=B, seed=seed, same_x=same, same_e0=same, gain_scale=gain_scale,
                      ctx_lens=ctx_lens).run()
    rows = synth.sample_rows(cfg.L, 256)
    kv = None
    if same:
        k, v = O.self_attn_kv(np64(run.x0[:1]), np64(run.e0[:1]), weights64(run.w), cfg.heads,
                              (cfg.F, cfg.H, cfg.W), cfg.eps, cfg.theta)
        kv = (np.broadcast_to(k, (B,) + k.shape[1:]), np.broadcast_to(v, (B,) + v.shape[1:]))
    inter = {}
    ref = run.oracle_rows(rows, kv=kv, intermediates=inter)
    got = np64(run.x[:, torch.as_tensor(rows, device="cuda")])
    x0 = np64(run.x0[:, torch.as_tensor(rows, device="cuda")])
    errs = {
        "out": rel_l2(got, ref),
        "delta": rel_l2(got - x0, ref - x0),
        "o_self": rel_l2(run.ws_rows(wan.WAN_WS_O, cfg.dim, rows), inter["o_self"]),
        "o_cross": rel_l2(run.ws_rows(wan.WAN_WS_OC, cfg.dim, rows), inter["o_cross"]),
        "h": rel_l2(run.ws_rows(wan.WAN_WS_H, cfg.ffn_dim, rows), inter["h"]),
    }
    print(cfg.name, {k: f"{v:.2e}" for k, v in errs.items()})
    for k, v in errs.items():
        assert v <= BF16_REL_L2, (k, v)
    return errs


def test_block_bf16_small_ragged():
    cfg = BlockConfig("bf16-small", 3, 5, 7, 256, 2, 512, 24, "bf16")
    _bf16_block_check(cfg, B=2, ctx_lens=[24, 9])


def test_block_bf16_small_sharp():
    cfg = BlockConfig("bf16-sharp", 2, 8, 16, 512, 4, 1024, 64, "bf16")
    _bf16_block_check(cfg, B=2, gain_scale=4.0)


@pytest.mark.parametrize("dim", [4096, 7168, 8192])
def test_block_bf16_wide_dims(dim):
    """Model widths beyond the configs' (up to the LayerNorm's 8192 limit): every
    row layout of the LayerNorm kernel (float4 chunks per thread: 4, 7 and 8)
    and head counts 32 to 64, on a small ragged token grid."""
    cfg = BlockConfig(f"bf16-wide-{dim}", 2, 3, 5, dim, dim // 128, dim, 16, "bf16")
    _bf16_block_check(cfg, B=2, ctx_lens=[16, 5])


@pytest.mark.parametrize("dim,ffn", [(256, 576), (4096, 4160)])
def test_block_bf16_ffn_partial_tiles(dim, ffn):
    """FFN widths that are multiples of 64 but not of 256: the FFN1 GEMM ends in
    a partial column tile (64 of 256 columns on the narrow tile, K = 256; 64 of
    512 on the wide tile, K = 4096, whose second column half holds no output at
    all); the FFN2 GEMM then runs K = 576 / 4160, 9 and 65 K stages of 64."""
    cfg = BlockConfig(f"bf16-ffn{ffn}", 2, 3, 5, dim, dim // 128, ffn, 16, "bf16")
    _bf16_block_check(cfg, B=2, ctx_lens=[16, 7])


def test_block_1p3b_short():
    _bf16_block_check(configs.get("1.3b-short"))


def test_block_1p3b_long():
    _bf16_block_check(configs.get("1.3b-long"))


def test_block_5b():
    _bf16_block_check(configs.get("5b"))


def test_block_a14b_cfg_pair():
    """The A14B block in the step's launch configuration: B = 2 (cond and
    uncond share x and e0, contexts differ)."""
    _bf16_block_check(configs.get("a14b-step"), B=2, same=True)


def test_block_1p3b_long_f32_pass():
    """The 1.3B block at L = 32760 entirely in fp32 (LN, RoPE and attention
    at full length), max-abs on sampled rows."""
    cfg = configs.get("1.3b-long")
    run = GpuBlockRun(cfg, B=1, seed=21, dtype="f32").run()
    rows = synth.sample_rows(cfg.L, 64)
    ref = run.oracle_rows(rows)
    got = np64(run.x[:, torch.as_tensor(rows, device="cuda")])
    assert np.abs(got - ref).max() <= F32_MAX_ABS


# ------------------------------------------------------------------ failure path, full-size step

def test_watchdog_wait_expires_and_context_survives():
    """A bounded wait that can never complete gives up, the host reads
    WAN_ETIMEOUT, and the next library call still works."""
    s = torch.cuda.current_stream().cuda_stream
    wan.check(wan.wan_selftest_watchdog(s))
    assert wan.wan_device_status(s) == wan.WAN_ETIMEOUT
    assert wan.wan_device_status(s) == wan.WAN_OK            # the status was cleared
    got, ref = _attn_case(1, 130, 200, 2, 128, "bf16")       # tensor-core path runs again
    assert rel_l2(got, ref) <= BF16_REL_L2


def test_a14b_step_full_size_identity():
    """The full-size A14B step (40 blocks, CFG pair, L = 32760) in the bench's
    launch sequence, with every gate and the cross-attention output projection
    zeroed: each block is then exactly the identity, so v_c = v_u = x and the
    step is x + (sigma' - sigma) x."""
    from video_diffusion_transformer_fwd_b200.step import DenoiseStep
    cfg = configs.get("a14b-step")
    st = DenoiseStep(cfg, seed=7)
    for w in st.weights:
        w["modulation"][2].zero_()
        w["modulation"][5].zero_()
        w["cwo"].zero_()
        w["cbo"].zero_()
    st.e0[:, 2].zero_()
    st.e0[:, 5].zero_()
    x0 = st.x.clone()
    st.step()
    torch.cuda.synchronize()
    assert wan.device_status() == wan.WAN_OK
    assert torch.equal(st.xb[0], x0) and torch.equal(st.xb[1], x0)
    dt = float(np.float32(cfg.sigma_next) - np.float32(cfg.sigma))
    ref = O.euler_cfg_step(np64(x0), np64(x0), np64(x0), cfg.guide_scale, 0.0, dt)
    assert np.abs(np64(st.x) - ref).max() <= 1e-5
