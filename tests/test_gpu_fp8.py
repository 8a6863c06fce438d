"""FP8 GEMM path ("Wan paper deep dive", inference-optimisation table, "FP8
GEMM"): e4m3 quantization bit-exact against the oracle on the same inputs,
the FP8 linear layer against the oracle's exact product of the same codes,
and the FP8 block against the oracle's FP8 block."""
import numpy as np
import pytest
import torch

from oracle import wan_oracle as O
from video_diffusion_transformer_fwd_b200 import synth, wan
from video_diffusion_transformer_fwd_b200.configs import BlockConfig

from parity_util import BF16_REL_L2, np64, rel_l2, weights64

pytestmark = pytest.mark.gpu

# FP8 block against the oracle's FP8 block: an upstream relative discrepancy
# eps between the two sides (bf16 storage, attention; ~3e-3 to 8e-3 on the bf16
# path) moves a fraction ~eps/delta of the e4m3 codes by one step delta
# (~2^-3.5 of the value), a relative L2 change of ~sqrt(eps * delta) <= 2.7e-2
# in a projection's input; 5e-2 leaves a factor ~2 for their sum over a branch.
FP8_REL_L2 = 5e-2


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    wan.load()


def _rows_input(rows, cols, dtype, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    x = torch.randn(rows, cols, device="cuda", generator=g)
    x *= torch.exp2(torch.randint(-20, 20, (rows, 1), device="cuda", generator=g).float())
    if rows > 2:
        x[2] = 0.0                                     # an all-zero row
    return x.to(synth.TORCH_DTYPES[dtype])


def _codes_equal(q_gpu, q_ref):
    v = O.e4m3_decode(q_gpu.cpu().numpy())
    assert not np.isnan(v).any()
    return np.array_equal(v, q_ref)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("rows,cols", [(1, 4), (37, 300), (64, 1024), (5, 13824), (300, 5120)])
def test_quantize_rows_bit_exact(dtype, rows, cols):
    x = _rows_input(rows, cols, dtype, rows * 7 + cols)
    q, sc = wan.quantize_fp8(x, per_row=True)
    torch.cuda.synchronize()
    qr, sr = O.quantize_fp8(np64(x), per_row=True)
    assert np.array_equal(np64(sc), sr[:, 0])
    assert _codes_equal(q, qr)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("shape", [(4,), (5120, 512), (13824, 640)])
def test_quantize_tensor_bit_exact(dtype, shape):
    g = torch.Generator(device="cuda").manual_seed(11)
    w = (torch.randn(shape, device="cuda", generator=g) * 0.02).to(synth.TORCH_DTYPES[dtype])
    q, sc = wan.quantize_fp8(w.reshape(1, -1) if len(shape) == 1 else w, per_row=False)
    torch.cuda.synchronize()
    qr, sr = O.quantize_fp8(np64(w), per_row=False)
    assert np64(sc)[0] == sr
    assert _codes_equal(q.reshape(shape), qr)


def test_quantize_zero_tensor_and_empty():
    z = torch.zeros(8, 64, device="cuda")
    q, sc = wan.quantize_fp8(z, per_row=False)
    q2, sc2 = wan.quantize_fp8(z, per_row=True)
    torch.cuda.synchronize()
    assert not q.any() and sc.item() == 0.0 and not q2.any() and not sc2.any()
    e = torch.zeros(0, 64, device="cuda")
    wan.quantize_fp8(e, per_row=True)


@pytest.mark.parametrize("M,N,K", [(1, 32, 128), (200, 256, 640), (300, 608, 1024), (4096, 5120, 5120)])
@pytest.mark.parametrize("with_bias", [True, False])
def test_linear_fp8(M, N, K, with_bias):
    g = torch.Generator(device="cuda").manual_seed(M + N + K)
    a = torch.randn(M, K, device="cuda", generator=g)
    w = (torch.randn(N, K, device="cuda", generator=g) * 0.02).to(torch.bfloat16)
    b = (torch.randn(N, device="cuda", generator=g) * 0.02).to(torch.bfloat16) if with_bias else None
    qa, sa = wan.quantize_fp8(a, per_row=True)
    qw, sw = wan.quantize_fp8(w, per_row=False)
    out = wan.linear_fp8(qa, sa, qw, sw, b)
    torch.cuda.synchronize()
    rows = synth.sample_rows(M, 256, seed=3)
    a64, w64 = np64(a)[rows], np64(w)
    ref = O.linear_fp8(a64, w64, None if b is None else np64(b))
    got = np64(out)[rows]
    # the oracle's own codes are the GPU's (bit-exact quantization), so the
    # only difference is the fp32 accumulation and scaling: bounded by
    # K 2^-24 times the sum of |products|, plus the final rounding
    qa_r, sa_r = O.quantize_fp8(a64, per_row=True)
    qw_r, sw_r = O.quantize_fp8(w64, per_row=False)
    mag = (np.abs(qa_r) @ np.abs(qw_r).T) * sa_r * sw_r
    bound = (K + 4) * 2.0 ** -24 * mag + 2.0 ** -23 * np.abs(ref) + 1e-30
    assert (np.abs(got - ref) <= bound).all()


def test_linear_fp8_rejects_bad_shapes():
    z8 = torch.zeros(64, 100, dtype=torch.uint8, device="cuda")
    s = torch.ones(64, device="cuda")
    out = torch.empty(64, 64, device="cuda")
    rc = wan.wan_linear_fp8(64, 64, 100, z8.data_ptr(), s.data_ptr(), z8.data_ptr(), s.data_ptr(), None,
                            out.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert rc == wan.WAN_EUNSUPPORTED


# ------------------------------------------------------------------ FP8 block

def _fp8_block(cfg, B=2, seed=0, ctx_lens=None, same_x=False, same_e0=False):
    w16 = synth.block_weights(cfg.dim, cfg.ffn_dim, "bf16", "cuda", seed)
    w8 = wan.quantize_block_weights(w16)
    acts = synth.block_activations(B, cfg.L, cfg.dim, cfg.text_len, "bf16", "cuda", seed + 100,
                                   same_x=same_x, same_e0=same_e0)
    dims = wan.make_dims(cfg.F, cfg.H, cfg.W, cfg.dim, cfg.heads, cfg.ffn_dim, cfg.text_len, cfg.eps, "fp8")
    rope = wan.rope_freqs(cfg.head_dim, 1024, cfg.theta)
    ws = wan.alloc_workspace(dims, B)
    x0 = acts["x"].clone()
    kl = None if ctx_lens is None else torch.tensor(ctx_lens, dtype=torch.int32, device="cuda")
    wan.block_forward(dims, acts["x"], acts["ctx"], acts["e0"], w8, rope, ws, ctx_lens=kl)
    torch.cuda.synchronize()
    assert wan.device_status() == wan.WAN_OK
    return dims, ws, w16, acts, x0


def test_block_fp8_small_full():
    cfg = BlockConfig("fp8-small", 2, 8, 8, 256, 2, 512, 16, "bf16")
    lens = [16, 9]
    dims, ws, w16, acts, x0 = _fp8_block(cfg, ctx_lens=lens)
    args = (np64(x0), np64(acts["ctx"]), np.array(lens), np64(acts["e0"]), weights64(w16), cfg.heads,
            (cfg.F, cfg.H, cfg.W), cfg.eps)
    inter = {}
    ref = O.block_forward(*args, fp8=True, intermediates=inter)
    got = np64(acts["x"])
    x = np64(x0)
    assert rel_l2(got, ref) <= BF16_REL_L2
    assert rel_l2(got - x, ref - x) <= FP8_REL_L2
    # the three branch intermediates
    L, D = cfg.L, cfg.dim
    for which, key, width in ((wan.WAN_WS_O, "o_self", D), (wan.WAN_WS_OC, "o_cross", D),
                              (wan.WAN_WS_H, "h", cfg.ffn_dim)):
        v = wan.workspace_view(ws, dims, 2, which, (2, L, width), torch.bfloat16)
        assert rel_l2(np64(v), inter[key]) <= FP8_REL_L2, key
    # and the FP8 block stays near the exact block (the quantization error itself)
    exact = O.block_forward(*args)
    assert rel_l2(got - x, exact - x) <= 0.15


@pytest.mark.parametrize("name", ["1.3b-short", "a14b-step"])
def test_block_fp8_sampled_rows(name):
    from video_diffusion_transformer_fwd_b200 import configs
    cfg = configs.get(name)
    step = name == "a14b-step"
    dims, ws, w16, acts, x0 = _fp8_block(cfg, B=2, same_x=step, same_e0=step)
    rows = synth.sample_rows(cfg.L, 256, seed=5)
    w64, grid = weights64(w16), (cfg.F, cfg.H, cfg.W)
    x64, e064 = np64(x0), np64(acts["e0"])
    kv = None
    if step:        # one x and one timestep for both sequences: their keys and values agree
        k1, v1 = O.self_attn_kv(x64[:1], e064[:1], w64, cfg.heads, grid, cfg.eps, cfg.theta, fp8=True)
        kv = (np.repeat(k1, 2, axis=0), np.repeat(v1, 2, axis=0))
    ref = O.block_forward_rows(x64, np64(acts["ctx"]), None, e064, w64, cfg.heads, grid, cfg.eps, rows,
                               theta=cfg.theta, kv=kv, fp8=True)
    got = np64(acts["x"])[:, rows]
    x = np64(x0)[:, rows]
    assert rel_l2(got, ref) <= BF16_REL_L2
    assert rel_l2(got - x, ref - x) <= FP8_REL_L2


def test_block_fp8_deterministic():
    cfg = BlockConfig("fp8-det", 2, 8, 8, 256, 2, 512, 16, "bf16")
    a = _fp8_block(cfg, seed=4)[3]["x"].clone()
    b = _fp8_block(cfg, seed=4)[3]["x"]
    assert torch.equal(a, b)
