"""8-bit attention ("Wan paper deep dive", inference-optimisation table, "8-bit
FlashAttention") through wan_attention_8bit and the WAN_FP8_ATTN block mode,
against the oracle's 8-bit attention on the same bf16 inputs."""
import numpy as np
import pytest
import torch

from oracle import wan_oracle as O
from video_diffusion_transformer_fwd_b200 import synth, wan
from video_diffusion_transformer_fwd_b200.configs import BlockConfig

from parity_util import BF16_REL_L2, np64, rel_l2, weights64

pytestmark = pytest.mark.gpu

# Kernel against oracle. Both sides take the same int8 / e4m3 decisions for
# q, k and v (fp32 rules) and differ only in how P is rounded: the oracle
# rounds 448 p with p = exp(s - m), m the exact row max; the kernel, which
# streams the keys, rounds P = p * sigma with sigma = 2^(m - F + 8) > 1 for
# the power-of-two frame F it held when that key tile was processed (F is
# below m + 8), so P <= 2^8 never saturates. An e4m3 value in its normal range
# (>= 2^-6) is within half an ulp, 2^-4 relative, of what it rounds; below
# 2^-6 the spacing is 2^-9, so within 2^-10 absolute. Per key j therefore
#   |P_kernel / sigma - p_j| <= e_k(j) = 2^-4 p_j   (p_j >= 2^-6), else 2^-10
#   |oracle's P - p_j|       <= e_o(j) = 2^-4 p_j   (448 p_j >= 2^-6), else 2^-10 / 448
# and, elementwise, with A = sum_j (e_k + e_o)(j) |vq_j| sv / l,
#   |o_kernel - o_oracle| <= A + the kernel's fp32 sums (Lk 2^-23 relative,
#   on l and on P V) + its bf16 output rounding (2^-9 relative).
# The roundings of the two sides fall on unrelated grids, so their errors are
# independent: a rounding error uniform within +-h has variance h^2 / 3, with
# h <= 2^-4 p_j (normal) or 2^-10 (subnormal) on the kernel's side and the
# oracle's exact half-spacing on its side. The squared difference summed over
# all outputs concentrates at E = sum (var_k + var_o)(j) vq_j^2 sv^2 / l^2, so
# the relative L2 difference is checked against 1.25 sqrt(E) / |o_oracle|
# plus the bf16 rounding.
FP8_REL_L2 = 5e-2          # block delta, as for the FP8 GEMM block
# o_self and the delta of the block with the 8-bit attention: the FP8 GEMM
# block's bound (2.7e-2 from the projections' code flips, see
# test_gpu_fp8.py) and the independent P roundings (at most
# sqrt(2 / 3) 2^-4 = 5.1e-2 relative when every p sits at the bottom of its
# binade) add in quadrature: 5.8e-2.
ATTN8_BLOCK_REL_L2 = 6e-2


def attn8_bounds(q, k, v, k_len=None):
    """(oracle output [Lq, n, d], elementwise bound on |kernel - oracle|,
    bound on the relative L2 difference) for one sequence."""
    p, l, vq, sv = O.attention_8bit_terms(q, k, v, k_len)
    ref = O.attention_8bit(q, k, v, k_len)
    kl = p.shape[2]
    if kl == 0:
        return ref, np.zeros_like(ref), 0.0
    e_k = np.where(p >= 2.0 ** -6, 2.0 ** -4 * p, 2.0 ** -10)
    p448 = p * 448.0
    ex = np.floor(np.log2(np.maximum(p448, 2.0 ** -6)))
    h_o = 2.0 ** (ex - 4.0) / 448.0                 # half the e4m3 spacing at 448 p, in units of p
    e_o = np.where(p448 >= 2.0 ** -6, 2.0 ** -4 * p, 2.0 ** -10 / 448.0)
    vabs = np.abs(vq)                                # [kl, n, d]
    A = np.einsum("nqk,knd->nqd", e_k + e_o, vabs) / l
    A1 = np.einsum("nqk,knd->nqd", p, vabs) / l
    A = np.transpose(A, (1, 0, 2)) * sv
    A1 = np.transpose(A1, (1, 0, 2)) * sv
    acc = kl * 2.0 ** -23
    elem = A + acc * (np.abs(ref) + A1) + 2.0 ** -9 * (np.abs(ref) + A) + 1e-30
    var = (e_k ** 2 + np.minimum(h_o, e_o) ** 2) / 3.0
    E = float((np.einsum("nqk,knd->nqd", var, vq ** 2) / l ** 2 * np.transpose(sv, (1, 0, 2)) ** 2).sum())
    nref = float(np.linalg.norm(ref))
    rel = 1.25 * np.sqrt(E) / nref + 2.0 ** -9 if nref > 0 else 0.0
    return ref, elem, rel


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    wan.load()


def _case(B, Lq, Lk, n, k_lens=None, std=1.0, seed=700):
    q, k, v = synth.attention_inputs(B, Lq, Lk, n, 128, "bf16", "cuda", seed, std)
    kl = None if k_lens is None else torch.tensor(k_lens, dtype=torch.int32, device="cuda")
    o = wan.attention_8bit(q, k, v, k_lens=kl)
    torch.cuda.synchronize()
    assert wan.device_status() == wan.WAN_OK
    got = np64(o)
    out = [attn8_bounds(np64(q[b]), np64(k[b]), np64(v[b]), None if k_lens is None else k_lens[b])
           for b in range(B)]
    exact = np.stack([O.attention(np64(q[b]), np64(k[b]), np64(v[b]), None if k_lens is None else k_lens[b])
                      for b in range(B)])
    return got, out, exact


def _check(got, out):
    for b, (ref, elem, rel) in enumerate(out):
        assert np.all(np.abs(got[b] - ref) <= elem), (b, float((np.abs(got[b] - ref) / elem).max()))
        assert rel_l2(got[b], ref) <= rel, (b, rel_l2(got[b], ref), rel)


@pytest.mark.parametrize("B,Lq,Lk,n,k_lens", [
    (1, 128, 128, 1, None),
    (2, 300, 300, 3, [300, 77]),
    (1, 200, 1000, 2, None),
    (2, 1, 129, 2, [129, 1]),
    (1, 513, 7, 1, None),
])
def test_attention_8bit_matches_oracle(B, Lq, Lk, n, k_lens):
    got, out, exact = _case(B, Lq, Lk, n, k_lens)
    _check(got, out)
    assert rel_l2(got, exact) <= 0.08


def test_attention_8bit_sharp_logits():
    got, out, exact = _case(2, 256, 640, 2, std=3.0, seed=701)
    _check(got, out)
    assert rel_l2(got, exact) <= 0.1


def test_attention_8bit_long_sequence_sampled():
    """One head at 16384 tokens (128 key tiles), checked on sampled rows."""
    B, L, n = 1, 16384, 1
    q, k, v = synth.attention_inputs(B, L, L, n, 128, "bf16", "cuda", 702)
    o = wan.attention_8bit(q, k, v)
    torch.cuda.synchronize()
    rows = synth.sample_rows(L, 128, seed=9)
    ref, elem, rel = attn8_bounds(np64(q[0])[rows], np64(k[0]), np64(v[0]))
    got = np64(o[0])[rows]
    assert np.all(np.abs(got - ref) <= elem)
    assert rel_l2(got, ref) <= rel


def test_attention_8bit_deterministic_and_rejects():
    q, k, v = synth.attention_inputs(1, 256, 256, 2, 128, "bf16", "cuda", 703)
    a = wan.attention_8bit(q, k, v)
    b = wan.attention_8bit(q, k, v)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    ws = torch.empty(16, dtype=torch.uint8, device="cuda")
    rc = wan.wan_attention_8bit(1, 2, 256, 256, q.data_ptr(), k.data_ptr(), v.data_ptr(), a.data_ptr(), None,
                                0.0, ws.data_ptr(), 16, torch.cuda.current_stream().cuda_stream)
    assert rc == wan.WAN_EINVAL
    assert wan.wan_attention_8bit_workspace_bytes(1, 2, 256, 0) == 0


# ------------------------------------------------------------------ block mode

def _block(cfg, B=2, seed=0, ctx_lens=None, same_x=False, same_e0=False):
    w16 = synth.block_weights(cfg.dim, cfg.ffn_dim, "bf16", "cuda", seed)
    w8 = wan.quantize_block_weights(w16)
    acts = synth.block_activations(B, cfg.L, cfg.dim, cfg.text_len, "bf16", "cuda", seed + 100,
                                   same_x=same_x, same_e0=same_e0)
    dims = wan.make_dims(cfg.F, cfg.H, cfg.W, cfg.dim, cfg.heads, cfg.ffn_dim, cfg.text_len, cfg.eps, "fp8attn")
    rope = wan.rope_freqs(cfg.head_dim, 1024, cfg.theta)
    ws = wan.alloc_workspace(dims, B)
    x0 = acts["x"].clone()
    kl = None if ctx_lens is None else torch.tensor(ctx_lens, dtype=torch.int32, device="cuda")
    wan.block_forward(dims, acts["x"], acts["ctx"], acts["e0"], w8, rope, ws, ctx_lens=kl)
    torch.cuda.synchronize()
    assert wan.device_status() == wan.WAN_OK
    return dims, ws, w16, acts, x0


def test_block_fp8_attn8_small_full():
    cfg = BlockConfig("fp8a-small", 2, 8, 12, 256, 2, 512, 16, "bf16")
    lens = [16, 5]
    dims, ws, w16, acts, x0 = _block(cfg, ctx_lens=lens)
    inter = {}
    ref = O.block_forward(np64(x0), np64(acts["ctx"]), np.array(lens), np64(acts["e0"]), weights64(w16),
                          cfg.heads, (cfg.F, cfg.H, cfg.W), cfg.eps, fp8=True, attn8=True, intermediates=inter)
    got, x = np64(acts["x"]), np64(x0)
    assert rel_l2(got, ref) <= BF16_REL_L2
    assert rel_l2(got - x, ref - x) <= ATTN8_BLOCK_REL_L2
    o = wan.workspace_view(ws, dims, 2, wan.WAN_WS_O, (2, cfg.L, cfg.dim), torch.bfloat16)
    assert rel_l2(np64(o), inter["o_self"]) <= ATTN8_BLOCK_REL_L2


def test_block_fp8_attn8_a14b_sampled():
    from video_diffusion_transformer_fwd_b200 import configs
    cfg = configs.get("a14b-step")
    dims, ws, w16, acts, x0 = _block(cfg, same_x=True, same_e0=True)
    rows = synth.sample_rows(cfg.L, 256, seed=5)
    w64, grid = weights64(w16), (cfg.F, cfg.H, cfg.W)
    x64, e064 = np64(x0), np64(acts["e0"])
    k1, v1 = O.self_attn_kv(x64[:1], e064[:1], w64, cfg.heads, grid, cfg.eps, cfg.theta, fp8=True)
    kv = (np.repeat(k1, 2, axis=0), np.repeat(v1, 2, axis=0))
    ref = O.block_forward_rows(x64, np64(acts["ctx"]), None, e064, w64, cfg.heads, grid, cfg.eps, rows,
                               theta=cfg.theta, kv=kv, fp8=True, attn8=True)
    got, x = np64(acts["x"])[:, rows], x64[:, rows]
    assert rel_l2(got, ref) <= BF16_REL_L2
    assert rel_l2(got - x, ref - x) <= ATTN8_BLOCK_REL_L2
