"""Plain fp64 CPU oracle for the Wan2.1 / Wan2.2 DiT block forward and the
CFG-combined flow-matching Euler step.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import, call or
execute this module: only the test suite (``tests/``), the smoke check in
``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference``
legs of ``bench.py`` use it. It shares no code with the CUDA library: it
takes plain numpy arrays (the exact values handed to the GPU, upcast to
float64) and returns float64 arrays.

Sources (the pages that define what is computed):

* [WALK] "Wan2.2 code walkthrough" (newtid.com/chuangyezixun/14194.html):
  the ``WanModel`` structure snippet, the forward snippet (patch, flatten,
  blocks), the time-projection snippet (6 x dim modulation), the
  ``WanAttentionBlock`` core-logic snippet, the 3D RoPE snippet, the
  self-attention snippet (global window, no causal mask) and the sampling
  loop snippet (classifier-free guidance).
* [DIGEST] "Wan paper deep dive" (charles2530.github.io), section
  "Video DiT and Flow Matching": token count formula, shared AdaLN MLP with a
  per-block bias, flow-matching path x_t = t x1 + (1-t) x0 and v = x1 - x0;
  and its inference-optimisation table (FP8 GEMM: one scale per weight
  tensor, one per activation token).
* [TRACE] "Wan2.2 I2V inference trace" (damodev.csdn.net), section 4 "DIT":
  token shapes and the CFG scale meaning (s = 1: prompt only).
* [DIFFUSERS] "diffusers WanPipeline walkthrough" (huan-yin.github.io),
  sections "3D Patchify" and "3D RoPE coordinate system".

Readings taken where the pages are silent:

* RoPE: every axis has its own frequency ladder omega_j = theta^(-2j/d_a),
  d_a the axis width in real dims (t: d - 4(d//6), h = w: 2(d//6)), and
  positions are 0-based grid indices; pairs are interleaved (2j, 2j+1).
* QK-RMSNorm normalises the full dim-wide projection (before the head split)
  with a learnable gain, for both self- and cross-attention q and k.
* norm1 / norm2 carry no affine; norm3 is an affine LayerNorm. LayerNorm uses
  the population variance with eps inside the square root.
* Softmax scale 1/sqrt(head_dim); every Linear has a bias.
* A query row with zero valid keys (key length 0) outputs zeros.
* FP8 GEMM: codes are e4m3 ("fn": no infinities, largest finite 448), the
  scale of a row or tensor is amax / 448, an element's code is the nearest
  e4m3 value to x * (448 / amax) (ties to even, clamped to +-448), and these
  decisions are taken in fp32; an all-zero row or tensor gets scale 0.

Every function cites the passage it follows.
"""
from __future__ import annotations

import math

import numpy as np

F64 = np.float64


# --------------------------------------------------------------------------
# Token grid  ([WALK] forward snippet: Conv3d patch, flatten(2).transpose;
# [DIGEST] token-count formula; [DIFFUSERS] "3D Patchify")
# --------------------------------------------------------------------------

def latent_grid(frames: int, height: int, width: int,
                vae_stride=(4, 8, 8), patch=(1, 2, 2)):
    """Token grid (F, H, W) of a clip after the VAE and the (1,2,2) patching.

    The causal VAE keeps the first frame and folds every further 4 frames into
    one latent frame ([TRACE] section 3.1 "encoder": 81 frames -> 21 latents),
    and divides height and width by the spatial stride; the DiT patch
    embedding then divides each axis by the patch size ([WALK] forward).
    """
    st, sh, sw = vae_stride
    pt, ph, pw = patch
    f_lat = 1 + (frames - 1) // st
    h_lat = height // sh
    w_lat = width // sw
    return (f_lat // pt, h_lat // ph, w_lat // pw)


def token_positions(F: int, H: int, W: int) -> np.ndarray:
    """(t, h, w) grid position of every token, shape [F*H*W, 3], int64.

    ``flatten(2)`` of a [C, F, H, W] tensor makes F the slowest and W the
    fastest index ([WALK] forward snippet), so token i sits at
    t = i // (H W), h = (i // W) mod H, w = i mod W.
    """
    i = np.arange(F * H * W, dtype=np.int64)
    return np.stack([i // (H * W), (i // W) % H, i % W], axis=1)


# --------------------------------------------------------------------------
# 3D RoPE ([WALK] "3D RoPE" snippet; [DIFFUSERS] "3D RoPE coordinate system")
# --------------------------------------------------------------------------

def rope_axis_pairs(head_dim: int):
    """Complex pairs given to the (t, h, w) axes: [c - 2(c//3), c//3, c//3],
    c = head_dim / 2 ([WALK] 3D RoPE snippet, the ``split`` of the table)."""
    if head_dim % 2:
        raise ValueError("head_dim must be even")
    c = head_dim // 2
    return (c - 2 * (c // 3), c // 3, c // 3)


def rope_omegas(head_dim: int, theta: float = 1e4) -> np.ndarray:
    """Angular frequency of each complex pair j in [0, head_dim/2), fp64.

    The table is the concatenation of one frequency ladder per axis; an axis
    that owns p pairs (d_a = 2p real dims) has omega_j = theta^(-2j/d_a),
    j = 0..p-1 (the plainest reading of a per-axis precomputed table split as in
    the [WALK] snippet).
    """
    out = []
    for p in rope_axis_pairs(head_dim):
        d_a = 2 * p
        j = np.arange(p, dtype=F64)
        out.append(theta ** (-(2.0 * j) / d_a))
    return np.concatenate(out)


def rope_pair_axis(head_dim: int) -> np.ndarray:
    """Axis (0 = t, 1 = h, 2 = w) that rotates each complex pair."""
    pt, ph, pw = rope_axis_pairs(head_dim)
    return np.concatenate([np.zeros(pt, np.int64), np.ones(ph, np.int64),
                           np.full(pw, 2, np.int64)])


def rope_table(head_dim: int, max_pos: int = 1024, theta: float = 1e4) -> np.ndarray:
    """Precomputed table of (cos, sin) of pos * omega_j, shape
    [max_pos, head_dim/2, 2], fp64 ([WALK]: a 1024-position table computed
    once and sliced per grid)."""
    ang = np.arange(max_pos, dtype=F64)[:, None] * rope_omegas(head_dim, theta)[None, :]
    return np.stack([np.cos(ang), np.sin(ang)], axis=-1)


def rope_apply(x: np.ndarray, grid, theta: float = 1e4,
               positions: np.ndarray | None = None) -> np.ndarray:
    """Rotate q or k ([L, heads, d]) by the 3D RoPE of each token.

    Pair j = (x[2j], x[2j+1]) is read as the complex number x[2j] + i x[2j+1]
    (``view_as_real(...).flatten`` in the [WALK] snippet: interleaved pairs) and is
    multiplied by exp(i * pos_axis(j) * omega_j), where pos_axis(j) is the
    token's t, h or w grid index for the axis that owns pair j.
    """
    L, n, d = x.shape
    if positions is None:
        positions = token_positions(*grid)
    assert positions.shape[0] == L
    pos = positions[:, rope_pair_axis(d)].astype(F64)           # [L, d/2]
    ang = pos * rope_omegas(d, theta)[None, :]                  # [L, d/2]
    c = np.cos(ang)[:, None, :]
    s = np.sin(ang)[:, None, :]
    x = np.asarray(x, F64)
    re = x[..., 0::2]
    im = x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = re * c - im * s
    out[..., 1::2] = re * s + im * c
    return out


# --------------------------------------------------------------------------
# Norms and activation ([WALK] block snippet and structure snippet)
# --------------------------------------------------------------------------

def layer_norm(x: np.ndarray, eps: float, gamma=None, beta=None) -> np.ndarray:
    """LayerNorm over the last axis: (x - mean) / sqrt(var + eps), population
    variance; optional affine gamma, beta (norm3)."""
    x = np.asarray(x, F64)
    mu = x.mean(-1, keepdims=True)
    var = ((x - mu) ** 2).mean(-1, keepdims=True)
    y = (x - mu) / np.sqrt(var + eps)
    if gamma is not None:
        y = y * np.asarray(gamma, F64)
    if beta is not None:
        y = y + np.asarray(beta, F64)
    return y


def rms_norm(x: np.ndarray, gamma, eps: float) -> np.ndarray:
    """RMSNorm over the last axis: x / sqrt(mean(x^2) + eps) * gamma
    (the optional q/k RMSNorm, ``qk_norm`` in the [WALK] structure snippet)."""
    x = np.asarray(x, F64)
    r = 1.0 / np.sqrt((x * x).mean(-1, keepdims=True) + eps)
    return x * r * np.asarray(gamma, F64)


def gelu_tanh(z: np.ndarray) -> np.ndarray:
    """GELU, tanh form (``nn.GELU(approximate="tanh")`` in the [WALK]
    structure snippet): 0.5 z (1 + tanh(sqrt(2/pi) (z + 0.044715 z^3)))."""
    z = np.asarray(z, F64)
    return 0.5 * z * (1.0 + np.tanh(math.sqrt(2.0 / math.pi) * (z + 0.044715 * z ** 3)))


def linear(a: np.ndarray, w: np.ndarray, b) -> np.ndarray:
    """y = a W^T + b with W stored [out, in] (``nn.Linear``)."""
    y = np.asarray(a, F64) @ np.asarray(w, F64).T
    if b is not None:
        y = y + np.asarray(b, F64)
    return y


_linear = linear


# --------------------------------------------------------------------------
# FP8 GEMM ([DIGEST] inference-optimisation table, "FP8 GEMM": per-tensor
# weight quantization, per-token activation quantization for the GEMMs of the
# DiT block). Code layout of e4m3 from the OCP 8-bit floating-point format
# (1 sign, 4 exponent bits with bias 7, 3 mantissa bits; exponent field 15
# with mantissa 7 is NaN, there is no infinity).
# --------------------------------------------------------------------------

E4M3_MAX = 448.0


def e4m3_decode(codes) -> np.ndarray:
    """Value of each e4m3 byte (NaN for 0x7F and 0xFF)."""
    c = np.asarray(codes, np.int64) & 0xFF
    sign = np.where(c >= 128, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 7).astype(F64)
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * 2.0 ** (e.astype(F64) - 7))
    mag = np.where((e == 15) & ((c & 7) == 7), np.nan, mag)
    return sign * mag


def e4m3_round(x) -> np.ndarray:
    """Nearest e4m3 value (ties to the even code), magnitudes above 448 clamped
    to 448. Values are spaced 2^(e-3) within the binade [2^e, 2^(e+1)), e >= -6;
    below 2^-6 the spacing stays 2^-9 (subnormals)."""
    x = np.asarray(x, F64)
    a = np.abs(x)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, -6.0)
    step = 2.0 ** (e - 3.0)
    r = np.round(a / step) * step              # numpy rounds halves to even
    r = np.minimum(r, E4M3_MAX)
    return np.copysign(r, x)


def quantize_fp8(x, per_row: bool = True):
    """(codes as values, scales): per row of the last axis (one scale per
    token) or per tensor. amax, 448 / amax, x * (448 / amax) and amax / 448
    are each rounded to fp32 as they are formed."""
    x32 = np.asarray(x, F64).astype(np.float32)
    if per_row:
        amax = np.abs(x32).max(axis=-1, keepdims=True) if x32.shape[-1] else np.zeros(x32.shape[:-1] + (1,), np.float32)
    else:
        amax = np.array(np.abs(x32).max() if x32.size else 0.0, np.float32)
    amax = amax.astype(np.float32)
    nz = amax > 0
    with np.errstate(divide="ignore"):
        inv = np.where(nz, np.float32(E4M3_MAX) / np.where(nz, amax, np.float32(1)), np.float32(0)).astype(np.float32)
    y = (x32 * inv).astype(np.float32)
    q = e4m3_round(y.astype(F64))
    scale = (amax / np.float32(E4M3_MAX)).astype(np.float32)
    return q, scale.astype(F64)


def linear_fp8(a, w, b) -> np.ndarray:
    """FP8 linear layer: a quantized per row, W per tensor, the product of the
    codes accumulated exactly (fp64), times both scales, plus the bias."""
    qa, sa = quantize_fp8(a, per_row=True)
    qw, sw = quantize_fp8(w, per_row=False)
    y = (qa @ qw.T) * sa * sw
    if b is not None:
        y = y + np.asarray(b, F64)
    return y


# --------------------------------------------------------------------------
# Attention ([WALK] self-attention snippet: global window, no causal mask,
# key lengths)
# --------------------------------------------------------------------------

def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray,
              k_len: int | None = None, scale: float | None = None) -> np.ndarray:
    """Softmax attention of one sequence, every head.

    q [Lq, n, d], k and v [Lk, n, d]; only the first ``k_len`` keys are valid.
    o_i = sum_j softmax_j(q_i . k_j * scale) v_j with scale = 1/sqrt(d)
    (the pages are silent; the usual default). A row with no valid key returns zeros.
    """
    q = np.asarray(q, F64)
    k = np.asarray(k, F64)
    v = np.asarray(v, F64)
    Lq, n, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if k_len is not None:
        k = k[:k_len]
        v = v[:k_len]
    if k.shape[0] == 0:
        return np.zeros((Lq, n, v.shape[2]), F64)
    s = np.einsum("qnd,knd->nqk", q, k) * scale
    s = s - s.max(-1, keepdims=True)
    p = np.exp(s)
    p = p / p.sum(-1, keepdims=True)
    return np.einsum("nqk,knd->qnd", p, v)


# --------------------------------------------------------------------------
# 8-bit attention ([DIGEST] inference-optimisation table, "8-bit
# FlashAttention": int8 for S = Q K^T, FP8 for O = P V, fp32 accumulation).
# The page gives only the types, so this is the plain definition with each
# product's operands quantized: S from int8 q and k (exact integer products
# times the two scales and the logit scale), the softmax probabilities
# p = exp(s - m) with m the exact row max over the valid keys, and O = P V
# with P and V in e4m3. Readings where the page is silent: q is quantized per
# token and head (scale amax / 127 over the head's d values), k per head over
# all keys of the sequence, v to e4m3 per head and channel over all keys (the
# channel scale factors out of P V); P by the FP8 rule of the GEMMs (one
# scale per row = amax / 448, and the row's amax is p = 1 at the max, so the
# codes are e4m3(448 p)); the normaliser sums the unrounded p. int8 codes
# are round-half-even of x * (127 / amax), clamped to +-127, decided in fp32.
# Sums are exact (fp64); no blocking or running max.
# --------------------------------------------------------------------------
I8_MAX = 127.0


def quantize_int8(x, axes):
    """(codes as values, scales) with one scale per slice over ``axes``
    (kept as size-1 axes): amax, 127 / amax, x * (127 / amax) and amax / 127
    each rounded to fp32 as formed; an all-zero slice gets codes 0, scale 0."""
    x32 = np.asarray(x, F64).astype(np.float32)
    amax = np.abs(x32).max(axis=axes, keepdims=True).astype(np.float32)
    nz = amax > 0
    inv = np.where(nz, np.float32(I8_MAX) / np.where(nz, amax, np.float32(1)), np.float32(0)).astype(np.float32)
    y = (x32 * inv).astype(np.float32).astype(F64)
    q = np.clip(np.rint(y), -I8_MAX, I8_MAX)
    return q, (amax / np.float32(I8_MAX)).astype(np.float32).astype(F64)


def quantize_fp8_axes(x, axes):
    """e4m3 codes with one scale per slice over ``axes`` (the rule of
    ``quantize_fp8``)."""
    x32 = np.asarray(x, F64).astype(np.float32)
    amax = np.abs(x32).max(axis=axes, keepdims=True).astype(np.float32)
    nz = amax > 0
    inv = np.where(nz, np.float32(E4M3_MAX) / np.where(nz, amax, np.float32(1)), np.float32(0)).astype(np.float32)
    y = (x32 * inv).astype(np.float32)
    return e4m3_round(y.astype(F64)), (amax / np.float32(E4M3_MAX)).astype(np.float32).astype(F64)


def attention_8bit_terms(q, k, v, k_len: int | None = None, scale: float | None = None):
    """The quantities the 8-bit attention of one sequence is formed from
    (q [Lq, n, d], k, v [Lk, n, d]; the first ``k_len`` keys valid):
    p [n, Lq, kl] = exp(s - rowmax s) over the valid keys, with s the
    quantized logits; l [n, Lq, 1] = sum of p; vq [kl, n, d] the e4m3 codes
    of v and sv [1, n, d] their per-channel scales."""
    q = np.asarray(q, F64)
    k = np.asarray(k, F64)
    v = np.asarray(v, F64)
    Lq, n, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    qi, sq = quantize_int8(q, axes=(2,))           # [Lq, n, 1]
    ki, sk = quantize_int8(k, axes=(0, 2))         # [1, n, 1]
    vq, sv = quantize_fp8_axes(v, axes=(0,))       # [1, n, d]
    kl = k.shape[0] if k_len is None else k_len
    s = np.einsum("qnd,knd->nqk", qi, ki[:kl]) * (np.transpose(sq, (1, 0, 2)) * sk[0][:, :, None] * scale)
    if kl == 0:
        return np.zeros((n, Lq, 0)), np.zeros((n, Lq, 1)), vq[:0], sv
    p = np.exp(s - s.max(-1, keepdims=True))
    return p, p.sum(-1, keepdims=True), vq[:kl], sv


def attention_8bit(q, k, v, k_len: int | None = None, scale: float | None = None) -> np.ndarray:
    """8-bit softmax attention of one sequence (q [Lq, n, d], k, v [Lk, n, d];
    the first ``k_len`` keys valid): o = (sum_j e4m3(448 p_j) / 448 vq_j) / l
    times the channel scales of v. A row with no valid key returns zeros."""
    Lq, n, d = np.shape(q)
    p, l, vq, sv = attention_8bit_terms(q, k, v, k_len, scale)
    if p.shape[2] == 0:
        return np.zeros((Lq, n, d), F64)
    pq = e4m3_round(p * E4M3_MAX) / E4M3_MAX
    o = np.einsum("nqk,knd->nqd", pq, vq) / l
    return np.transpose(o, (1, 0, 2)) * sv


# --------------------------------------------------------------------------
# The block ([WALK] WanAttentionBlock core-logic snippet; [DIGEST] shared
# AdaLN MLP + per-block bias)
# --------------------------------------------------------------------------

BLOCK_WEIGHT_NAMES = (
    "modulation",
    "wq", "bq", "wk", "bk", "wv", "bv", "wo", "bo", "gq", "gk",
    "g3", "b3",
    "cwq", "cbq", "cwk", "cbk", "cwv", "cbv", "cwo", "cbo", "cgq", "cgk",
    "w1", "b1", "w2", "b2",
)


def block_param_count(dim: int, ffn_dim: int, biases: bool = True) -> int:
    """Parameters of one block under this reading: four dim x dim projections
    in each attention, two FFN matrices, their biases, the q/k gains, the
    norm3 affine and the 6 x dim modulation bias."""
    n = 8 * dim * dim + 2 * dim * ffn_dim
    if biases:
        n += 8 * dim + ffn_dim + dim          # attention + FFN biases
        n += 4 * dim + 2 * dim + 6 * dim      # q/k gains, norm3 affine, modulation
    return n


def _mod(w, e0):
    """e = (modulation + e0).chunk(6): shift, scale, gate, shift2, scale2,
    gate2. e0 is [B, 6, D] (one timestep per sequence) or [B, L, 6, D] (one
    per token: [WALK] time-projection snippet, ``unflatten(0, (bt, seq_len))``)."""
    e0 = np.asarray(e0, F64)
    mod = np.asarray(w["modulation"], F64)
    return (mod[None] if e0.ndim == 3 else mod[None, None]) + e0


def _chunk(m, k, b=None, rows=None):
    """Chunk k of the modulation for every row: [B, L or 1, D] (b None) or
    [R or 1, D] for sequence b at ``rows``."""
    if m.ndim == 3:                                   # per sequence
        return m[:, k, None, :] if b is None else m[b, k][None]
    return m[:, :, k, :] if b is None else m[b, rows, k]


def self_attn_kv(x, e0, w, heads, grid, eps, theta=1e4, fp8=False):
    """K (RMSNorm'd, rotated) and V of the self-attention for every row of
    every sequence: [B, L, n, d] each. Rows interact only through these.
    ``fp8``: the projections are FP8 linear layers."""
    linear = linear_fp8 if fp8 else _linear
    x = np.asarray(x, F64)
    B, L, D = x.shape
    d = D // heads
    m = _mod(w, e0)
    u = layer_norm(x, eps) * (1.0 + _chunk(m, 1)) + _chunk(m, 0)
    k = rms_norm(linear(u, w["wk"], w["bk"]), w["gk"], eps).reshape(B, L, heads, d)
    v = linear(u, w["wv"], w["bv"]).reshape(B, L, heads, d)
    k = np.stack([rope_apply(k[b], grid, theta) for b in range(B)])
    return k, v


def block_forward_rows(x, ctx, ctx_lens, e0, w, heads, grid, eps, rows,
                       theta=1e4, kv=None, intermediates=None, fp8=False, attn8=False):
    """Output of one WanAttentionBlock at the token rows ``rows`` of every
    sequence: [B, len(rows), D]. Follows the [WALK] block snippet:

        m = modulation + e0                        (shift, scale, gate, x2)
        x += m2 * SelfAttn(LN(x) (1 + m1) + m0)
        x += CrossAttn(LN_affine3(x), ctx)          (no gate, no modulation)
        x += m5 * FFN(LN(x) (1 + m4) + m3)

    SelfAttn: q, k = RMSNorm(Linear(u)), v = Linear(u); q, k rotated by the
    3D RoPE; full softmax attention over all L tokens; output Linear.
    CrossAttn: same without RoPE; keys/values from ctx, first ctx_lens[b] valid.
    FFN: Linear, GELU-tanh, Linear.

    Self-attention K and V need every row; everything else is row-local, so
    only the requested rows are carried past the key/value projection.
    ``intermediates`` (a dict) receives the per-branch outputs at those rows.
    ``fp8``: the ten projections (q, k, v, o, cross q, k, v, o, FFN 1 and 2)
    are FP8 linear layers (``linear_fp8``); everything else is unchanged.
    ``attn8``: the self-attention is the 8-bit attention (``attention_8bit``).
    """
    linear = linear_fp8 if fp8 else _linear
    x = np.asarray(x, F64)
    ctx = np.asarray(ctx, F64)
    B, L, D = x.shape
    T = ctx.shape[1]
    d = D // heads
    rows = np.asarray(rows, np.int64)
    m = _mod(w, e0)
    if kv is None:
        kv = self_attn_kv(x, e0, w, heads, grid, eps, theta, fp8=fp8)
    k_all, v_all = kv
    pos = token_positions(*grid)[rows]

    xr = x[:, rows, :].copy()                                    # [B, R, D]
    R = rows.shape[0]
    inter = {"o_self": [], "y_self": [], "o_cross": [], "y_cross": [], "y_ffn": [], "h": []}
    out = np.empty_like(xr)
    for b in range(B):
        xb = xr[b]
        # self-attention branch
        u = layer_norm(xb, eps) * (1.0 + _chunk(m, 1, b, rows)) + _chunk(m, 0, b, rows)
        q = rms_norm(linear(u, w["wq"], w["bq"]), w["gq"], eps).reshape(R, heads, d)
        q = rope_apply(q, grid, theta, positions=pos)
        o = (attention_8bit if attn8 else attention)(q, k_all[b], v_all[b]).reshape(R, D)
        y = linear(o, w["wo"], w["bo"])
        xb = xb + y * _chunk(m, 2, b, rows)
        inter["o_self"].append(o)
        inter["y_self"].append(y)
        # cross-attention branch
        a3 = layer_norm(xb, eps, w["g3"], w["b3"])
        qc = rms_norm(linear(a3, w["cwq"], w["cbq"]), w["cgq"], eps).reshape(R, heads, d)
        kc = rms_norm(linear(ctx[b], w["cwk"], w["cbk"]), w["cgk"], eps).reshape(T, heads, d)
        vc = linear(ctx[b], w["cwv"], w["cbv"]).reshape(T, heads, d)
        klen = T if ctx_lens is None else int(ctx_lens[b])
        oc = attention(qc, kc, vc, k_len=klen).reshape(R, D)
        yc = linear(oc, w["cwo"], w["cbo"])
        xb = xb + yc
        inter["o_cross"].append(oc)
        inter["y_cross"].append(yc)
        # FFN branch
        a2 = layer_norm(xb, eps) * (1.0 + _chunk(m, 4, b, rows)) + _chunk(m, 3, b, rows)
        h = gelu_tanh(linear(a2, w["w1"], w["b1"]))
        yf = linear(h, w["w2"], w["b2"])
        xb = xb + yf * _chunk(m, 5, b, rows)
        inter["h"].append(h)
        inter["y_ffn"].append(yf)
        out[b] = xb
    if intermediates is not None:
        for key, val in inter.items():
            intermediates[key] = np.stack(val)
    return out


def block_forward(x, ctx, ctx_lens, e0, w, heads, grid, eps, theta=1e4,
                  intermediates=None, fp8=False, attn8=False):
    """Full block output [B, L, D] (all rows)."""
    L = np.asarray(x).shape[1]
    return block_forward_rows(x, ctx, ctx_lens, e0, w, heads, grid, eps,
                              np.arange(L), theta=theta, intermediates=intermediates, fp8=fp8,
                              attn8=attn8)


# --------------------------------------------------------------------------
# CFG + flow-matching Euler step ([WALK] sampling-loop snippet; [DIGEST]
# "Video DiT and Flow Matching")
# --------------------------------------------------------------------------

def cfg_combine(v_cond, v_uncond, guide_scale: float):
    """v = v_u + s (v_c - v_u); without an unconditional branch v = v_c."""
    v_cond = np.asarray(v_cond, F64)
    if v_uncond is None:
        return v_cond
    v_uncond = np.asarray(v_uncond, F64)
    return v_uncond + guide_scale * (v_cond - v_uncond)


def euler_cfg_step(x, v_cond, v_uncond, guide_scale: float,
                   sigma: float, sigma_next: float):
    """One explicit Euler step of the flow ODE in sigma: x + (sigma' - sigma) v."""
    return np.asarray(x, F64) + (sigma_next - sigma) * cfg_combine(v_cond, v_uncond, guide_scale)


def denoise_step(x_tokens, ctx_cond, ctx_uncond, ctx_lens, e0, blocks, heads, grid,
                 eps, guide_scale, sigma, sigma_next, theta=1e4):
    """One denoising step on the token stream: the block stack runs on the
    same x for the conditional and the unconditional context, the two outputs
    are combined by CFG and the Euler step moves x (there is no patch
    embedding or head on this path)."""
    x_tokens = np.asarray(x_tokens, F64)
    xb = np.stack([x_tokens, x_tokens])
    ctx = np.stack([np.asarray(ctx_cond, F64), np.asarray(ctx_uncond, F64)])
    e = np.stack([np.asarray(e0, F64)] * 2) if np.asarray(e0).ndim == 2 else np.asarray(e0, F64)
    for w in blocks:
        xb = block_forward(xb, ctx, ctx_lens, e, w, heads, grid, eps, theta)
    return euler_cfg_step(x_tokens, xb[0], xb[1], guide_scale, sigma, sigma_next)


# --------------------------------------------------------------------------
# Whole-model step on latents ([WALK] structure, forward and time-projection
# snippets, MoE expert-switch and sampling-loop snippets; [DIFFUSERS]
# "3D Patchify" and "Unpatchify"; [TRACE] section 4 "DIT").
#
# Readings taken where the pages are silent:
# * freq_dim = 256 and the sinusoidal embedding of t is [cos(t w_j), sin(t w_j)],
#   w_j = 10000^(-j / (freq_dim/2)), j < freq_dim/2.
# * The head (``Head(dim, out_dim, patch_size, eps)`` called as head(x, e))
#   is LayerNorm without affine, modulated like the block's AdaLN by two
#   chunks (shift, scale) of (head_modulation + e), then Linear(dim ->
#   out_dim * 1*2*2); e is the time embedding before the 6 x dim projection.
# * Patch embedding weight [dim, C, 1, 2, 2] (Conv3d); a token's input
#   features are ordered (c, kt, kh, kw) like the flattened weight.
# * The head's out_dim*4 features of a token are ordered (kt, kh, kw, c),
#   channel fastest, when folded back into [C, F, 2H, 2W].
# * The denoiser is called at timestep t = 1000 * sigma.
# --------------------------------------------------------------------------

MODEL_WEIGHT_NAMES = ("patch_w", "patch_b", "text_w1", "text_b1", "text_w2", "text_b2",
                      "time_w1", "time_b1", "time_w2", "time_b2", "proj_w", "proj_b",
                      "head_mod", "head_w", "head_b")


def sinusoidal_embedding(freq_dim: int, t) -> np.ndarray:
    """[B, freq_dim]: cos then sin of t * 10000^(-j/half), j < half."""
    t = np.asarray(t, F64).reshape(-1)
    half = freq_dim // 2
    w = 10000.0 ** (-np.arange(half, dtype=F64) / half)
    a = t[:, None] * w[None, :]
    return np.concatenate([np.cos(a), np.sin(a)], axis=1)


def silu(z):
    z = np.asarray(z, F64)
    return z / (1.0 + np.exp(-z))


def time_embed(t, mw, freq_dim=256):
    """e = Linear(SiLU(Linear(sinusoid(t)))) and e0 = Linear(SiLU(e)) as
    [B, 6, dim] ([WALK] structure and time-projection snippets)."""
    shape = np.shape(t)                                # [B] or [B, L] (one timestep per token)
    s = sinusoidal_embedding(freq_dim, t)
    e = linear(silu(linear(s, mw["time_w1"], mw["time_b1"])), mw["time_w2"], mw["time_b2"])
    e0 = linear(silu(e), mw["proj_w"], mw["proj_b"])
    return e.reshape(shape + (-1,)), e0.reshape(shape + (6, -1))


def text_embed(ctx_raw, mw):
    """Linear(4096 -> dim), GELU-tanh, Linear(dim -> dim) per text token."""
    return linear(gelu_tanh(linear(ctx_raw, mw["text_w1"], mw["text_b1"])), mw["text_w2"], mw["text_b2"])


def patchify(latent):
    """[B, C, F, H, W] -> tokens [B, F*(H/2)*(W/2), C*4], token order (f, h, w),
    features (c, kh, kw) with kt = 0 (the (1, 2, 2) Conv3d's receptive field)."""
    x = np.asarray(latent, F64)
    B, C, F, H, W = x.shape
    x = x.reshape(B, C, F, H // 2, 2, W // 2, 2)          # b c f h kh w kw
    x = x.transpose(0, 2, 3, 5, 1, 4, 6)                  # b f h w c kh kw
    return x.reshape(B, F * (H // 2) * (W // 2), C * 4)


def patch_embed(latent, mw):
    """Conv3d(C, dim, kernel (1,2,2), stride (1,2,2)) flattened to tokens."""
    dim = np.asarray(mw["patch_w"]).shape[0]
    return linear(patchify(latent), np.asarray(mw["patch_w"], F64).reshape(dim, -1), mw["patch_b"])


def head(x, e, mw, eps):
    """LN(x) (1 + m1) + m0 with m = head_modulation + e, then Linear; e is
    [B, dim] or, with per-token timesteps, [B, L, dim]."""
    e = np.asarray(e, F64)
    hm = np.asarray(mw["head_mod"], F64)
    if e.ndim == 2:
        m0, m1 = (hm[0][None] + e)[:, None, :], (hm[1][None] + e)[:, None, :]
    else:
        m0, m1 = hm[0] + e, hm[1] + e
    u = layer_norm(x, eps) * (1.0 + m1) + m0
    return linear(u, mw["head_w"], mw["head_b"])


def unpatchify(tokens, grid, channels):
    """tokens [B, L, 4*C] (features (kt, kh, kw, c)) -> [B, C, F, 2H, 2W]."""
    F, H, W = grid
    t = np.asarray(tokens, F64)
    B = t.shape[0]
    t = t.reshape(B, F, H, W, 1, 2, 2, channels)           # b f h w kt kh kw c
    t = t.transpose(0, 7, 1, 4, 2, 5, 3, 6)                # b c f kt h kh w kw
    return t.reshape(B, channels, F, 2 * H, 2 * W)


def model_forward(latent, t, ctx_raw, ctx_lens, mw, blocks, heads, eps, theta=1e4, freq_dim=256):
    """WanModel forward on latents ([WALK] forward snippet): patch embedding,
    flatten, time and text embeddings, the block stack, head, unpatchify.
    t is [B] or [B, L] (a timestep per token, L = F (H/2) (W/2))."""
    latent = np.asarray(latent, F64)
    B, C, Fl, Hl, Wl = latent.shape
    grid = (Fl, Hl // 2, Wl // 2)
    x = patch_embed(latent, mw)
    e, e0 = time_embed(t, mw, freq_dim)
    ctx = text_embed(ctx_raw, mw)
    for w in blocks:
        x = block_forward(x, ctx, ctx_lens, e0, w, heads, grid, eps, theta)
    out_c = np.asarray(mw["head_w"]).shape[0] // 4
    return unpatchify(head(x, e, mw, eps), grid, out_c)


def select_expert(t: float, boundary: float) -> str:
    """Two-expert switch ([WALK] MoE snippet): the high-noise model when
    t >= boundary (boundary = 0.875 * 1000 for T2V, 900 for I2V)."""
    return "high" if t >= boundary else "low"


def model_denoise_step(latent, sigma, sigma_next, ctx_cond, ctx_uncond, mw, blocks, heads, eps,
                       guide_scale, theta=1e4, freq_dim=256):
    """One CFG flow-matching Euler step on the latent: the model runs on the
    same latent at t = 1000 sigma for both contexts, v = v_u + s (v_c - v_u),
    latent + (sigma' - sigma) v."""
    latent = np.asarray(latent, F64)
    lat2 = np.stack([latent, latent])
    ctx = np.stack([np.asarray(ctx_cond, F64), np.asarray(ctx_uncond, F64)])
    t = np.array([1000.0 * sigma] * 2)
    v = model_forward(lat2, t, ctx, None, mw, blocks, heads, eps, theta, freq_dim)
    return euler_cfg_step(latent, v[0], v[1], guide_scale, sigma, sigma_next)


# --------------------------------------------------------------------------
# UniPC multistep sampler ("Wan2.2 I2V inference trace" (damodev.csdn.net),
# section 4 "DIT": the latent update "UniPC: x_noise <- step(v, t, x_noise)";
# "Wan architecture overview", scheduler: Euler or UniPC multistep). The pages
# name the method only; its steps follow the UniPC paper (Zhao et al., 2023,
# "UniPC: A Unified Predictor-Corrector Framework for Fast Sampling of
# Diffusion Models"): the data-prediction form, B(h) = e^h - 1 ("bh2"),
# predictor UniP-p and corrector UniC-p sharing one model evaluation per step.
# Readings: flow matching x = (1 - sigma) x0 + sigma eps gives alpha = 1 - sigma
# and the data prediction x0 = x - sigma v; lambda = log(alpha / sigma);
# order 2 with one first-order warm-up step and a first-order final step;
# the schedule's first sigma is below 1 and its last is 0.
# --------------------------------------------------------------------------

def flow_lambda(sigma: float) -> float:
    """log(alpha / sigma) with alpha = 1 - sigma (+inf at sigma = 0)."""
    if sigma == 0.0:
        return math.inf
    return math.log(1.0 - sigma) - math.log(sigma)


def _unipc_phis(h: float, order: int):
    """h_phi_1, B(h) and the right-hand side b of the order conditions
    (data prediction: hh = -h)."""
    hh = -h
    h_phi_1 = math.expm1(hh)
    B_h = math.expm1(hh)
    h_phi_k = h_phi_1 / hh - 1.0
    b, fact = [], 1.0
    for j in range(1, order + 1):
        b.append(h_phi_k * fact / B_h)
        fact *= j + 1
        h_phi_k = h_phi_k / hh - 1.0 / fact
    return h_phi_1, B_h, np.array(b)


def unipc_predict(x, m_hist, sigmas, i: int, order: int):
    """UniP-p from sigma_i to sigma_{i+1}: m_hist[-1] is m_i (at sigma_i),
    m_hist[-1-k] the output k steps earlier."""
    s0, t = sigmas[i], sigmas[i + 1]
    lam_s0, lam_t = flow_lambda(s0), flow_lambda(t)
    h = lam_t - lam_s0
    m0 = np.asarray(m_hist[-1], F64)
    h_phi_1, B_h, b = _unipc_phis(h, order)
    x_t = (t / s0) * np.asarray(x, F64) - (1.0 - t) * h_phi_1 * m0
    if order >= 2:
        rks = np.array([(flow_lambda(sigmas[i - k]) - lam_s0) / h for k in range(1, order)])
        D1s = [(np.asarray(m_hist[-1 - k], F64) - m0) / rks[k - 1] for k in range(1, order)]
        if order == 2:
            rho = np.array([0.5])
        else:
            R = np.stack([np.append(rks, 1.0) ** (j - 1) for j in range(1, order + 1)])
            rho = np.linalg.solve(R[:-1, :-1], b[:-1])
        x_t = x_t - (1.0 - t) * B_h * sum(r * d for r, d in zip(rho, D1s))
    return x_t


def unipc_correct(last, m_hist, m_new, sigmas, i: int, order: int):
    """UniC-p at sigma_i: refines the sample reached from sigma_{i-1} (whose
    corrected value is ``last``) with the new output m_new at sigma_i;
    m_hist[-1] is the output at sigma_{i-1}, m_hist[-1-k] k steps earlier."""
    s0, t = sigmas[i - 1], sigmas[i]
    lam_s0, lam_t = flow_lambda(s0), flow_lambda(t)
    h = lam_t - lam_s0
    m0 = np.asarray(m_hist[-1], F64)
    h_phi_1, B_h, b = _unipc_phis(h, order)
    rks = np.array([(flow_lambda(sigmas[i - 1 - k]) - lam_s0) / h for k in range(1, order)] + [1.0])
    D1s = [(np.asarray(m_hist[-1 - k], F64) - m0) / rks[k - 1] for k in range(1, order)]
    if order == 1:
        rho = np.array([0.5])
    else:
        R = np.stack([rks ** (j - 1) for j in range(1, order + 1)])
        rho = np.linalg.solve(R, b)
    x_t = (t / s0) * np.asarray(last, F64) - (1.0 - t) * h_phi_1 * m0
    corr = sum(r * d for r, d in zip(rho[:-1], D1s))
    return x_t - (1.0 - t) * B_h * (corr + rho[-1] * (np.asarray(m_new, F64) - m0))


def unipc_sample(x, velocity, sigmas, order: int = 2, corrector: bool = True,
                 lower_order_final: bool = True):
    """Run the sampler from sigmas[0] to sigmas[-1] = 0 with one evaluation of
    ``velocity(x, sigma, i)`` per step (i = 0 .. len(sigmas) - 2). Returns the
    final sample and the list of samples handed to the evaluations.
    ``corrector`` False leaves out UniC; ``lower_order_final`` False keeps the
    full order on the last step."""
    sigmas = [float(s) for s in sigmas]
    n = len(sigmas) - 1
    x = np.asarray(x, F64)
    m_hist, last, prev_order, seen = [], None, 0, []
    for i in range(n):
        seen.append(x)
        m = x - sigmas[i] * np.asarray(velocity(x, sigmas[i], i), F64)   # data prediction
        if i > 0 and corrector:
            x = unipc_correct(last, m_hist, m, sigmas, i, prev_order)
        m_hist = (m_hist + [m])[-order:]
        this_order = min(order, n - i if lower_order_final else order, i + 1)   # warm-up, final step
        last = x
        x = unipc_predict(x, m_hist, sigmas, i, this_order)
        prev_order = this_order
    return x, seen


def flow_sigmas(num_steps: int, shift: float = 5.0, sigma_max: float = 0.999) -> np.ndarray:
    """A flow-matching schedule: num_steps values from sigma_max down to
    1 / num_steps of it, time-shifted sigma -> s sigma / (1 + (s - 1) sigma),
    then the final 0."""
    base = np.linspace(sigma_max, sigma_max / num_steps, num_steps)
    shifted = shift * base / (1.0 + (shift - 1.0) * base)
    return np.append(shifted, 0.0)
