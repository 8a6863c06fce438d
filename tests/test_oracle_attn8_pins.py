"""Pins of the oracle's 8-bit attention ("Wan paper deep dive",
inference-optimisation table, "8-bit FlashAttention": int8 S = Q K^T, FP8
O = P V): the int8 quantizer's invariants, exactness when every
quantization step is the identity, P relative to the exact row max, no
dependence on key order, how each scale enters, and the size of the
approximation."""
import math

import numpy as np

from oracle import wan_oracle as O


def test_quantize_int8_rules():
    x = np.array([[127.0, 63.5, -0.5, 1.5, 2.5, -126.5, 0.0, 3.0]])
    q, s = O.quantize_int8(x, axes=(1,))
    assert s[0, 0] == 1.0                                    # 127 / 127
    assert np.array_equal(q[0], [127, 64, -0.0, 2, 2, -126, 0, 3])   # halves to even
    rng = np.random.default_rng(0)
    y = rng.standard_normal((6, 40)) * np.exp(rng.standard_normal((6, 1)) * 4)
    y[2] = 0.0
    q, s = O.quantize_int8(y, axes=(1,))
    assert not q[2].any() and s[2, 0] == 0.0
    for r in (0, 1, 3, 4, 5):
        assert np.abs(q[r]).max() == 127.0
        assert np.array_equal(q[r], np.rint(q[r])) and np.abs(q[r]).max() <= 127
        assert np.abs(q[r] * s[r, 0] - y[r]).max() <= 0.5 * s[r, 0] * (1 + 1e-6)
    # a scale shared over several axes
    q, s = O.quantize_int8(rng.standard_normal((5, 3, 8)), axes=(0, 2))
    assert s.shape == (1, 3, 1)


def _exact_case(n=2, Lq=12, Lk=300, d=128, seed=1):
    """Inputs whose int8 / e4m3 quantization is exact (every scale is 1) and
    whose logits with scale ln 2 are small integers, so exp(s - max) is a
    power of two that e4m3 holds exactly."""
    rng = np.random.default_rng(seed)
    q = np.zeros((Lq, n, d))
    k = np.zeros((Lk, n, d))
    q[:, :, 0] = 127.0                       # each (token, head) amax = 127
    k[0, :, 1] = 127.0                       # each head's key amax = 127
    for arr, L in ((q, Lq), (k, Lk)):
        for t in range(L):
            for h in range(n):
                idx = rng.choice(np.arange(2, d), size=3, replace=False)
                arr[t, h, idx] = rng.choice([-1.0, 1.0], size=3)
    vals = O.e4m3_decode(np.arange(0x7F))
    v = rng.choice(np.concatenate([vals, -vals]), size=(Lk, n, d))
    v[0] = 448.0                              # each (head, channel) amax = 448
    return q, k, v


def test_attention_8bit_exact_when_quantization_is_identity():
    q, k, v = _exact_case()
    ln2 = math.log(2.0)
    got = O.attention_8bit(q, k, v, scale=ln2)
    ref = O.attention(q, k, v, scale=ln2)
    assert np.abs(got - ref).max() <= 1e-12 * np.abs(ref).max()
    for kl in (17, 128, 129, 255):
        got = O.attention_8bit(q, k, v, k_len=kl, scale=ln2)
        ref = O.attention(q, k, v, k_len=kl, scale=ln2)
        assert np.abs(got - ref).max() <= 1e-12 * np.abs(ref).max()


def test_attention_8bit_p_is_relative_to_the_exact_row_max():
    """P is exp(s - m) with m the row's exact maximum, quantized as 448 p:
    the probability at the max is exactly 1 (code 448), so a single valid key
    returns that key's dequantized value exactly, and a key whose logit is
    ln(2) * j below the max carries weight 2^-j exactly while 448 * 2^-j is
    an e4m3 value (j <= 15)."""
    rng = np.random.default_rng(4)
    q, k, v = (rng.standard_normal((9, 2, 128)) for _ in range(3))
    vq, sv = O.quantize_fp8_axes(v, axes=(0,))
    one = O.attention_8bit(q, k, v, k_len=1)
    assert np.array_equal(one, np.broadcast_to(vq[0] * sv[0], one.shape))
    # two keys: logits 0 and -j ln 2 exactly (int8 codes, scale ln 2)
    for j in (1, 5, 15):
        qq = np.zeros((1, 1, 128))
        kk = np.zeros((2, 1, 128))
        qq[0, 0, 0] = 127.0
        kk[0, 0, 1] = 127.0                  # logit 0 (orthogonal), amax of k = 127
        kk[1, 0, 0] = -float(j)              # logit -127 j: with scale ln2 / 127, -j ln 2
        vv = np.zeros((2, 1, 128))
        vv[0, 0, :] = 448.0
        vv[1, 0, :] = -448.0
        got = O.attention_8bit(qq, kk, vv, scale=math.log(2.0) / 127.0)
        w = 2.0 ** -j
        assert np.abs(got - (1.0 - w) / (1.0 + w) * 448.0).max() <= 1e-12 * 448.0


def test_attention_8bit_is_invariant_to_key_order():
    """No blocking and no running max: permuting the keys (with their values)
    leaves every output unchanged up to fp64 summation order."""
    rng = np.random.default_rng(5)
    q = rng.standard_normal((16, 2, 128)) * 3.0
    k = rng.standard_normal((700, 2, 128)) * 3.0
    v = rng.standard_normal((700, 2, 128))
    perm = rng.permutation(700)
    a = O.attention_8bit(q, k, v)
    b = O.attention_8bit(q, k[perm], v[perm])
    assert np.abs(a - b).max() <= 1e-12 * np.abs(a).max()


def test_attention_8bit_scales_enter_where_they_should():
    rng = np.random.default_rng(2)
    q, k, v = (rng.standard_normal((20, 2, 128)) for _ in range(3))
    k, v = np.concatenate([k, rng.standard_normal((30, 2, 128))]), np.concatenate([v, rng.standard_normal((30, 2, 128))])
    base = O.attention_8bit(q, k, v)
    # a power of two on one v channel scales that output channel exactly
    v2 = v.copy()
    v2[:, 1, 7] *= 2.0 ** 5
    o2 = O.attention_8bit(q, k, v2)
    assert np.array_equal(o2[:, 1, 7], base[:, 1, 7] * 2.0 ** 5)
    mask = np.ones(base.shape, bool)
    mask[:, 1, 7] = False
    assert np.array_equal(o2[mask], base[mask])
    # q and k scales multiply: 2^a on q, 2^-a on k leaves everything unchanged
    assert np.array_equal(O.attention_8bit(q * 8.0, k / 8.0, v), base)
    # the logit scale and a power of two on q trade places
    assert np.allclose(O.attention_8bit(q * 2.0, k, v, scale=0.5 / math.sqrt(128)), base, rtol=0, atol=1e-13)


def test_attention_8bit_approximates_attention():
    rng = np.random.default_rng(3)
    q, k, v = rng.standard_normal((64, 2, 128)), rng.standard_normal((256, 2, 128)), rng.standard_normal((256, 2, 128))
    ref = O.attention(q, k, v)
    err = np.linalg.norm(O.attention_8bit(q, k, v) - ref) / np.linalg.norm(ref)
    assert 1e-3 < err < 0.08
    assert not O.attention_8bit(q, k, v, k_len=0).any()
    # the only approximations are the quantizers: with P unrounded (the terms'
    # p) the result is attention over the int8 / e4m3 inputs exactly
    p, l, vq, sv = O.attention_8bit_terms(q, k, v)
    qi, sq = O.quantize_int8(q, axes=(2,))
    ki, sk = O.quantize_int8(k, axes=(0, 2))
    deq = O.attention(qi * sq, ki * sk, vq * sv)
    unrounded = np.transpose(np.einsum("nqk,knd->nqd", p, vq) / l, (1, 0, 2)) * sv
    assert np.abs(unrounded - deq).max() <= 1e-12 * np.abs(deq).max()


def test_block_with_8bit_attention_close_to_fp8_block():
    from video_diffusion_transformer_fwd_b200 import synth
    D, Fh, heads, grid = 256, 512, 2, (2, 3, 4)
    w = {k: v.double().numpy() for k, v in synth.block_weights(D, Fh, "f32", seed=3).items()}
    acts = synth.block_activations(1, 24, D, 5, "f32", seed=9)
    x, ctx, e0 = (acts[k].double().numpy() for k in ("x", "ctx", "e0"))
    inter8, inter = {}, {}
    y8 = O.block_forward(x, ctx, None, e0, w, heads, grid, 1e-6, fp8=True, attn8=True, intermediates=inter8)
    y = O.block_forward(x, ctx, None, e0, w, heads, grid, 1e-6, fp8=True, intermediates=inter)
    d_o = np.linalg.norm(inter8["o_self"] - inter["o_self"]) / np.linalg.norm(inter["o_self"])
    assert 1e-3 < d_o < 0.1
    assert np.linalg.norm(y8 - y) / np.linalg.norm(y - x) < 0.1
