"""Pins of the oracle's FP8 GEMM ("Wan paper deep dive", inference-optimisation
table, "FP8 GEMM": per-tensor weight and per-token activation quantization):
the e4m3 code table against its bit layout and an independent library cast,
rounding ties, saturation, the quantizer's invariants, and the FP8 linear
layer against the exact linear layer where quantization is the identity."""
import math

import numpy as np
import pytest
import torch

from oracle import wan_oracle as O


def test_e4m3_decode_fixed_codes():
    d = O.e4m3_decode
    assert d(0x00) == 0.0 and math.copysign(1.0, d(0x80)) == -1.0
    assert d(0x01) == 2.0 ** -9                      # smallest subnormal
    assert d(0x07) == 7 * 2.0 ** -9                  # largest subnormal
    assert d(0x08) == 2.0 ** -6                      # smallest normal
    assert d(0x38) == 1.0 and d(0x40) == 2.0 and d(0x3C) == 1.5
    assert d(0x7E) == 448.0 and d(0xFE) == -448.0
    assert math.isnan(d(0x7F)) and math.isnan(d(0xFF))
    assert d(0x77) == 240.0                          # exponent field 14: 1.875 * 2^7


def test_e4m3_decode_matches_library_cast():
    codes = np.arange(256)
    ours = O.e4m3_decode(codes)
    lib = torch.tensor(codes, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(ours), np.isnan(lib))
    ok = ~np.isnan(ours)
    assert np.array_equal(ours[ok], lib[ok])
    # 254 finite values (two NaN codes), 253 distinct (+0 and -0)
    assert ok.sum() == 254 and np.unique(ours[ok]).size == 253


def _finite_values():
    v = O.e4m3_decode(np.arange(128))
    return np.unique(v[~np.isnan(v)])               # 0 .. 448, ascending


def test_e4m3_round_fixed_points_ties_and_saturation():
    v = _finite_values()
    assert np.array_equal(O.e4m3_round(v), v)
    assert np.array_equal(O.e4m3_round(-v), -v)
    # midpoints between neighbours go to the neighbour with the even code
    lo, hi = v[:-1], v[1:]
    mid = (lo + hi) / 2
    r = O.e4m3_round(mid)
    code_of = {float(x): i for i, x in enumerate(O.e4m3_decode(np.arange(127)))}
    even = np.array([lo[i] if code_of[float(lo[i])] % 2 == 0 else hi[i] for i in range(mid.size)])
    assert np.array_equal(r, even)
    # just off the midpoint: nearest
    eps = (hi - lo) * 1e-3
    assert np.array_equal(O.e4m3_round(mid - eps), lo)
    assert np.array_equal(O.e4m3_round(mid + eps), hi)
    # saturation
    assert np.array_equal(O.e4m3_round([449.0, 464.0, 1e6, -1e30]), [448.0, 448.0, 448.0, -448.0])


def test_e4m3_round_matches_library_cast_in_range():
    x = np.random.default_rng(0).standard_normal(200000).astype(np.float32)
    x = x * np.float32(2.0) ** np.random.default_rng(1).integers(-12, 8, x.size).astype(np.float32)
    x = x[np.abs(x) <= 448]
    lib = torch.tensor(x).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(O.e4m3_round(x), lib)


def test_quantize_rows_invariants():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((7, 300)) * np.exp(rng.standard_normal((7, 1)) * 3)
    x[3] = 0.0
    q, s = O.quantize_fp8(x, per_row=True)
    assert q.shape == x.shape and s.shape == (7, 1)
    assert s[3, 0] == 0.0 and not q[3].any()
    for r in (0, 1, 2, 4, 5, 6):
        a = np.abs(np.float32(x[r])).max()
        assert s[r, 0] == np.float32(a) / np.float32(448)
        assert np.abs(q[r]).max() == 448.0           # the row's max-abs element lands on 448
        # every code is an e4m3 value and the dequantized error is at most half a step
        assert np.array_equal(O.e4m3_round(q[r]), q[r])
        deq = q[r] * s[r, 0]
        rel = np.abs(deq - x[r]) / np.maximum(np.abs(x[r]), 2.0 ** -6 * s[r, 0])
        assert rel.max() <= 2.0 ** -4 * 1.0001


def test_quantize_power_of_two_scaling_and_per_tensor():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((5, 64))
    q, s = O.quantize_fp8(x)
    q2, s2 = O.quantize_fp8(x * 2.0 ** 5)
    assert np.array_equal(q, q2) and np.array_equal(s2, s * 2.0 ** 5)
    qt, st = O.quantize_fp8(x, per_row=False)
    assert np.ndim(st) == 0 and st == np.float32(np.abs(np.float32(x)).max()) / np.float32(448)
    row = int(np.argmax(np.abs(x).max(1)))
    assert np.array_equal(qt[row], q[row])           # the row holding the tensor's amax


def test_linear_fp8_is_exact_when_quantization_is_identity():
    rng = np.random.default_rng(4)
    v = _finite_values()
    a = rng.choice(np.concatenate([v, -v]), size=(6, 128))
    a[:, 0] = 448.0                                  # every row's amax is 448: scale 1
    w = rng.choice(np.concatenate([v, -v]), size=(40, 128))
    w[0, 0] = -448.0                                 # the tensor's amax is 448
    b = rng.standard_normal(40)
    assert np.array_equal(O.linear_fp8(a, w, b), O.linear(a, w, b))


def test_linear_fp8_scales_follow_rows_and_tensor():
    rng = np.random.default_rng(5)
    a = rng.standard_normal((4, 256))
    w = rng.standard_normal((32, 256)) * 0.02
    y = O.linear_fp8(a, w, None)
    a2 = a.copy()
    a2[1] *= 2.0 ** -7
    y2 = O.linear_fp8(a2, w, None)
    assert np.array_equal(y2[1], y[1] * 2.0 ** -7) and np.array_equal(y2[[0, 2, 3]], y[[0, 2, 3]])
    assert np.array_equal(O.linear_fp8(a, w * 8.0, None), y * 8.0)
    # and it is a linear layer up to the e4m3 rounding of both operands
    ref = O.linear(a, w, None)
    assert 0 < np.linalg.norm(y - ref) / np.linalg.norm(ref) < 0.06


def test_block_fp8_close_to_exact_block():
    from video_diffusion_transformer_fwd_b200 import synth
    D, Fh, heads, grid = 128, 256, 2, (2, 3, 4)
    w = {k: v.double().numpy() for k, v in synth.block_weights(D, Fh, "f32", seed=3).items()}
    acts = synth.block_activations(1, 24, D, 5, "f32", seed=9)
    x, ctx, e0 = (acts[k].double().numpy() for k in ("x", "ctx", "e0"))
    y = O.block_forward(x, ctx, None, e0, w, heads, grid, 1e-6)
    y8 = O.block_forward(x, ctx, None, e0, w, heads, grid, 1e-6, fp8=True)
    rel = np.linalg.norm((y8 - x) - (y - x)) / np.linalg.norm(y - x)
    assert 1e-3 < rel < 0.1
