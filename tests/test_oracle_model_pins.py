"""Pins for the whole-model part of the oracle (patch embedding, time and
text embeddings, head, unpatchify, expert switch, latent denoising step)
against library routines, closed forms and the pages' printed values."""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as Fn

from oracle import wan_oracle as O

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_shapes.json")))
RNG = np.random.default_rng(99)


def test_patch_embed_matches_torch_conv3d():
    B, C, F, H, W, dim = 2, 3, 2, 6, 8, 5
    lat = RNG.standard_normal((B, C, F, H, W))
    w = RNG.standard_normal((dim, C, 1, 2, 2))
    b = RNG.standard_normal(dim)
    out = O.patch_embed(lat, {"patch_w": w, "patch_b": b})               # [B, L, dim]
    ref = Fn.conv3d(torch.tensor(lat), torch.tensor(w), torch.tensor(b), stride=(1, 2, 2))
    ref = ref.flatten(2).transpose(1, 2).numpy()                           # flatten(2).transpose as in the forward snippet
    np.testing.assert_allclose(out, ref, atol=1e-12)


def test_unpatchify_places_features():
    """Feature (kt, kh, kw, c) of token (f, h, w) lands at [c, f, 2h+kh, 2w+kw];
    checked on every element against torch's view / permute."""
    B, F, H, W, C = 1, 2, 3, 4, 5
    tok = RNG.standard_normal((B, F * H * W, 4 * C))
    out = O.unpatchify(tok, (F, H, W), C)
    assert out.shape == (B, C, F, 2 * H, 2 * W)
    t = torch.tensor(tok).view(B, F, H, W, 1, 2, 2, C)
    ref = torch.einsum("bfhwpqrc->bcfphqwr", t).reshape(B, C, F, 2 * H, 2 * W).numpy()
    np.testing.assert_array_equal(out, ref)
    f, h, w, kh, kw, c = 1, 2, 3, 1, 0, 4
    i = (f * H + h) * W + w
    assert out[0, c, f, 2 * h + kh, 2 * w + kw] == tok[0, i, (kh * 2 + kw) * C + c]


def test_head_output_width_is_the_pages_64():
    assert 16 * 1 * 2 * 2 == GOLD["diffusers_trace"]["head_out"]


def test_sinusoidal_embedding_closed_forms():
    e = O.sinusoidal_embedding(256, [0.0, 875.0])
    assert e.shape == (2, 256)
    np.testing.assert_array_equal(e[0, :128], 1.0)                         # cos(0)
    np.testing.assert_array_equal(e[0, 128:], 0.0)                         # sin(0)
    assert abs(e[1, 0] - math.cos(875.0)) < 1e-12 and abs(e[1, 128] - math.sin(875.0)) < 1e-12
    w_last = 10000.0 ** (-127 / 128)
    assert abs(e[1, 127] - math.cos(875.0 * w_last)) < 1e-12
    np.testing.assert_allclose(e[:, :128] ** 2 + e[:, 128:] ** 2, 1.0, atol=1e-12)


def test_time_and_text_embedding_match_torch_modules():
    dim, fd = 16, 256
    mw = {"time_w1": RNG.standard_normal((dim, fd)) * 0.1, "time_b1": RNG.standard_normal(dim),
          "time_w2": RNG.standard_normal((dim, dim)) * 0.1, "time_b2": RNG.standard_normal(dim),
          "proj_w": RNG.standard_normal((6 * dim, dim)) * 0.1, "proj_b": RNG.standard_normal(6 * dim),
          "text_w1": RNG.standard_normal((dim, 40)) * 0.1, "text_b1": RNG.standard_normal(dim),
          "text_w2": RNG.standard_normal((dim, dim)) * 0.1, "text_b2": RNG.standard_normal(dim)}
    T = {k: torch.tensor(v) for k, v in mw.items()}
    t = np.array([900.0, 12.5])
    e, e0 = O.time_embed(t, mw, fd)
    s = torch.tensor(O.sinusoidal_embedding(fd, t))
    te = Fn.linear(Fn.silu(Fn.linear(s, T["time_w1"], T["time_b1"])), T["time_w2"], T["time_b2"])
    np.testing.assert_allclose(e, te.numpy(), atol=1e-12)
    np.testing.assert_allclose(e0, Fn.linear(Fn.silu(te), T["proj_w"], T["proj_b"]).view(2, 6, dim).numpy(), atol=1e-12)
    ctx = RNG.standard_normal((2, 7, 40))
    ref = Fn.linear(Fn.gelu(Fn.linear(torch.tensor(ctx), T["text_w1"], T["text_b1"]), approximate="tanh"),
                    T["text_w2"], T["text_b2"]).numpy()
    np.testing.assert_allclose(O.text_embed(ctx, mw), ref, atol=1e-12)


def test_head_zeroed_input_gives_bias():
    dim = 8
    mw = {"head_mod": np.zeros((2, dim)), "head_w": RNG.standard_normal((64, dim)),
          "head_b": RNG.standard_normal(64)}
    e = np.zeros((1, dim))
    e[0] = -1.0                                                            # scale chunk: 1 + (-1) = 0
    mw["head_mod"][0] = 1.0                                                # shift chunk: 1 + (-1) = 0
    x = RNG.standard_normal((1, 5, dim))
    np.testing.assert_allclose(O.head(x, e, mw, 1e-6), np.broadcast_to(mw["head_b"], (1, 5, 64)), atol=1e-12)


def test_expert_switch_boundaries():
    g = GOLD["expert_switch"]
    b = g["t2v_boundary_fraction"] * g["num_train_timesteps"]
    assert b == 875.0
    assert O.select_expert(875.0, b) == "high" and O.select_expert(874.999, b) == "low"
    assert O.select_expert(900.0, g["i2v_high_noise_from"]) == "high"
    assert O.select_expert(899.0, g["i2v_high_noise_from"]) == "low"


def _tiny_model(C=4, dim=32, heads=2, ffn=64, text_dim=24, nblocks=2, seed=5):
    rs = np.random.default_rng(seed)
    mw = {"patch_w": rs.standard_normal((dim, C, 1, 2, 2)) * 0.2, "patch_b": rs.standard_normal(dim) * 0.1,
          "text_w1": rs.standard_normal((dim, text_dim)) * 0.2, "text_b1": rs.standard_normal(dim) * 0.1,
          "text_w2": rs.standard_normal((dim, dim)) * 0.2, "text_b2": rs.standard_normal(dim) * 0.1,
          "time_w1": rs.standard_normal((dim, 256)) * 0.05, "time_b1": rs.standard_normal(dim) * 0.1,
          "time_w2": rs.standard_normal((dim, dim)) * 0.2, "time_b2": rs.standard_normal(dim) * 0.1,
          "proj_w": rs.standard_normal((6 * dim, dim)) * 0.1, "proj_b": rs.standard_normal(6 * dim) * 0.1,
          "head_mod": rs.standard_normal((2, dim)) * 0.1, "head_w": rs.standard_normal((4 * C, dim)) * 0.2,
          "head_b": rs.standard_normal(4 * C) * 0.1}
    blocks = []
    for i in range(nblocks):
        w = {}
        for n in O.BLOCK_WEIGHT_NAMES:
            shape = {"modulation": (6, dim), "w1": (ffn, dim), "b1": (ffn,), "w2": (dim, ffn)}.get(
                n, (dim, dim) if n.startswith(("w", "cw")) else (dim,))
            w[n] = rs.standard_normal(shape) * (0.2 if len(shape) == 2 else 0.1)
            if n in ("gq", "gk", "cgq", "cgk", "g3"):
                w[n] = 1 + w[n]
        blocks.append(w)
    return mw, blocks


def test_model_forward_with_zero_blocks_is_embed_head_unpatch():
    """No blocks: the output is head(patch_embed(latent)) folded back — the
    composition of the separately pinned parts, and its shape is the latent's."""
    mw, _ = _tiny_model()
    lat = RNG.standard_normal((2, 4, 3, 4, 6))
    out = O.model_forward(lat, [500.0, 100.0], RNG.standard_normal((2, 5, 24)), None, mw, [], 2, 1e-6)
    assert out.shape == lat.shape
    e, _ = O.time_embed(np.array([500.0, 100.0]), mw)
    ref = O.unpatchify(O.head(O.patch_embed(lat, mw), e, mw, 1e-6), (3, 2, 3), 4)
    np.testing.assert_allclose(out, ref, atol=1e-12)


def test_model_denoise_step_identity_blocks_and_guidance():
    """Blocks reduced to the identity (gates 0, cross output 0) and a head
    returning zero velocity (zero weights and bias) leave the latent
    unchanged; with identical contexts the guidance scale drops out."""
    mw, blocks = _tiny_model()
    for w in blocks:
        w["modulation"][2] = 0.0
        w["modulation"][5] = 0.0
        w["cwo"][:] = 0.0
        w["cbo"][:] = 0.0
    mw["proj_w"][2 * 32:3 * 32] = 0.0; mw["proj_b"][2 * 32:3 * 32] = 0.0      # e0 gate chunks 0
    mw["proj_w"][5 * 32:6 * 32] = 0.0; mw["proj_b"][5 * 32:6 * 32] = 0.0
    lat = RNG.standard_normal((4, 2, 4, 4))
    ctx = RNG.standard_normal((5, 24))
    a = O.model_denoise_step(lat, 0.9, 0.875, ctx, ctx, mw, blocks, 2, 1e-6, 5.0)
    b = O.model_denoise_step(lat, 0.9, 0.875, ctx, ctx, mw, blocks, 2, 1e-6, 1.0)
    np.testing.assert_allclose(a, b, atol=1e-12)
    mw0 = dict(mw, head_w=np.zeros_like(mw["head_w"]), head_b=np.zeros_like(mw["head_b"]))
    c = O.model_denoise_step(lat, 0.9, 0.875, ctx, 2 * ctx, mw0, blocks, 2, 1e-6, 5.0)
    np.testing.assert_array_equal(c, lat)
