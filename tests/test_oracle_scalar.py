"""The two forms of the oracle agree: the scalar-loop form (plain Python
floats, one multiply-add at a time, no arrays) and the NumPy form, on the
tiny configuration (L = 32, dim 128, 4 heads of 32, ffn 512, text 8) with
ragged text lengths and a sharp softmax, to fp64 rounding. A slip in the
NumPy form's array axes (a transposed operand, a wrong einsum index, the
wrong RoPE pair) would show here, since the scalar form names every index."""
import numpy as np
import pytest

from oracle import wan_oracle as O
from oracle import wan_oracle_scalar as S
from video_diffusion_transformer_fwd_b200 import configs, synth


def _case(seed, gain_scale=1.0):
    cfg = configs.get("tiny")
    w = {k: v.double().numpy() for k, v in synth.block_weights(cfg.dim, cfg.ffn_dim, "f32", seed=seed,
                                                                  gain_scale=gain_scale).items()}
    acts = synth.block_activations(2, cfg.L, cfg.dim, cfg.text_len, "f32", seed=seed + 100)
    return cfg, w, {k: v.double().numpy() for k, v in acts.items()}


@pytest.mark.parametrize("seed,gain_scale,lens", [(0, 1.0, None), (3, 4.0, [5, 0])])
def test_scalar_and_numpy_oracles_agree(seed, gain_scale, lens):
    cfg, w, a = _case(seed, gain_scale)
    grid = (cfg.F, cfg.H, cfg.W)
    ref = O.block_forward(a["x"], a["ctx"], None if lens is None else np.array(lens), a["e0"], w,
                          cfg.heads, grid, cfg.eps, cfg.theta)
    for b in range(2):
        got = np.array(S.block_forward(a["x"][b], a["ctx"][b], None if lens is None else lens[b],
                                       a["e0"][b], w, cfg.heads, grid, cfg.eps, cfg.theta))
        assert np.abs(got - ref[b]).max() <= 1e-12 * max(1.0, np.abs(ref[b]).max())


def test_scalar_euler_matches():
    rng = np.random.default_rng(0)
    x, vc, vu = (rng.standard_normal(50) for _ in range(3))
    got = np.array(S.euler_cfg_step(list(x), list(vc), list(vu), 5.0, 0.9, 0.875))
    assert np.abs(got - O.euler_cfg_step(x, vc, vu, 5.0, 0.9, 0.875)).max() <= 1e-15


def test_scalar_rope_matches_the_table():
    """The scalar rotation against the NumPy form's table, every pair of a
    head at a few grid positions."""
    rng = np.random.default_rng(1)
    v = rng.standard_normal(128)
    for pos in ((0, 0, 0), (3, 1, 7), (20, 29, 51)):
        got = np.array(S.rope_rotate_head(list(v), *pos, 1e4))
        ref = O.rope_apply(v.reshape(1, 1, 128), None, positions=np.array([pos]))[0, 0]
        assert np.abs(got - ref).max() <= 1e-13
