"""Pins of the oracle's per-token timestep modulation ("Wan2.2 code
walkthrough", time-projection snippet: the timestep embedding unflattened to
(batch, seq_len), e0 [B, L, 6, dim]): equal per-token values reproduce the
per-sequence path exactly, and a token's gates act on that token only."""
import numpy as np

from oracle import wan_oracle as O
from video_diffusion_transformer_fwd_b200 import synth


def _block_case(B=2, grid=(2, 3, 4), D=128, Fh=256, T=5, seed=3):
    L = grid[0] * grid[1] * grid[2]
    w = {k: v.double().numpy() for k, v in synth.block_weights(D, Fh, "f32", seed=seed).items()}
    acts = synth.block_activations(B, L, D, T, "f32", seed=seed + 100)
    x, ctx, e0 = (acts[k].double().numpy() for k in ("x", "ctx", "e0"))
    return w, x, ctx, e0, L


def test_equal_per_token_modulation_is_the_per_sequence_path():
    w, x, ctx, e0, L = _block_case()
    e0_tok = np.repeat(e0[:, None], L, axis=1)                  # [B, L, 6, D]
    a = O.block_forward(x, ctx, None, e0, w, 2, (2, 3, 4), 1e-6)
    b = O.block_forward(x, ctx, None, e0_tok, w, 2, (2, 3, 4), 1e-6)
    assert np.array_equal(a, b)
    rows = np.array([0, 7, 23])
    # (a different row count changes only the BLAS summation order)
    assert np.allclose(O.block_forward_rows(x, ctx, None, e0_tok, w, 2, (2, 3, 4), 1e-6, rows), a[:, rows],
                       rtol=0, atol=1e-12)


def test_a_tokens_gates_act_on_that_token_only():
    w, x, ctx, e0, L = _block_case()
    w = dict(w, cwo=np.zeros_like(w["cwo"]), cbo=np.zeros_like(w["cbo"]))   # no cross residual
    e0_tok = np.repeat(e0[:, None], L, axis=1).copy()
    r = 9
    e0_tok[1, r, 2] = -w["modulation"][2]                         # this token's gates: 0
    e0_tok[1, r, 5] = -w["modulation"][5]
    y = O.block_forward(x, ctx, None, e0_tok, w, 2, (2, 3, 4), 1e-6)
    assert np.array_equal(y[1, r], x[1, r])
    others = np.ones(L, bool)
    others[r] = False
    assert (np.abs(y[1, others] - x[1, others]).max(axis=1) > 0).all()
    assert (np.abs(y[0] - x[0]).max(axis=1) > 0).all()


def test_per_token_time_embedding_and_head():
    rng = np.random.default_rng(0)
    mw = {k: rng.standard_normal(s) * 0.05 for k, s in (
        ("time_w1", (32, 256)), ("time_b1", (32,)), ("time_w2", (32, 32)), ("time_b2", (32,)),
        ("proj_w", (192, 32)), ("proj_b", (192,)), ("head_mod", (2, 32)), ("head_w", (64, 32)),
        ("head_b", (64,)))}
    t = np.array([[0.0, 875.0, 875.0], [500.0, 1.0, 999.0]])
    e, e0 = O.time_embed(t, mw)
    assert e.shape == (2, 3, 32) and e0.shape == (2, 3, 6, 32)
    for b in range(2):
        for i in range(3):
            eb, e0b = O.time_embed(np.array([t[b, i]]), mw)
            assert np.allclose(e[b, i], eb[0], rtol=0, atol=1e-13) and np.allclose(e0[b, i], e0b[0], rtol=0, atol=1e-13)
    x = rng.standard_normal((2, 3, 32))
    e_seq = e[:, 0]                                              # per-sequence e, repeated per token
    assert np.array_equal(O.head(x, np.repeat(e_seq[:, None], 3, axis=1), mw, 1e-6), O.head(x, e_seq, mw, 1e-6))
