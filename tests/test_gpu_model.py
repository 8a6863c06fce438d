"""Parity of the whole-model forward on latents (patch embedding, time and
text embeddings, the block stack, head, unpatchify) and of the model-level
CFG Euler step, CUDA path through the C ABI against the fp64 oracle on the
same seeded inputs. fp32: max-abs <= 1e-4; bf16: relative L2 <= 2e-2."""
import numpy as np
import pytest
import torch

from oracle import wan_oracle as O
from video_diffusion_transformer_fwd_b200 import step, synth, wan

from parity_util import BF16_REL_L2, F32_MAX_ABS, np64, rel_l2, weights64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    wan.load()


class ModelCase:
    """Seeded small model: embeddings, head and ``nblocks`` blocks."""

    def __init__(self, C_in, C_out, F, H, W, dim, heads, ffn, T, text_dim, nblocks, dtype, B=2,
                 seed=0, same_latent=False):
        dev = "cuda"
        self.dims = wan.make_model_dims(C_in, C_out, F, H, W, dim, heads, ffn, T, text_dim, 256,
                                        1e-6, dtype)
        self.mw = synth.model_weights(C_in, C_out, dim, text_dim, 256, dtype, dev, seed + 50000)
        self.blocks = [synth.block_weights(dim, ffn, dtype, dev, seed + 1000 * i)
                       for i in range(nblocks)]
        inp = synth.model_inputs(B, C_in, F, H, W, T, text_dim, dtype, dev, seed + 60000,
                                 same_latent=same_latent)
        self.latent, self.text = inp["latent"], inp["text"]
        self.heads = heads
        self.rope = wan.rope_freqs(dim // heads, 1024, 1e4, device=dev)
        self.ws = wan.alloc_model_workspace(self.dims, B, device=dev)

    def run(self, t, ctx_lens=None):
        tt = torch.tensor(t, dtype=torch.float32, device="cuda")
        kl = None if ctx_lens is None else torch.tensor(ctx_lens, dtype=torch.int32, device="cuda")
        out = wan.model_forward(self.dims, self.latent, tt, self.text, self.mw, self.blocks,
                                self.rope, self.ws, ctx_lens=kl)
        torch.cuda.synchronize()
        assert wan.device_status() == wan.WAN_OK
        return np64(out)

    def oracle(self, t, ctx_lens=None):
        t32 = np.asarray(t, np.float32).astype(np.float64)
        return O.model_forward(np64(self.latent), t32, np64(self.text),
                               None if ctx_lens is None else np.asarray(ctx_lens),
                               weights64(self.mw), [weights64(w) for w in self.blocks],
                               self.heads, 1e-6)


@pytest.mark.parametrize("C_in", [16, 36])
def test_model_forward_f32(C_in):
    """fp32 small model, T2V (16 channels in) and I2V (36 in: noise, mask and
    image latent concatenated), ragged text lengths, two blocks."""
    c = ModelCase(C_in, 16, 3, 8, 10, 128, 4, 256, 9, 64, 2, "f32")
    t, lens = [875.0, 312.5], [9, 4]
    got, ref = c.run(t, lens), c.oracle(t, lens)
    assert got.shape == ref.shape == (2, 16, 3, 8, 10)
    assert np.abs(got - ref).max() <= F32_MAX_ABS


def test_model_forward_f32_no_blocks_no_text():
    """Zero blocks and zero text tokens: patch embedding straight into the head."""
    c = ModelCase(16, 16, 2, 4, 6, 128, 4, 256, 0, 64, 0, "f32", B=3)
    t = [0.0, 500.0, 999.0]
    got, ref = c.run(t), c.oracle(t)
    assert np.abs(got - ref).max() <= F32_MAX_ABS


def test_model_forward_bf16():
    """bf16 model on the tensor-core path: head_dim 128, 512 tokens a
    sequence (grid 2 x 16 x 16), two blocks, ragged text."""
    c = ModelCase(16, 16, 2, 32, 32, 256, 2, 512, 20, 256, 2, "bf16")
    t, lens = [937.5, 937.5], [20, 13]
    got, ref = c.run(t, lens), c.oracle(t, lens)
    assert rel_l2(got, ref) <= BF16_REL_L2
    for b in range(2):
        assert rel_l2(got[b], ref[b]) <= BF16_REL_L2


def test_model_forward_bf16_48_channels():
    """Latent width of the 5B model (48 channels in and out), bf16."""
    c = ModelCase(48, 48, 2, 16, 32, 256, 2, 512, 16, 256, 1, "bf16")
    t = [400.0, 12.0]
    got, ref = c.run(t), c.oracle(t)
    assert rel_l2(got, ref) <= BF16_REL_L2


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("sigma,sigma_next", [(0.95, 0.9), (0.5, 0.45)])
def test_model_denoise_step_two_experts(dtype, sigma, sigma_next):
    """The CFG pair through the whole model, then the Euler move of the latent;
    the expert is picked by t = 1000 sigma against the boundary 875."""
    if dtype == "f32":
        shape = dict(C_in=16, C_out=16, F=2, H=8, W=8, dim=128, heads=4, ffn=256, T=7,
                     text_dim=64, nblocks=2)
    else:
        shape = dict(C_in=16, C_out=16, F=2, H=16, W=32, dim=256, heads=2, ffn=512, T=12,
                     text_dim=256, nblocks=2)
    hi = ModelCase(**shape, dtype=dtype, seed=0, same_latent=True)
    lo = ModelCase(**shape, dtype=dtype, seed=7)
    lat = hi.latent[0].clone()
    ds = step.ModelDenoiseStep(hi.dims, {"high": (hi.mw, hi.blocks), "low": (lo.mw, lo.blocks)},
                               hi.text, lat, boundary=875.0)
    name = ds.expert(sigma)
    assert name == O.select_expert(1000.0 * sigma, 875.0)
    ex = hi if name == "high" else lo
    lat0 = np64(lat)
    ds.step(sigma, sigma_next, 5.0)
    torch.cuda.synchronize()
    assert wan.device_status() == wan.WAN_OK
    # the kernel moves by the fp32 difference of the two fp32 sigmas
    dt = float(np.float32(sigma_next) - np.float32(sigma))
    w_blocks = [weights64(w) for w in ex.blocks]
    ref = O.model_denoise_step(lat0, sigma, sigma + dt, np64(hi.text[0]), np64(hi.text[1]),
                               weights64(ex.mw), w_blocks, ex.heads, 1e-6, 5.0)
    got = np64(ds.latent)
    v = np64(ds.v)
    v_ref = O.model_forward(np.stack([lat0, lat0]), [1000.0 * sigma] * 2, np64(hi.text), None,
                            weights64(ex.mw), w_blocks, ex.heads, 1e-6)
    # the Euler move of the GPU's own two velocities
    assert np.abs(got - O.euler_cfg_step(lat0, v[0], v[1], 5.0, sigma, sigma + dt)).max() <= 1e-5
    if dtype == "f32":
        assert np.abs(v - v_ref).max() <= F32_MAX_ABS
        assert np.abs(got - ref).max() <= F32_MAX_ABS
    else:
        for b in range(2):
            assert rel_l2(v[b], v_ref[b]) <= BF16_REL_L2
        # v = (1 - s) v_u + s v_c: its error is at most |1 - s| |e_u| + s |e_c|
        vg = 5.0 * v_ref[0] - 4.0 * v_ref[1]
        bound = BF16_REL_L2 * (4.0 * np.linalg.norm(v_ref[1]) + 5.0 * np.linalg.norm(v_ref[0]))
        assert np.linalg.norm((got - lat0) - (ref - lat0)) <= abs(dt) * bound
        assert np.linalg.norm(vg) > 0


def test_model_forward_rejects_bad_dims():
    d = wan.make_model_dims(16, 16, 2, 7, 8, 128, 4, 256, 0, 64, 256, 1e-6, "f32")   # H odd
    assert wan.wan_model_workspace_bytes(d, 1) == 0
    d = wan.make_model_dims(16, 16, 2, 8, 8, 128, 4, 256, 4, 60, 256, 1e-6, "f32")   # text_dim
    assert wan.wan_model_workspace_bytes(d, 1) == 0
