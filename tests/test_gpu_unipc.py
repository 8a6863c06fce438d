"""The UniPC sampler on the GPU (wan_unipc_step with the library's host
coefficients) against the oracle's UniPC: on fixed velocity sequences (the
whole recursion, every step) and through the whole model on a latent."""
import numpy as np
import pytest
import torch

from oracle import wan_oracle as O
from video_diffusion_transformer_fwd_b200 import step, synth, wan

from parity_util import np64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    wan.load()


@pytest.mark.parametrize("vdt", ["f32", "bf16"])
@pytest.mark.parametrize("order,lof,n,N", [(2, True, 8, 1 << 20), (1, True, 5, 1001), (2, False, 12, 4099)])
def test_unipc_trajectory_matches_oracle(vdt, order, lof, n, N):
    sig = list(O.flow_sigmas(n, shift=5.0))
    if not lof:
        sig[-1] = sig[-2] * 0.5
    g = torch.Generator(device="cuda").manual_seed(n + N)
    x = torch.randn(N, device="cuda", generator=g)
    vc = [torch.randn(N, device="cuda", generator=g).to(synth.TORCH_DTYPES[vdt]) for _ in range(n)]
    vu = [torch.randn(N, device="cuda", generator=g).to(synth.TORCH_DTYPES[vdt]) for _ in range(n)]
    x0 = np64(x)
    sampler = wan.UniPCSampler(x, sig, order=order, lower_order_final=lof)
    seen = []
    for i in range(n):
        seen.append(np64(x))
        sampler.step(vc[i], vu[i], 5.0)
    torch.cuda.synchronize()
    vc64, vu64 = [np64(v) for v in vc], [np64(v) for v in vu]
    ref, ref_seen = O.unipc_sample(x0, lambda xx, s, i: vu64[i] + 5.0 * (vc64[i] - vu64[i]), sig, order=order,
                                   lower_order_final=lof)
    scale = max(1.0, np.abs(ref).max())
    for a, b in zip(seen, ref_seen):
        assert np.abs(a - b).max() <= 2e-5 * scale
    assert np.abs(np64(x) - ref).max() <= 2e-5 * scale


def test_unipc_through_the_model():
    """Four UniPC steps of a small fp32 model on its latent (CFG pair, t =
    1000 sigma), against the oracle's sampler driving the oracle's model."""
    from test_gpu_model import ModelCase
    c = ModelCase(16, 16, 2, 8, 8, 128, 4, 256, 7, 64, 2, "f32", seed=0, same_latent=True)
    lat = c.latent[0].clone()
    ds = step.ModelDenoiseStep(c.dims, {"high": (c.mw, c.blocks)}, c.text, lat, boundary=0.0)
    sig = list(O.flow_sigmas(4, shift=5.0))
    sampler = wan.UniPCSampler(lat, sig)
    lat0 = np64(lat)
    for _ in range(4):
        ds.unipc_step(sampler, 5.0)
    torch.cuda.synchronize()
    assert wan.device_status() == wan.WAN_OK
    mw = {k: np64(v) for k, v in c.mw.items()}
    blocks = [{k: np64(v) for k, v in b.items()} for b in c.blocks]
    text = np64(c.text)

    def velocity(x, s, i):
        t = float(np.float32(1000.0 * s))
        v = O.model_forward(np.stack([x, x]), [t, t], text, None, mw, blocks, c.heads, 1e-6)
        return v[1] + 5.0 * (v[0] - v[1])
    ref, _ = O.unipc_sample(lat0, velocity, sig)
    assert np.abs(np64(lat) - ref).max() <= 1e-4 * max(1.0, np.abs(ref).max())
