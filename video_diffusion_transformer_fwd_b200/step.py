"""One denoising step on the token stream, driven through the C ABI.

The block stack runs on the CFG pair (the same x and timestep against the
conditional and the unconditional context, batched as B = 2), then
wan_euler_cfg_step combines the two outputs with the guidance scale and
moves x by (sigma_next - sigma) * v ("Wan2.2 code walkthrough" (newtid.com),
sampling-loop snippet). Device memory comes from torch; every step of the
computation runs in libwan.
"""
from __future__ import annotations

import torch

from . import synth, wan
from .configs import BlockConfig


class DenoiseStep:
    def __init__(self, cfg: BlockConfig, seed: int = 0, device: str = "cuda", weights=None,
                 fp8: bool = False, attn8: bool = False):
        """``fp8``: the blocks run their projections as FP8 GEMMs (the bf16
        weights are quantized per tensor once, here); ``attn8`` also runs the
        self-attention as the 8-bit attention."""
        self.cfg = cfg
        self.dims = wan.dims_of(cfg)
        self.device = device
        self.weights = weights if weights is not None else synth.step_weights(cfg, device, seed)
        if fp8 or attn8:
            self.dims.dtype = wan.WAN_FP8_ATTN if attn8 else wan.WAN_FP8
            self.weights = [wan.quantize_block_weights(w) for w in self.weights]
        self.cweights = [wan.make_weights(w) for w in self.weights]
        acts = synth.block_activations(2, cfg.L, cfg.dim, cfg.text_len, cfg.dtype, device,
                                       seed + 100, same_e0=True)
        self.x = acts["x"][0].contiguous()                 # [L, D] float32, the state
        self.ctx = acts["ctx"]                             # [2, T, D]: cond, uncond
        self.e0 = acts["e0"]                               # [2, 6, D], one timestep
        self.xb = torch.empty((2, cfg.L, cfg.dim), dtype=torch.float32, device=device)
        self.rope = wan.rope_freqs(cfg.head_dim, 1024, cfg.theta, device=device)
        self.ws = wan.alloc_workspace(self.dims, 2, device=device)
        self.ws_bytes = self.ws.numel()

    def blocks(self, stream=None):
        """The block stack on xb (in place)."""
        s = wan._stream(stream)
        for cw in self.cweights:
            wan.check(wan.wan_block_forward(self.dims, 2, self.xb.data_ptr(), self.ctx.data_ptr(),
                                            None, self.e0.data_ptr(), cw, self.rope.data_ptr(),
                                            self.rope.shape[0], self.ws.data_ptr(), self.ws_bytes,
                                            s))

    def step(self, stream=None):
        c = self.cfg
        self.xb[0].copy_(self.x)
        self.xb[1].copy_(self.x)
        self.blocks(stream)
        wan.check(wan.wan_euler_cfg_step(self.x.data_ptr(), self.xb[0].data_ptr(),
                                         self.xb[1].data_ptr(), wan.WAN_F32, self.x.numel(),
                                         c.guide_scale, c.sigma, c.sigma_next,
                                         wan._stream(stream)))
        return self.x


class ModelDenoiseStep:
    """One CFG flow-matching Euler step on the latent through the whole model
    (wan_model_forward on the CFG pair at t = 1000 sigma, then
    wan_euler_cfg_step on the latent). With two experts, the high-noise one
    runs while t >= boundary ("Wan2.2 code walkthrough" (newtid.com), MoE
    snippet: boundary 0.875 * 1000 for text-to-video, 900 for image-to-video).

    ``experts`` maps "high" / "low" to (model weight dict, list of block weight
    dicts); a single expert may be passed as {"high": ...} with boundary 0.
    """

    def __init__(self, dims: "wan.wan_model_dims", experts: dict, text, latent,
                 boundary: float = 875.0, ctx_lens=None, rope_max_pos: int = 1024,
                 theta: float = 1e4, device: str = "cuda"):
        self.dims = dims
        self.boundary = boundary
        self.experts = {k: (wan.make_model_weights(mw), wan.make_block_array(bl))
                        for k, (mw, bl) in experts.items()}
        self._keep = experts                         # device tensors stay alive
        self.text = text                             # [2, T, text_dim]: cond, uncond
        self.ctx_lens = ctx_lens
        self.latent = latent                         # [C_in, F, H, W] float32, the state
        head_dim = dims.dim // dims.heads
        self.rope = wan.rope_freqs(head_dim, rope_max_pos, theta, device=device)
        self.lat2 = torch.empty((2,) + tuple(latent.shape), dtype=torch.float32, device=device)
        self.t = torch.empty(2, dtype=torch.float32, device=device)
        self.v = torch.empty((2, dims.C_out, dims.F, dims.H, dims.W), dtype=torch.float32,
                             device=device)
        self.ws = wan.alloc_model_workspace(dims, 2, device=device)

    def expert(self, sigma: float) -> str:
        t = 1000.0 * sigma
        if "low" not in self.experts or t >= self.boundary:
            return "high"
        return "low"

    def _guide(self, name, guide_scale):
        """A (low-noise, high-noise) pair picks the expert's scale ([WALK]
        sampling-loop snippet: e.g. (3.0, 4.0) for text-to-video)."""
        if isinstance(guide_scale, (tuple, list)):
            return guide_scale[1] if name == "high" else guide_scale[0]
        return guide_scale

    def velocity(self, sigma: float, stream=None):
        """The model on the CFG pair at t = 1000 sigma: self.v[0] (cond),
        self.v[1] (uncond). Returns the expert used."""
        s = wan._stream(stream)
        name = self.expert(sigma)
        mw, blocks = self.experts[name]
        self.lat2[0].copy_(self.latent)
        self.lat2[1].copy_(self.latent)
        self.t.fill_(1000.0 * sigma)
        wan.check(wan.wan_model_forward(self.dims, 2, self.lat2.data_ptr(), self.t.data_ptr(),
                                        wan._ptr(self.text), wan._ptr(self.ctx_lens), mw, blocks,
                                        len(blocks), self.rope.data_ptr(), self.rope.shape[0],
                                        self.v.data_ptr(), self.ws.data_ptr(), self.ws.numel(), s))
        return name

    def step(self, sigma: float, sigma_next: float, guide_scale, stream=None):
        """Euler step from sigma to sigma_next."""
        name = self.velocity(sigma, stream)
        wan.check(wan.wan_euler_cfg_step(self.latent.data_ptr(), self.v[0].data_ptr(),
                                         self.v[1].data_ptr(), wan.WAN_F32, self.latent.numel(),
                                         self._guide(name, guide_scale), sigma, sigma_next,
                                         wan._stream(stream)))
        return self.latent

    def unipc_step(self, sampler: "wan.UniPCSampler", guide_scale, stream=None):
        """One UniPC step (the sampler's x is this latent): the model at the
        sampler's current sigma, then the fused UniPC update."""
        name = self.velocity(sampler.sigma, stream)
        sampler.step(self.v[0], self.v[1], self._guide(name, guide_scale), stream)
        return self.latent
