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
    def __init__(self, cfg: BlockConfig, seed: int = 0, device: str = "cuda", weights=None):
        self.cfg = cfg
        self.dims = wan.dims_of(cfg)
        self.device = device
        self.weights = weights if weights is not None else synth.step_weights(cfg, device, seed)
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
