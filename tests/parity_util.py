"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI
on seeded inputs, and run the oracle on the same values."""
from __future__ import annotations

import numpy as np
import torch

from oracle import wan_oracle as O
from video_diffusion_transformer_fwd_b200 import synth, wan
from video_diffusion_transformer_fwd_b200.configs import BlockConfig

BF16_REL_L2 = 2e-2      # bf16 configs: relative L2 error bound on sampled rows
F32_MAX_ABS = 1e-4      # fp32 configs: max-abs error bound


def rel_l2(a, b) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    den = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (den if den > 0 else 1.0))


def np64(t):
    return synth.to_numpy64(t)


def weights64(w):
    return {k: np64(v) for k, v in w.items()}


class GpuBlockRun:
    """One wan_block_forward call on seeded inputs, keeping everything the
    oracle needs."""

    def __init__(self, cfg: BlockConfig, B=1, seed=0, gain_scale=1.0, same_x=False,
                 same_e0=False, ctx_lens=None, dtype=None, weights=None, zero_gates=False):
        dev = "cuda"
        self.cfg = cfg
        self.dtype = dtype or cfg.dtype
        self.B = B
        self.dims = wan.make_dims(cfg.F, cfg.H, cfg.W, cfg.dim, cfg.heads, cfg.ffn_dim,
                                  cfg.text_len, cfg.eps, self.dtype)
        self.w = weights if weights is not None else synth.block_weights(
            cfg.dim, cfg.ffn_dim, self.dtype, dev, seed, gain_scale=gain_scale)
        acts = synth.block_activations(B, cfg.L, cfg.dim, cfg.text_len, self.dtype, dev,
                                       seed + 100, same_x=same_x, same_e0=same_e0)
        if zero_gates:
            acts["e0"][:, 2] = -self.w["modulation"][2]
            acts["e0"][:, 5] = -self.w["modulation"][5]
        self.x0 = acts["x"].clone()
        self.x = acts["x"]
        self.ctx = acts["ctx"]
        self.e0 = acts["e0"]
        self.ctx_lens = None if ctx_lens is None else torch.tensor(ctx_lens, dtype=torch.int32,
                                                                    device=dev)
        self.rope = wan.rope_freqs(cfg.head_dim, 1024, cfg.theta, device=dev)
        self.ws = wan.alloc_workspace(self.dims, B, device=dev)

    def run(self, times=1):
        for _ in range(times):
            wan.block_forward(self.dims, self.x, self.ctx, self.e0, self.w, self.rope, self.ws,
                              ctx_lens=self.ctx_lens)
        torch.cuda.synchronize()
        assert wan.device_status() == wan.WAN_OK
        return self

    def ws_rows(self, which, width, rows):
        """Rows (token indices of every sequence) of a [B*L, width] workspace buffer."""
        tdt = synth.TORCH_DTYPES[self.dtype]
        L = self.cfg.L
        v = wan.workspace_view(self.ws, self.dims, self.B, which, (self.B, L, width), tdt)
        return np64(v[:, torch.as_tensor(rows, device=v.device)])

    def oracle_rows(self, rows, kv=None, intermediates=None):
        c = self.cfg
        lens = None if self.ctx_lens is None else self.ctx_lens.cpu().numpy()
        return O.block_forward_rows(np64(self.x0), np64(self.ctx), lens, np64(self.e0),
                                    weights64(self.w), c.heads, (c.F, c.H, c.W), c.eps, rows,
                                    theta=c.theta, kv=kv, intermediates=intermediates)
