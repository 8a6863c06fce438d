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

# Canary guard bytes: outputs and workspaces of the parity tests sit inside a
# larger allocation whose GUARD_BYTES before and after are filled with
# GUARD_VALUE; a kernel writing past either end of its buffer changes them.
GUARD_BYTES = 4096      # keeps the buffer's alignment (a multiple of 256)
GUARD_VALUE = 0xA5


class Guarded:
    """A device tensor of ``shape`` / ``dtype`` (``t``) with canary bytes on
    both sides; ``check()`` asserts they are untouched."""

    def __init__(self, shape, dtype, device="cuda", init=None):
        es = torch.empty((), dtype=dtype).element_size()
        n = 1
        for d in shape:
            n *= int(d)
        self.nbytes = n * es
        self.raw = torch.full((2 * GUARD_BYTES + self.nbytes,), GUARD_VALUE, dtype=torch.uint8,
                              device=device)
        self.t = self.raw[GUARD_BYTES:GUARD_BYTES + self.nbytes].view(dtype).view(*shape)
        if init is not None:
            self.t.copy_(init)

    def check(self, what="buffer"):
        torch.cuda.synchronize()
        lo = self.raw[:GUARD_BYTES]
        hi = self.raw[GUARD_BYTES + self.nbytes:]
        assert bool((lo == GUARD_VALUE).all()), f"{what}: bytes before the buffer overwritten"
        assert bool((hi == GUARD_VALUE).all()), f"{what}: bytes after the buffer overwritten"


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
        self._gx = Guarded(tuple(acts["x"].shape), acts["x"].dtype, dev, init=acts["x"])
        self.x = self._gx.t
        self.ctx = acts["ctx"]
        self.e0 = acts["e0"]
        self.ctx_lens = None if ctx_lens is None else torch.tensor(ctx_lens, dtype=torch.int32,
                                                                    device=dev)
        self.rope = wan.rope_freqs(cfg.head_dim, 1024, cfg.theta, device=dev)
        self._gws = Guarded((wan.wan_block_workspace_bytes(self.dims, B),), torch.uint8, dev)
        self.ws = self._gws.t

    def run(self, times=1):
        for _ in range(times):
            wan.block_forward(self.dims, self.x, self.ctx, self.e0, self.w, self.rope, self.ws,
                              ctx_lens=self.ctx_lens)
        torch.cuda.synchronize()
        assert wan.device_status() == wan.WAN_OK
        self._gx.check("x")
        self._gws.check("workspace")
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
