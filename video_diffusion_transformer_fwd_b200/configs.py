"""Workload table: the block shapes of the Wan2.1 / Wan2.2 DiT that the
library is exercised on.

Dims follow the model table of the "Wan2.2 code walkthrough" (newtid.com;
T2V/I2V-A14B dim 5120, 40 heads, 40 layers; TI2V-5B dim 3072, 24 heads) and
the Wan2.1-1.3B block (dim 1536, 12 heads, ffn 8960). Token grids come from
the clip size through the VAE stride and the (1, 2, 2) patch embedding.
"""
from __future__ import annotations

from dataclasses import dataclass, field


@dataclass(frozen=True)
class BlockConfig:
    name: str
    F: int
    H: int
    W: int
    dim: int
    heads: int
    ffn_dim: int
    text_len: int
    dtype: str                      # "f32" or "bf16"
    batch: int = 1                  # sequences per block call (2 = cond + uncond)
    blocks: int = 1                 # blocks in the stack
    eps: float = 1e-6
    theta: float = 1e4
    guide_scale: float = 5.0
    sigma: float = 0.9
    sigma_next: float = 0.875
    note: str = ""

    @property
    def L(self) -> int:
        return self.F * self.H * self.W

    @property
    def head_dim(self) -> int:
        return self.dim // self.heads

    # ---- algorithmic work of one block call (all `batch` sequences) ----
    def gemm_flops(self) -> float:
        D, Fh, L, T, B = self.dim, self.ffn_dim, self.L, self.text_len, self.batch
        per_seq = 2.0 * L * D * (3 * D + D + D + D + 2 * Fh) + 2.0 * T * D * (2 * D)
        return B * per_seq

    def self_attn_flops(self) -> float:
        return self.batch * 4.0 * self.L * self.L * self.dim

    def cross_attn_flops(self) -> float:
        return self.batch * 4.0 * self.L * self.text_len * self.dim

    def block_flops(self) -> float:
        return self.gemm_flops() + self.self_attn_flops() + self.cross_attn_flops()


CONFIGS = {
    "tiny": BlockConfig("tiny", 2, 4, 4, 128, 4, 512, 8, "f32",
                        note="tiny fp32 block, L=32, head_dim 32"),
    "1.3b-short": BlockConfig("1.3b-short", 5, 30, 52, 1536, 12, 8960, 512, "bf16",
                              note="Wan2.1-1.3B block, 17-frame 480x832 clip, L=7800"),
    "1.3b-long": BlockConfig("1.3b-long", 21, 30, 52, 1536, 12, 8960, 512, "bf16",
                             note="Wan2.1-1.3B block, 81-frame 480x832 clip, L=32760"),
    "5b": BlockConfig("5b", 31, 22, 40, 3072, 24, 14336, 512, "bf16",
                      note="TI2V-5B block, 121-frame 704x1280 clip, VAE (4,16,16), L=27280"),
    "a14b-step": BlockConfig("a14b-step", 21, 30, 52, 5120, 40, 13824, 512, "bf16",
                             batch=2, blocks=40,
                             note="A14B denoising step: 40 blocks, cond+uncond batched, "
                                  "CFG 5.0, Euler sigma 0.9 -> 0.875, L=32760"),
}


def get(name: str) -> BlockConfig:
    return CONFIGS[name]
