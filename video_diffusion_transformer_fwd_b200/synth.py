"""Seeded synthetic inputs for the block and the denoising step.

This module holds no arithmetic of the method: it only draws numbers. Each
tensor is drawn by its own ``torch.Generator`` seeded ``seed + index`` (the
index is the tensor's position in the fixed lists below), as float32 normals
scaled and shifted, then rounded once to the run dtype. Both sides of every
parity check consume exactly these values: the CUDA library receives the
device tensors and the oracle receives their upcast host copies.

Distributions (no trained weights or real text features exist here; these
stand in for them):
  weights and biases      N(0, 0.02)
  RMSNorm / norm3 gains   1 + N(0, 0.02); norm3 beta N(0, 0.02)
  x (token stream), ctx   N(0, 1)
  e0 and the block's 6 x dim modulation   N(0, 0.1)
"""
from __future__ import annotations

import torch

WEIGHT_SPECS = (
    # name, shape key, kind, is_matrix_dtype
    ("modulation", "6D", "mod", False),
    ("wq", "DD", "w", True), ("bq", "D", "w", True),
    ("wk", "DD", "w", True), ("bk", "D", "w", True),
    ("wv", "DD", "w", True), ("bv", "D", "w", True),
    ("wo", "DD", "w", True), ("bo", "D", "w", True),
    ("gq", "D", "gain", False), ("gk", "D", "gain", False),
    ("g3", "D", "gain", False), ("b3", "D", "w", False),
    ("cwq", "DD", "w", True), ("cbq", "D", "w", True),
    ("cwk", "DD", "w", True), ("cbk", "D", "w", True),
    ("cwv", "DD", "w", True), ("cbv", "D", "w", True),
    ("cwo", "DD", "w", True), ("cbo", "D", "w", True),
    ("cgq", "D", "gain", False), ("cgk", "D", "gain", False),
    ("w1", "FD", "w", True), ("b1", "F", "w", True),
    ("w2", "DF", "w", True), ("b2", "D", "w", True),
)

TORCH_DTYPES = {"f32": torch.float32, "bf16": torch.bfloat16}


def _shape(key, D, Fh):
    return {"6D": (6, D), "DD": (D, D), "D": (D,), "FD": (Fh, D), "F": (Fh,),
            "DF": (D, Fh)}[key]


def _normal(shape, seed, device, std, mean=0.0):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    t = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    if mean != 0.0:
        t.add_(mean)
    return t


def block_weights(dim, ffn_dim, dtype="bf16", device="cpu", seed=0,
                  gain_scale=1.0, std=0.02, mod_std=0.1):
    """One block's parameters. Matrices and biases in ``dtype``; gains, norm3
    affine and modulation in float32. ``gain_scale`` multiplies the q/k
    RMSNorm gains (a larger value sharpens the softmax)."""
    tdt = TORCH_DTYPES[dtype]
    out = {}
    for idx, (name, key, kind, is_mat) in enumerate(WEIGHT_SPECS):
        shape = _shape(key, dim, ffn_dim)
        s = seed + idx
        if kind == "mod":
            t = _normal(shape, s, device, mod_std)
        elif kind == "gain":
            t = _normal(shape, s, device, std, 1.0)
            if name in ("gq", "gk", "cgq", "cgk") and gain_scale != 1.0:
                t.mul_(gain_scale)
        else:
            t = _normal(shape, s, device, std)
        out[name] = t.to(tdt).contiguous() if is_mat else t.contiguous()
    return out


def block_activations(B, L, dim, text_len, dtype="bf16", device="cpu", seed=100,
                      same_x=False, same_e0=False, mod_std=0.1):
    """x [B, L, D] float32, ctx [B, T, D] in ``dtype``, e0 [B, 6, D] float32.
    ``same_x`` / ``same_e0`` repeat sequence 0 across the batch (the CFG
    pair runs one x and one timestep against two contexts)."""
    tdt = TORCH_DTYPES[dtype]
    if same_x:
        x = _normal((1, L, dim), seed, device, 1.0).expand(B, L, dim).contiguous()
    else:
        x = _normal((B, L, dim), seed, device, 1.0)
    ctx = _normal((B, text_len, dim), seed + 1, device, 1.0).to(tdt).contiguous()
    if same_e0:
        e0 = _normal((1, 6, dim), seed + 2, device, mod_std).expand(B, 6, dim).contiguous()
    else:
        e0 = _normal((B, 6, dim), seed + 2, device, mod_std)
    return {"x": x, "ctx": ctx, "e0": e0}


def step_weights(cfg, device="cpu", seed=0):
    """The block stack of a denoising step: block i drawn with seed
    ``seed + 1000 * i``."""
    return [block_weights(cfg.dim, cfg.ffn_dim, cfg.dtype, device, seed + 1000 * i)
            for i in range(cfg.blocks)]


MODEL_WEIGHT_SPECS = (
    # name, shape key, is_matrix_dtype (False: float32)
    ("patch_w", "D,4C", True), ("patch_b", "D", True),
    ("text_w1", "D,TD", True), ("text_b1", "D", True),
    ("text_w2", "D,D", True), ("text_b2", "D", True),
    ("time_w1", "D,FD", False), ("time_b1", "D", False),
    ("time_w2", "D,D", False), ("time_b2", "D", False),
    ("proj_w", "6D,D", False), ("proj_b", "6D", False),
    ("head_mod", "2,D", False),
    ("head_w", "4CO,D", True), ("head_b", "4CO", True),
)


def model_weights(C_in, C_out, dim, text_dim, freq_dim=256, dtype="bf16", device="cpu",
                  seed=50000, std=0.02, head_mod_std=0.1):
    """The embeddings and head around the block stack (all N(0, std) except
    head_mod, N(0, head_mod_std)). The patch weight is the Conv3d weight
    [dim, C_in, 1, 2, 2] flattened to [dim, C_in * 4]."""
    tdt = TORCH_DTYPES[dtype]
    sizes = {"D": dim, "4C": 4 * C_in, "TD": text_dim, "FD": freq_dim, "6D": 6 * dim, "2": 2,
             "4CO": 4 * C_out}
    out = {}
    for idx, (name, key, is_mat) in enumerate(MODEL_WEIGHT_SPECS):
        shape = tuple(sizes[k] for k in key.split(","))
        t = _normal(shape, seed + idx, device, head_mod_std if name == "head_mod" else std)
        out[name] = t.to(tdt).contiguous() if is_mat else t.contiguous()
    return out


def model_inputs(B, C_in, F, H, W, text_len, text_dim, dtype="bf16", device="cpu", seed=60000,
                 same_latent=False):
    """latent [B, C_in, F, H, W] float32 N(0, 1) (``same_latent``: sequence 0
    repeated, the CFG pair), text features [B, text_len, text_dim] N(0, 1) in
    ``dtype``."""
    tdt = TORCH_DTYPES[dtype]
    nb = 1 if same_latent else B
    lat = _normal((nb, C_in, F, H, W), seed, device, 1.0).expand(B, C_in, F, H, W).contiguous()
    text = _normal((B, text_len, text_dim), seed + 1, device, 1.0).to(tdt).contiguous()
    return {"latent": lat, "text": text}


def attention_inputs(B, Lq, Lk, heads, head_dim, dtype="bf16", device="cpu", seed=500,
                     std=1.0):
    """q [B, Lq, n, d], k and v [B, Lk, n, d] in ``dtype``."""
    tdt = TORCH_DTYPES[dtype]
    q = _normal((B, Lq, heads, head_dim), seed, device, std).to(tdt)
    k = _normal((B, Lk, heads, head_dim), seed + 1, device, std).to(tdt)
    v = _normal((B, Lk, heads, head_dim), seed + 2, device, 1.0).to(tdt)
    return q, k, v


def sample_rows(L, n=256, seed=1):
    """Rows checked at full size: the first, the last and n - 2 more drawn
    without replacement by ``numpy.random.default_rng(seed)``."""
    import numpy as np
    if L <= n:
        return np.arange(L)
    rng = np.random.default_rng(seed)
    mid = rng.choice(np.arange(1, L - 1), size=n - 2, replace=False)
    return np.unique(np.concatenate([[0, L - 1], mid]))


def to_numpy64(t):
    """Exact float64 copy of a (possibly bf16, possibly device) tensor."""
    return t.detach().to("cpu", torch.float64).numpy()
