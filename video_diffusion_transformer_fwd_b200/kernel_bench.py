"""Micro-benchmark of single C-ABI entry points on seeded inputs (also the
driver used for ncu captures of one kernel on a small case).

    python -m video_diffusion_transformer_fwd_b200.kernel_bench attention --B 1 --L 16384 --heads 40
    python -m video_diffusion_transformer_fwd_b200.kernel_bench block --config a14b-step --B 2
    python -m video_diffusion_transformer_fwd_b200.kernel_bench block --config a14b-step --F 5 ...
    python -m video_diffusion_transformer_fwd_b200.kernel_bench model --blocks 0
    python -m video_diffusion_transformer_fwd_b200.kernel_bench euler --n 33554432

Prints one JSON line with the mean device time per call (CUDA events on the
launching stream, after warm-up) and the per-kernel-class times.
"""
from __future__ import annotations

import argparse
import dataclasses
import json

import torch

from . import configs, synth, wan


def _time(fn, iters, warmup):
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    wan.check(wan.wan_profile_enable(1))
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(iters):
        fn()
    b.record()
    torch.cuda.synchronize()
    prof = wan.profile_read()
    wan.check(wan.wan_profile_enable(0))
    if wan.device_status() != wan.WAN_OK:
        raise RuntimeError(wan.last_error())
    return a.elapsed_time(b) / iters, {k: v[1] / iters for k, v in prof.items() if v[0]}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("what", choices=["attention", "block", "model", "euler"])
    ap.add_argument("--n", type=int, default=1 << 25, help="euler: elements of the token state")
    ap.add_argument("--blocks", type=int, default=0)
    ap.add_argument("--fp8", action="store_true", help="block: FP8 GEMM mode")
    ap.add_argument("--attn8", action="store_true", help="8-bit attention (block: with FP8 GEMMs)")
    ap.add_argument("--per-token", action="store_true", help="block: e0 per token [B, L, 6, dim]")
    ap.add_argument("--config", default="a14b-step")
    ap.add_argument("--B", type=int, default=1)
    ap.add_argument("--L", type=int, default=16384)
    ap.add_argument("--Lk", type=int, default=0)
    ap.add_argument("--heads", type=int, default=40)
    ap.add_argument("--F", type=int, default=0)
    ap.add_argument("--iters", type=int, default=3)
    ap.add_argument("--warmup", type=int, default=1)
    a = ap.parse_args()
    torch.cuda.set_device(0)
    if a.what == "attention":
        Lk = a.Lk or a.L
        q, k, v = synth.attention_inputs(a.B, a.L, Lk, a.heads, 128, "bf16", "cuda", 1)
        o = torch.empty_like(q)
        if a.attn8:
            ws8 = torch.empty(wan.wan_attention_8bit_workspace_bytes(a.B, a.heads, a.L, Lk), dtype=torch.uint8,
                              device="cuda")
            ms, prof = _time(lambda: wan.attention_8bit(q, k, v, out=o, workspace=ws8), a.iters, a.warmup)
        else:
            ms, prof = _time(lambda: wan.attention(q, k, v, out=o), a.iters, a.warmup)
        flops = 4.0 * a.B * a.L * Lk * a.heads * 128
        print(json.dumps({"what": "attention", "attn8": a.attn8, "B": a.B, "Lq": a.L, "Lk": Lk, "heads": a.heads,
                          "ms": ms, "tflops": flops / ms / 1e9, "kernels_ms": prof}))
        return
    if a.what == "euler":
        # CFG + Euler on fp32 state and velocities: 16 bytes of HBM traffic per element
        g = torch.Generator(device="cuda").manual_seed(7)
        x, vc, vu = (torch.randn(a.n, device="cuda", generator=g) for _ in range(3))
        ms, prof = _time(lambda: wan.euler_cfg_step(x, vc, vu, 5.0, 0.9, 0.875), a.iters, a.warmup)
        print(json.dumps({"what": "euler", "n": a.n, "ms": ms, "gbs": 16.0 * a.n / ms / 1e6, "kernels_ms": prof}))
        return
    cfg = configs.get(a.config)
    if a.what == "model":
        model(cfg, a)
        return
    if a.F:
        cfg = dataclasses.replace(cfg, F=a.F)
    cfg = dataclasses.replace(cfg, batch=a.B)
    dims = wan.dims_of(cfg)
    w = synth.block_weights(cfg.dim, cfg.ffn_dim, cfg.dtype, "cuda", 0)
    if a.fp8 or a.attn8:
        dims.dtype = wan.WAN_FP8_ATTN if a.attn8 else wan.WAN_FP8
        w = wan.quantize_block_weights(w)
    acts = synth.block_activations(a.B, cfg.L, cfg.dim, cfg.text_len, cfg.dtype, "cuda", 100)
    if a.per_token:
        dims.e0_per_token = 1
        acts["e0"] = acts["e0"][:, None].expand(a.B, cfg.L, 6, cfg.dim).contiguous()
    rope = wan.rope_freqs(cfg.head_dim, 1024, cfg.theta)
    ws = wan.alloc_workspace(dims, a.B)
    cw = wan.make_weights(w)
    ms, prof = _time(lambda: wan.block_forward(dims, acts["x"], acts["ctx"], acts["e0"], cw, rope, ws),
                     a.iters, a.warmup)
    print(json.dumps({"what": "block", "config": cfg.name, "B": a.B, "L": cfg.L, "fp8": a.fp8, "attn8": a.attn8, "per_token": a.per_token, "ms": ms,
                      "tflops": cfg.block_flops() / ms / 1e9,
                      "gemm_tflops": cfg.gemm_flops() / (prof.get("gemm_tc", 0) or float("nan")) / 1e9,
                      "attn_tflops": cfg.self_attn_flops() / (prof.get("attn_self", 0) or float("nan")) / 1e9,
                      "kernels_ms": prof}))


def model(cfg, a):
    """wan_model_forward on the CFG pair (B = 2) at the config's token grid
    (latent [16, F, 2H, 2W], text 512 x 4096) with ``--blocks`` blocks; with 0
    blocks it times the embeddings, head and unpatchify alone."""
    F = a.F or cfg.F
    C, text_dim, B = 16, 4096, 2
    dims = wan.make_model_dims(C, C, F, 2 * cfg.H, 2 * cfg.W, cfg.dim, cfg.heads, cfg.ffn_dim,
                               cfg.text_len, text_dim, 256, cfg.eps, cfg.dtype)
    mw = synth.model_weights(C, C, cfg.dim, text_dim, 256, cfg.dtype, "cuda")
    blocks = wan.make_block_array([synth.block_weights(cfg.dim, cfg.ffn_dim, cfg.dtype, "cuda", i)
                                   for i in range(a.blocks)]) if a.blocks else wan.make_block_array([])
    inp = synth.model_inputs(B, C, F, 2 * cfg.H, 2 * cfg.W, cfg.text_len, text_dim, cfg.dtype,
                             "cuda", same_latent=True)
    t = torch.full((B,), 900.0, device="cuda")
    rope = wan.rope_freqs(cfg.head_dim, 1024, cfg.theta)
    ws = wan.alloc_model_workspace(dims, B)
    out = torch.empty((B, C, F, 2 * cfg.H, 2 * cfg.W), device="cuda")
    mwc = wan.make_model_weights(mw)
    ms, prof = _time(lambda: wan.model_forward(dims, inp["latent"], t, inp["text"], mwc, blocks,
                                               rope, ws, out=out), a.iters, a.warmup)
    L = F * cfg.H * cfg.W
    es = 2 if cfg.dtype == "bf16" else 4
    D = cfg.dim
    # bytes the embeddings and head must move at least: latent in, x written once (fp32),
    # x read by the head LN, its output written and read by the head GEMM, velocity out,
    # plus every weight once
    wbytes = sum(v.numel() * v.element_size() for v in mw.values())
    alg = (B * C * L * 4 * 4 + B * L * D * 4 + B * L * D * 4 + 2 * B * L * D * es
           + B * C * L * 4 * 4 + inp["text"].numel() * es + wbytes)
    print(json.dumps({"what": "model", "config": cfg.name, "B": B, "L": L, "blocks": a.blocks,
                      "ms": ms, "embed_head_algorithmic_bytes": alg,
                      "embed_head_gbs": alg / ms / 1e6 if a.blocks == 0 else None,
                      "kernels_ms": prof}))


if __name__ == "__main__":
    main()
