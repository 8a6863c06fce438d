"""Micro-benchmark of single C-ABI entry points on seeded inputs (also the
driver used for ncu captures of one kernel on a small case).

    python -m video_diffusion_transformer_fwd_b200.kernel_bench attention --B 1 --L 16384 --heads 40
    python -m video_diffusion_transformer_fwd_b200.kernel_bench block --config a14b-step --B 2
    python -m video_diffusion_transformer_fwd_b200.kernel_bench block --config a14b-step --F 5 ...

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
    ap.add_argument("what", choices=["attention", "block"])
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
        ms, prof = _time(lambda: wan.attention(q, k, v, out=o), a.iters, a.warmup)
        flops = 4.0 * a.B * a.L * Lk * a.heads * 128
        print(json.dumps({"what": "attention", "B": a.B, "Lq": a.L, "Lk": Lk, "heads": a.heads,
                          "ms": ms, "tflops": flops / ms / 1e9, "kernels_ms": prof}))
        return
    cfg = configs.get(a.config)
    if a.F:
        cfg = dataclasses.replace(cfg, F=a.F)
    cfg = dataclasses.replace(cfg, batch=a.B)
    dims = wan.dims_of(cfg)
    w = synth.block_weights(cfg.dim, cfg.ffn_dim, cfg.dtype, "cuda", 0)
    acts = synth.block_activations(a.B, cfg.L, cfg.dim, cfg.text_len, cfg.dtype, "cuda", 100)
    rope = wan.rope_freqs(cfg.head_dim, 1024, cfg.theta)
    ws = wan.alloc_workspace(dims, a.B)
    cw = wan.make_weights(w)
    ms, prof = _time(lambda: wan.block_forward(dims, acts["x"], acts["ctx"], acts["e0"], cw, rope, ws),
                     a.iters, a.warmup)
    print(json.dumps({"what": "block", "config": cfg.name, "B": a.B, "L": cfg.L, "ms": ms,
                      "tflops": cfg.block_flops() / ms / 1e9,
                      "gemm_tflops": cfg.gemm_flops() / (prof.get("gemm_tc", 0) or float("nan")) / 1e9,
                      "attn_tflops": cfg.self_attn_flops() / (prof.get("attn_self", 0) or float("nan")) / 1e9,
                      "kernels_ms": prof}))


if __name__ == "__main__":
    main()
