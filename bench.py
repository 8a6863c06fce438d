#!/usr/bin/env python
"""Benchmark of the Wan DiT hot path on B200: one A14B-shaped denoising step
per bench step (40 WanAttentionBlocks, dim 5120, 40 heads, ffn 13824, on the
CFG pair -- cond and uncond batched as B = 2 -- over L = 32760 tokens, then
the CFG-Euler update x += (sigma' - sigma) v with guidance 5, sigma 0.9 ->
0.875), all through the C ABI of libwan.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints ONE JSON line (rank 0). The metric is the DiT block forward time:
`value` = device time of the timed steps / (steps x blocks x 2 sequences x
N ranks), i.e. ms per block forward over one 32760-token sequence for the
whole job (lower is better); attention and GEMM TFLOP/s come from CUDA
events recorded around every kernel launch inside the timed region.
Multi-GPU runs are independent replicas (each rank its own step; weak
scaling), timed as the max over ranks.
`--impl reference` times the fp64 CPU oracle on a bounded sample of the same
workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "DiT block fwd ms & attention TFLOP/s (bf16, 32760 tok) vs tensor peak"
UNIT = "ms per block forward (one 32760-token sequence)"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM traffic per launch of the dominant kernel, from an ncu capture of the
# same kernel source (sha256 prefix below); reported as null once the source
# has changed since the capture.
TRAFFIC = {
    # profiles/attn_tc_B1_L16384.md: 653.4 MB per launch at B=1, L=16384, scaled by the
    # query/key rows (x4) to the step's launch at B=2, L=32760
    "attn_self": {"bytes_per_launch": 4 * 653.4e6, "source_sha": "39316987c6657670"},
}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=4)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default="a14b-step")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip the single-block rows of the other configurations (run after the timed step)")
    ap.add_argument("--fp8", action="store_true",
                    help="FP8 GEMM mode of the blocks (e4m3 projections, bf16 attention); not the default")
    ap.add_argument("--attn8", action="store_true",
                    help="FP8 GEMMs and the 8-bit self-attention (int8 Q K^T, e4m3 P V); not the default")
    ap.add_argument("--ulysses", action="store_true",
                    help="all ranks form one sequence-parallel group: tokens sharded, every block's self-attention "
                         "head-parallel between two all-to-alls (strong scaling); not the default")
    ap.add_argument("--cfg-parallel", action="store_true",
                    help="ranks 2p / 2p+1 run the conditional / unconditional branch of one step and "
                         "exchange their block outputs (even --gpus); not the default")
    return ap.parse_args()


def read_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def source_hash(*names):
    """Hash of the sources a kernel is compiled from (its .cu and the shared headers)."""
    h = hashlib.sha256()
    for name in names:
        with open(os.path.join(ROOT, "video_diffusion_transformer_fwd_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


ATTN_SOURCES = ("attn_tc.cu", "sm100.cuh", "common.cuh")


# ----------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, indices):
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-i", ",".join(str(i) for i in indices)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons, power = [], [], set(), []
        for line in out.splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
                power.append(float(f[3]))
            except ValueError:
                continue
            for name, val in zip(self.REASONS, f[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "power_w_max": max(power) if power else None,
                "samples": len(sm), "reasons": sorted(reasons)}


# ----------------------------------------------------------------- CPU oracle sample
class OracleSample:
    """Times the fp64 oracle (as it stands) on a bounded sample of one block
    forward of the workload and expresses it per block forward of one
    sequence: LayerNorm + K/V projection on r_kv rows (scaled by L / r_kv),
    and the rest of the block for r_q and 2 r_q query rows attending over
    all L keys (the difference gives the per-row cost, the remainder the
    fixed per-call cost of the text K/V projection). Inputs are drawn once
    by the seeded generators; only the oracle calls are timed."""

    def __init__(self, cfg, seed=0, r_kv=4096, r_q=12, fp8=False):
        import numpy as np

        from video_diffusion_transformer_fwd_b200 import synth
        self.cfg, self.r_kv, self.r_q, self.fp8 = cfg, r_kv, r_q, fp8
        w = synth.block_weights(cfg.dim, cfg.ffn_dim, cfg.dtype, "cpu", seed)
        self.w64 = {k: synth.to_numpy64(v) for k, v in w.items()}
        acts = synth.block_activations(1, r_kv, cfg.dim, cfg.text_len, cfg.dtype, "cpu", seed + 100)
        self.x = synth.to_numpy64(acts["x"])
        self.ctx = synth.to_numpy64(acts["ctx"])
        self.e0 = synth.to_numpy64(acts["e0"])
        reps = (cfg.L + r_kv - 1) // r_kv
        self.xq = np.ascontiguousarray(np.tile(self.x, (1, reps, 1))[:, :cfg.L])
        self.reps = reps

    def run(self):
        import numpy as np

        from oracle import wan_oracle as O
        cfg, r_kv, r_q = self.cfg, self.r_kv, self.r_q
        t0 = time.perf_counter()
        k, v = O.self_attn_kv(self.x, self.e0, self.w64, cfg.heads, (1, 1, r_kv), cfg.eps, cfg.theta,
                              fp8=self.fp8)
        t_kv = time.perf_counter() - t0
        # full-length keys/values (rows repeated: the attention cost depends only on L)
        kf = np.tile(k, (1, self.reps, 1, 1))[:, :cfg.L]
        vf = np.tile(v, (1, self.reps, 1, 1))[:, :cfg.L]
        grid = (cfg.F, cfg.H, cfg.W)
        times = []
        for r in (r_q, 2 * r_q):
            t0 = time.perf_counter()
            O.block_forward_rows(self.xq, self.ctx, None, self.e0, self.w64, cfg.heads, grid, cfg.eps,
                                 np.arange(r), theta=cfg.theta, kv=(kf, vf), fp8=self.fp8)
            times.append(time.perf_counter() - t0)
        per_row = max((times[1] - times[0]) / r_q, 0.0)
        fixed = max(times[0] - per_row * r_q, 0.0)
        est = t_kv * cfg.L / r_kv + fixed + per_row * cfg.L
        detail = (("FP8-GEMM " if self.fp8 else "") + f"ESTIMATE from a measured sample: fp64 oracle on one block "
                  f"forward of the workload's block shape (one sequence): LN + K/V projection timed on {r_kv} "
                  f"rows (scaled x{cfg.L / r_kv:.1f}); the rest of the block timed for {r_q} and {2 * r_q} "
                  f"query rows attending over all {cfg.L} keys (per-row cost x{cfg.L}, plus the per-call "
                  f"text K/V projection); {t_kv + sum(times):.1f} s of CPU time sampled")
        measured = {"kv_rows": r_kv, "kv_s": t_kv, "query_rows": [r_q, 2 * r_q], "query_s": times,
                    "sampled_s": t_kv + sum(times)}
        return est * 1e3, detail, measured


def _oracle_rows_worker(args):
    """One process of the full-block oracle run: the block at ``rows`` from
    inputs memory-mapped from ``d`` (spawned, one BLAS thread)."""
    d, heads, grid, eps, theta, rows = args
    import numpy as np
    try:
        from threadpoolctl import threadpool_limits
        threadpool_limits(1)
    except Exception:
        pass
    from oracle import wan_oracle as O
    ld = lambda n: np.load(os.path.join(d, n + ".npy"), mmap_mode="r")
    w = {k[2:]: ld(k) for k in (f[:-4] for f in os.listdir(d)) if k.startswith("w_")}
    t0 = time.perf_counter()
    out = O.block_forward_rows(ld("x"), ld("ctx"), None, ld("e0"), w, heads, grid, eps, rows,
                               theta=theta, kv=(ld("k"), ld("v")))
    return time.perf_counter() - t0, out.shape[1]


def oracle_full_block(cfg, procs, seed=0):
    """Un-extrapolated fp64 oracle time of one whole block forward of one
    sequence of ``cfg``: the key / value projection of every row (the
    oracle's self_attn_kv, multi-threaded BLAS), then block_forward_rows on
    every row, the rows split over ``procs`` spawned processes. Only the
    oracle calls are timed (inputs are drawn and shared beforehand)."""
    import multiprocessing as mp
    import shutil
    import tempfile

    import numpy as np

    from oracle import wan_oracle as O
    from video_diffusion_transformer_fwd_b200 import synth
    w = synth.block_weights(cfg.dim, cfg.ffn_dim, cfg.dtype, "cpu", seed)
    acts = synth.block_activations(1, cfg.L, cfg.dim, cfg.text_len, cfg.dtype, "cpu", seed + 100)
    grid = (cfg.F, cfg.H, cfg.W)
    d = tempfile.mkdtemp(prefix="wan_oracle_", dir="/dev/shm" if os.path.isdir("/dev/shm") else None)
    try:
        arr = {k: synth.to_numpy64(acts[k]) for k in ("x", "ctx", "e0")}
        for k, v in w.items():
            arr["w_" + k] = synth.to_numpy64(v)
        t0 = time.perf_counter()
        k, v = O.self_attn_kv(arr["x"], arr["e0"], {n[2:]: a for n, a in arr.items() if n.startswith("w_")},
                              cfg.heads, grid, cfg.eps, cfg.theta)
        t_kv = time.perf_counter() - t0
        arr["k"], arr["v"] = k, v
        for n, a in arr.items():
            np.save(os.path.join(d, n + ".npy"), a)
        chunks = [c for c in np.array_split(np.arange(cfg.L), procs) if len(c)]
        ctx = mp.get_context("spawn")
        with ctx.Pool(len(chunks)) as pool:
            pool.map(_oracle_rows_worker, [(d, cfg.heads, grid, cfg.eps, cfg.theta, chunks[0][:2])] * len(chunks))
            t0 = time.perf_counter()
            res = pool.map(_oracle_rows_worker, [(d, cfg.heads, grid, cfg.eps, cfg.theta, c) for c in chunks])
            t_rows = time.perf_counter() - t0
        assert sum(r[1] for r in res) == cfg.L
        return {"config": cfg.name, "kind": "full block, every row (not extrapolated)", "rows": cfg.L,
                "oracle_s": t_kv + t_rows, "kv_s": t_kv, "rows_s": t_rows, "processes": len(chunks),
                "cpu_s": t_kv + sum(r[0] for r in res)}
    finally:
        shutil.rmtree(d, ignore_errors=True)


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        return sum(i.get("num_threads", 0) for i in info if i.get("user_api") == "blas") or None
    except Exception:
        return None


# ----------------------------------------------------------------- multi-rank timing
def max_over_ranks(ms: float, world: int, device="cpu") -> float:
    """Max of a per-rank device time over all ranks (the job's time)."""
    if world <= 1:
        return float(ms)
    import torch
    import torch.distributed as dist
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def per_block_ms(job_ms: float, steps: int, blocks: int, world: int) -> float:
    """Whole-job ms per block forward of one sequence: every rank runs `steps`
    steps of `blocks` blocks on the CFG pair (2 sequences)."""
    return job_ms / (steps * blocks * 2 * world)


# ----------------------------------------------------------------- reference arm
def run_reference(args, rank, world):
    if rank != 0:
        return
    from video_diffusion_transformer_fwd_b200 import configs
    cfg = configs.get(args.config)
    sample = OracleSample(cfg, seed=0, r_kv=2048, r_q=8)
    vals = []
    detail, measured = "", {}
    for i in range(args.warmup + args.steps):
        ms, detail, measured = sample.run()
        if i >= args.warmup:
            vals.append(ms)
    value = statistics.mean(vals)
    cores = cpu_cores()
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": value * cfg.blocks * 2, "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "impl": "reference",
        "estimated": True,
        "config": workload_config(cfg, world),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "blas_threads": blas_threads(),
                         "kind": "oracle", "estimated": True, "measured": measured, "sample": detail},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def workload_config(cfg, world, cfg_parallel=False, ulysses=False):
    return {
        "workload": (f"{cfg.name}: {cfg.blocks} WanAttentionBlocks dim {cfg.dim}, {cfg.heads} heads "
                     f"(head_dim {cfg.head_dim}), ffn {cfg.ffn_dim}, grid {cfg.F}x{cfg.H}x{cfg.W} "
                     f"(L={cfg.L}), text {cfg.text_len}, cond+uncond batched (B=2), CFG "
                     f"{cfg.guide_scale}, Euler sigma {cfg.sigma}->{cfg.sigma_next}"),
        "seq_len": cfg.L, "batch_per_gpu": 1 if cfg_parallel else 2, "blocks": cfg.blocks,
        "global_batch": 2 if ulysses else world if cfg_parallel else 2 * world,
        "parallelism": (f"ulysses-{world} (tokens sharded, self-attention head-parallel between two "
                        f"all-to-alls per block)" if ulysses else
                        "cfg-pairs (branch outputs all-gathered within each pair)" if cfg_parallel else
                        "replicas" if world > 1 else "single"),
        "l2": "inputs larger than L2 (28 GB of block weights and a 671 MB token state per step)",
        "weights": "random N(0,0.02), synthetic x/ctx N(0,1)",
    }


# ----------------------------------------------------------------- per-config block rows
PER_CONFIG = (("1.3b-short", 1), ("1.3b-long", 1), ("5b", 1), ("a14b-step", 1), ("a14b-step", 2))


def per_config_rows(dev, peaks, iters=5, warmup=2):
    """One bf16 block forward per configuration of the workload table (random
    N(0, 0.02) weights, x and ctx N(0, 1)), timed alone with CUDA events:
    block ms and the attention / GEMM split from the per-launch events, with
    fractions of the measured burst bf16 peak (kernels timed in isolation)."""
    import dataclasses

    import torch

    from video_diffusion_transformer_fwd_b200 import configs, synth, wan
    burst = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    rows = []
    stream = torch.cuda.current_stream()
    for name, B in PER_CONFIG:
        cfg = dataclasses.replace(configs.get(name), batch=B, blocks=1)
        dims = wan.dims_of(cfg)
        wt = synth.block_weights(cfg.dim, cfg.ffn_dim, cfg.dtype, dev, 0)    # the tensors stay alive
        w = wan.make_weights(wt)
        acts = synth.block_activations(B, cfg.L, cfg.dim, cfg.text_len, cfg.dtype, dev, 100)
        rope = wan.rope_freqs(cfg.head_dim, 1024, cfg.theta, device=dev)
        ws = wan.alloc_workspace(dims, B, device=dev)
        for _ in range(warmup):
            wan.block_forward(dims, acts["x"], acts["ctx"], acts["e0"], w, rope, ws)
        torch.cuda.synchronize()
        clocks = ClockSampler([torch.cuda.current_device()])
        wan.check(wan.wan_profile_enable(1))
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(iters):
            wan.block_forward(dims, acts["x"], acts["ctx"], acts["e0"], w, rope, ws)
        t1.record(stream)
        torch.cuda.synchronize()
        prof = wan.profile_read()
        wan.check(wan.wan_profile_enable(0))
        ck = clocks.stop()
        if wan.device_status() != wan.WAN_OK:
            raise RuntimeError(f"per-config {name}: " + wan.last_error())
        ms = t0.elapsed_time(t1) / iters
        a_n, a_ms = prof["attn_self"]
        g_n, g_ms = prof["gemm_tc"]
        a_tf = cfg.self_attn_flops() * iters / (a_ms * 1e-3) / 1e12 if a_ms > 0 else None
        g_tf = cfg.gemm_flops() * iters / (g_ms * 1e-3) / 1e12 if g_ms > 0 else None
        rows.append({
            "config": name, "B": B, "L": cfg.L, "dim": cfg.dim, "heads": cfg.heads, "ffn": cfg.ffn_dim,
            "block_ms": ms, "block_tflops": cfg.block_flops() / (ms * 1e-3) / 1e12,
            "attention_tflops": a_tf, "gemm_tflops": g_tf,
            "attention_frac_of_measured_burst": None if a_tf is None else a_tf / burst,
            "gemm_frac_of_measured_burst": None if g_tf is None else g_tf / burst,
            "kernel_ms": {k: v[1] / iters for k, v in prof.items() if v[0]},
            "clocks": {"sm_mhz": ck.get("sm_mhz"), "reasons": ck.get("reasons")}})
        del w, wt, acts, ws
        torch.cuda.empty_cache()
    return rows


# ----------------------------------------------------------------- our arm
def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    from video_diffusion_transformer_fwd_b200 import configs, wan
    from video_diffusion_transformer_fwd_b200.step import CFGParallelStep, DenoiseStep, UlyssesStep, cfg_pairs

    torch.cuda.set_device(local_rank)
    dev = f"cuda:{local_rank}"
    cfg = configs.get(args.config)
    if args.ulysses:
        if args.fp8 or args.attn8 or args.cfg_parallel:
            raise SystemExit("--ulysses runs the bf16 blocks on the batched CFG pair")
        st = UlyssesStep(cfg, rank, world, group=dist.group.WORLD if world > 1 else None, seed=0, device=dev,
                         exchange=None if world > 1 else (lambda send, recv, group: recv.copy_(send)))
    elif args.cfg_parallel:
        if args.fp8 or args.attn8:
            raise SystemExit("--cfg-parallel runs the bf16 blocks")
        groups = [dist.new_group(pr) for pr in cfg_pairs(world)]     # every rank creates every group
        st = CFGParallelStep(cfg, rank % 2, groups[rank // 2], seed=1000 * (rank // 2), device=dev)
    else:
        st = DenoiseStep(cfg, seed=1000 * rank, device=dev, fp8=args.fp8, attn8=args.attn8)
    seqs = 1 if args.cfg_parallel else 2          # sequences of the CFG pair each rank runs
    # CFG pairs the job completes per step: one per rank (replicas), one per
    # rank pair (CFG-parallel), one for the whole group (Ulysses)
    pairs = 1 if args.ulysses else world * seqs // 2
    shards = world if args.ulysses else 1
    stream = torch.cuda.current_stream()

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        st.step()
    torch.cuda.synchronize()
    if wan.device_status() != wan.WAN_OK:
        raise RuntimeError("warm-up: " + wan.last_error())

    clocks = ClockSampler(list(range(world)) if rank == 0 else [local_rank]) if rank == 0 else None
    wan.check(wan.wan_profile_enable(1))
    barrier()
    torch.cuda.synchronize()
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    wall0 = time.perf_counter()
    t_start.record(stream)
    for _ in range(args.steps):
        st.step()
    t_end.record(stream)
    torch.cuda.synchronize()
    barrier()
    wall = time.perf_counter() - wall0
    ms_total = t_start.elapsed_time(t_end)
    prof = wan.profile_read()
    wan.check(wan.wan_profile_enable(0))
    clock_info = clocks.stop() if clocks else None
    if wan.device_status() != wan.WAN_OK:
        raise RuntimeError("timed region: " + wan.last_error())

    ms_max = max_over_ranks(ms_total, world, dev)

    # end to end: host (pinned) inputs in, result out, every step
    e2e = None
    if not args.no_e2e:
        x_h = torch.empty(st.x.shape, dtype=st.x.dtype, pin_memory=True)
        x_h.copy_(st.x)
        ctx_h = torch.empty(st.ctx.shape, dtype=st.ctx.dtype, pin_memory=True)
        ctx_h.copy_(st.ctx)
        e0_h = torch.empty(st.e0.shape, dtype=st.e0.dtype, pin_memory=True)
        e0_h.copy_(st.e0)
        out_h = torch.empty_like(x_h, pin_memory=True)
        h2d = x_h.numel() * x_h.element_size() + ctx_h.numel() * ctx_h.element_size() + \
            e0_h.numel() * e0_h.element_size()
        d2h = out_h.numel() * out_h.element_size()
        barrier()
        torch.cuda.synchronize()
        e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e_start.record(stream)
        for _ in range(args.steps):
            st.x.copy_(x_h, non_blocking=True)
            st.ctx.copy_(ctx_h, non_blocking=True)
            st.e0.copy_(e0_h, non_blocking=True)
            st.step()
            out_h.copy_(st.x, non_blocking=True)
        e_end.record(stream)
        torch.cuda.synchronize()
        barrier()
        e_ms = max_over_ranks(e_start.elapsed_time(e_end), world, dev)
        e2e = {"value": per_block_ms(e_ms, args.steps, cfg.blocks, pairs), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}

    if rank != 0:
        return
    value = per_block_ms(ms_max, args.steps, cfg.blocks, pairs)
    peaks, peak_src = read_peaks()
    blocks_run = args.steps * cfg.blocks
    import dataclasses
    c2 = dataclasses.replace(cfg, batch=seqs)
    attn_n, attn_ms = prof["attn_self"]
    gemm_n, gemm_ms = prof["gemm_tc"]
    attn_flops_launch = c2.self_attn_flops() / shards          # this rank's heads
    # this rank's GEMM work: its token rows, and the replicated cross K/V projection
    gemm_flops_block = (c2.gemm_flops() - seqs * 4.0 * cfg.text_len * cfg.dim * cfg.dim) / shards \
        + seqs * 4.0 * cfg.text_len * cfg.dim * cfg.dim
    attn_tflops = attn_flops_launch * attn_n / (attn_ms * 1e-3) / 1e12 if attn_ms > 0 else None
    gemm_tflops = gemm_flops_block * blocks_run / (gemm_ms * 1e-3) / 1e12 if gemm_ms > 0 else None
    # dominant kernel class by device time
    dom = max(prof.items(), key=lambda kv: kv[1][1])[0]
    peak_sust = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    roofline = None
    if dom == "attn_self" and attn_n:
        avg_ms = attn_ms / attn_n
        tr = TRAFFIC.get("attn_self")
        traffic = None
        if tr and not args.attn8 and shards == 1 and tr.get("source_sha") == source_hash(*ATTN_SOURCES):
            traffic = tr["bytes_per_launch"] * seqs / 2     # recorded for the B = 2 launch
        apk = peak_sust * (2.0 if args.attn8 else 1.0)
        roofline = {"kernel": ("attn8 (8-bit self-attention incl. its quantization passes" if args.attn8 else
                               "attn_tc (self-attention") + f", B={seqs}, L={cfg.L}, {cfg.heads // shards} heads, d=128)",
                    "bound": "tensor", "achieved": attn_flops_launch / (avg_ms * 1e-3) / 1e12,
                    "peak": apk, "unit": "TFLOP/s",
                    "frac": attn_flops_launch / (avg_ms * 1e-3) / 1e12 / apk,
                    "peak_source": f"{peak_src} bf16 sustained (kernel timed inside a long step)"
                                   + (" x 2 (8-bit / bf16 nominal ratio)" if args.attn8 else ""),
                    "traffic": traffic, "avg_launch_ms": avg_ms,
                    "algorithmic_flops_per_launch": attn_flops_launch}
    elif dom == "gemm_tc" and gemm_n:
        gpk = peak_sust * (2.0 if (args.fp8 or args.attn8) else 1.0)
        roofline = {"kernel": "gemm_tc (all block GEMMs)", "bound": "tensor", "achieved": gemm_tflops,
                    "peak": gpk, "unit": "TFLOP/s", "frac": gemm_tflops / gpk,
                    "peak_source": f"{peak_src} bf16 sustained" + (" x 2 (fp8 / bf16 nominal ratio)" if (args.fp8 or args.attn8) else ""),
                    "traffic": None}
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": False,
        "scaling": "strong" if args.ulysses else "weak", "vs_baseline": None,
        "dtype": ("fp8 e4m3 GEMMs, int8 QK^T / e4m3 PV self-attention" if args.attn8 else
                  "fp8 e4m3 GEMMs (per-token / per-tensor scales), bf16 attention" if args.fp8 else "bf16"),
        "data": "synthetic",
        "impl": "ours",
        "config": workload_config(cfg, world, args.cfg_parallel, args.ulysses),
        "attention_tflops": attn_tflops, "gemm_tflops": gemm_tflops,
        "attention_frac_of_2250": None if attn_tflops is None else attn_tflops / 2250.0,
        "gemm_frac_of_2250": None if gemm_tflops is None else gemm_tflops / 2250.0,
        "gemm_frac_of_fp8_4500": None if (gemm_tflops is None or not (args.fp8 or args.attn8)) else gemm_tflops / 4500.0,
        "kernel_ms_per_step": {k: v[1] / args.steps for k, v in prof.items() if v[0]},
        "gpu_launches": sum(v[0] for v in prof.values()),
        "roofline": roofline,
        "clocks": clock_info,
        "wall_s_timed": wall,
        "e2e": e2e,
    }
    if not args.no_per_config:
        del st
        torch.cuda.empty_cache()
        line["per_config"] = per_config_rows(dev, peaks)
    if world == 1 and not args.no_cpu_baseline:
        ms, detail, measured = OracleSample(cfg, seed=0, fp8=args.fp8 or args.attn8).run()
        full = oracle_full_block(configs.get("1.3b-short"), cpu_cores())
        for row in line.get("per_config", []):
            if row["config"] == full["config"] and row["B"] == 1:
                full["gpu_block_ms"] = row["block_ms"]
        line["cpu_baseline"] = {"value": ms, "unit": UNIT, "cores": cpu_cores(),
                                "blas_threads": blas_threads(), "kind": "oracle", "estimated": True,
                                "measured": measured, "sample": detail, "measured_full_block": full}
    print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device(f"cuda:{local_rank}"))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
