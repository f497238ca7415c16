#!/usr/bin/env python
"""Benchmark of the Wan DiT hot path on B200.

One step = one pass of the whole hot path over one batch of synthetic input
of the named workload: 3D RoPE (fused into the self-attention tile stage, or
as its own pass with --rope pre), full spatio-temporal self-attention,
length-masked cross-attention to 512 text tokens (queried by the
self-attention output), and the fused CFG + Euler step on the latent, with
the token grid and sigma schedule from the library's host calls.

Metric: self-attention TFLOP/s (4 * B * heads * L^2 * 128 FLOP per step)
over the whole step time; also reported against the measured dense bf16
peak.  Inputs (Q, K, V: 774 MB each at 75,600 tokens x 40 heads) are larger
than L2, so no flush is needed between steps.

Usage:  python bench.py [--gpus N] [--steps K] [--warmup W]
        [--workload 720p-81f|480p-81f|...] [--rope fused|pre]
        [--impl wan|reference]
Multi-GPU (weak scaling, independent problem per rank, no data-path
collective): python -m torch.distributed.run --nproc-per-node N bench.py
--gpus N ...
"""

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=10)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--workload", default="720p-81f")
    p.add_argument("--rope", choices=["fused", "fused-q", "pre"],
                   default="pre",
                   help="pre: the RoPE pass rotates Q and K before the "
                        "attention; fused: the attention kernel rotates Q "
                        "and K in its tile stage (--attn tiles); fused-q: "
                        "the pass rotates K alone and the kernel rotates Q "
                        "in its tile stage (with --attn pair, fused means "
                        "fused-q)")
    p.add_argument("--attn", choices=["tiles", "pair"], default="tiles",
                   help="self-attention kernel: two 128-row tiles per CTA, "
                        "or CTA pairs (one MMA over two SMs)")
    p.add_argument("--impl", choices=["wan", "reference"], default="wan")
    p.add_argument("--parallel", choices=["replicas", "ulysses"],
                   default="replicas",
                   help="N > 1: independent problems per rank (replicas), "
                        "or one problem split by Ulysses head sharding")
    p.add_argument("--no-points", action="store_true",
                   help="skip the per-workload self-attention launch points")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-hbm", action="store_true",
                   help="skip the HBM-bound kernel rooflines")
    p.add_argument("--no-causal", action="store_true",
                   help="skip the block-causal attention measurement")
    p.add_argument("--hbm-elems", type=int, default=1 << 30,
                   help="fp32 elements per buffer of the fm_step roofline")
    p.add_argument("--cpu-rows", type=int, default=4096,
                   help="query rows of one head timed on the oracle")
    return p.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0,
                "bf16_tflops_sustained": 1400.0}, "fallback"


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info()
             if i.get("user_api") == "blas"]
        if n:
            return max(n)
    except Exception:
        pass
    return os.cpu_count() or 1


class ClockSampler:
    """nvidia-smi clock / throttle-reason sampling during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,"
              "clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(device_index),
                 "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                 "sw_power_cap"]
        for line in out.splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for name, val in zip(names, parts[3:7]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "samples": len(sm), "reasons": sorted(reasons)}


# ------------------------------------------------------------- reference ---

def cpu_oracle_sample(w, rows, seed_rank=0):
    """Time the oracle (fp64 CPU) on `rows` query rows of one head of the
    workload: 3D RoPE of that head's Q rows and all K, then softmax
    attention against all L keys.  Returns (seconds, flops, sample text)."""
    import numpy as np
    from oracle import attention as oattn
    from oracle import grid as ogrid
    from oracle import rope as orope
    from video_diffusion_transformer_self_b200 import inputs

    grid = ogrid.token_grid(w.frames, w.height, w.width)
    L = ogrid.token_count(grid)
    shape = (1, L, 1, 128)
    q = inputs.randn_bf16(shape, inputs.seed_for(w.index, "q")).double().numpy()
    k = inputs.randn_bf16(shape, inputs.seed_for(w.index, "k")).double().numpy()
    v = inputs.randn_bf16(shape, inputs.seed_for(w.index, "v")).double().numpy()
    sel = inputs.sample_rows(L, rows, inputs.seed_for(w.index, "rows")).numpy()
    t0 = time.perf_counter()
    qr = orope.rope3d(q, grid)[:, sel]
    kr = orope.rope3d(k, grid)
    oattn.attention(qr, kr, v, 1.0 / math.sqrt(128))
    dt = time.perf_counter() - t0
    flops = 4.0 * len(sel) * L * 128
    text = ("%d sampled query rows x 1 head x %d keys (RoPE + fp64 softmax "
            "attention), %s" % (len(sel), L, w.name))
    return dt, flops, text


def run_reference(args, w, rank, world):
    if rank != 0:
        return
    rows = max(16, args.cpu_rows // 32)
    for _ in range(args.warmup):
        cpu_oracle_sample(w, rows)
    total_t, total_f, text = 0.0, 0.0, ""
    for _ in range(args.steps):
        dt, fl, text = cpu_oracle_sample(w, rows)
        total_t += dt
        total_f += fl
    tflops = total_f / total_t / 1e12
    cores = blas_threads()
    line = {
        "impl": "reference",
        "metric": "self-attn TFLOP/s",
        "value": tflops,
        "unit": "TFLOP/s",
        "n_gpus": args.gpus,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": 1e3 * total_t / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": w.name, "sample": text},
        "cpu_baseline": {"value": tflops, "unit": "TFLOP/s", "cores": cores,
                         "kind": "oracle", "sample": text},
        "e2e": {"value": tflops, "unit": "TFLOP/s",
                "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------- wan ---

# DRAM bytes per algorithmic byte (Q, K, V read once, O written once) of the
# self-attention kernel, from the ncu capture of the 480p-81f launch:
# 812.18 MB measured (626.39 read + 185.78 written) for 805.31 MB
# algorithmic.  The kernel's DRAM traffic grows in proportion to
# B * L * heads, so a launch's traffic is this ratio times its algorithmic
# bytes.
ATTN_DRAM_PER_ALG_BYTE = 812.18 / 805.31


def rank_seed_offset(rank):
    """Seed offset of a rank's inputs: every rank runs its own problem."""
    return 7919 * int(rank)


def max_over_ranks(values, dist=None, device=None):
    """Element-wise MAX of a list of floats over all ranks (identity at 1)."""
    import torch
    if dist is None:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64,
                     device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def job_throughput(world, flops_per_step, steps, max_ms):
    """Whole-job TFLOP/s: every rank's FLOPs over the slowest rank's time."""
    return world * flops_per_step * steps / (max_ms / 1e3) / 1e12


def hbm_rooflines(dev, g, L, H, n_lat, peak_gbs, n=1 << 30, reps=20):
    """Achieved bandwidth of the HBM-bound kernels, timed alone with CUDA
    events: the fused CFG + Euler step and the fused UniPC stop on n-element
    fp32 buffers (default 2^30: 16 GiB / 36 GiB of traffic per call, far above
    L2), the RoPE, QK-Norm + RoPE, AdaLN and gated-residual passes on the
    workload's tensors; plus the Euler step on the workload's own latent,
    timed cold (L2 flushed by a 512 MiB write before every call)."""
    import torch

    from video_diffusion_transformer_self_b200 import wan

    gen = torch.Generator(device=dev)
    gen.manual_seed(4242)
    out = {}
    x = torch.randn(n, device=dev, generator=gen)
    c = torch.randn(n, device=dev, generator=gen)
    u = torch.randn(n, device=dev, generator=gen)
    for _ in range(3):
        wan.fm_step(x, c, u, 4.0, 0.5, 0.49)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record()
    for _ in range(reps):
        wan.fm_step(x, c, u, 4.0, 0.5, 0.49)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / reps
    gbs = 16.0 * n / (ms / 1e3) / 1e9
    out["fm_step_cfg"] = {"elements": n, "bytes_per_call": 16 * n,
                          "ms": ms, "achieved_gbs": gbs, "peak_gbs": peak_gbs,
                          "frac": gbs / peak_gbs}
    # UniPC stop 20 of the 40-step shift-12 schedule: CFG, order-2 corrector
    # and predictor; 36 B per element (x, x_corr, m_(i-1), m_(i-2), v_cond,
    # v_uncond read; x, x_corr, m_i written, m_i over m_(i-2)).
    xc = torch.randn(n, device=dev, generator=gen)
    m1 = torch.randn(n, device=dev, generator=gen)
    m2 = torch.randn(n, device=dev, generator=gen)
    sig = wan.fm_sigmas(40, 12.0)
    for _ in range(3):
        wan.unipc_step(x, xc, m1, m2, m2, c, u, 4.0, sig, 20)
    torch.cuda.synchronize()
    e0.record()
    for _ in range(reps):
        wan.unipc_step(x, xc, m1, m2, m2, c, u, 4.0, sig, 20)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / reps
    gbs = 36.0 * n / (ms / 1e3) / 1e9
    out["unipc_step_cfg"] = {"elements": n, "bytes_per_call": 36 * n,
                             "stop": 20, "corrector_order": 2,
                             "ms": ms, "achieved_gbs": gbs,
                             "peak_gbs": peak_gbs, "frac": gbs / peak_gbs}
    del x, c, u, xc, m1, m2
    q = torch.randn(1, L, H, 128, device=dev, generator=gen).to(torch.bfloat16)
    k = torch.randn(1, L, H, 128, device=dev, generator=gen).to(torch.bfloat16)
    table = wan.rope3d_table(g)
    for _ in range(3):
        wan.rope3d_qk(q, k, g, table)
    torch.cuda.synchronize()
    e0.record()
    for _ in range(reps):
        wan.rope3d_qk(q, k, g, table)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / reps
    nbytes = 4 * q.numel() * 2
    gbs = nbytes / (ms / 1e3) / 1e9
    out["rope3d_qk"] = {"tokens": L, "heads": H, "bytes_per_call": nbytes,
                        "ms": ms, "achieved_gbs": gbs, "peak_gbs": peak_gbs,
                        "frac": gbs / peak_gbs}
    # QK-Norm + RoPE on the same Q / K (same traffic as the RoPE pass)
    wq = torch.randn(H * 128, device=dev, generator=gen)
    wk = torch.randn(H * 128, device=dev, generator=gen)

    def timed(fn):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        e0.record()
        for _ in range(reps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / reps

    ms = timed(lambda: wan.qk_norm_rope(q, k, wq, wk, g, table))
    out["qk_norm_rope"] = {"bytes_per_call": nbytes, "ms": ms,
                           "achieved_gbs": nbytes / (ms / 1e3) / 1e9,
                           "peak_gbs": peak_gbs,
                           "frac": nbytes / (ms / 1e3) / 1e9 / peak_gbs}
    # Ulysses layout move before the exchange on 8 ranks: Q's 40 heads split
    # into 8 groups of 5 (rows of 5 x 256 B), every byte read and written once
    P = 8
    if H % P == 0:
        send = torch.empty_like(q)
        rb = (H // P) * 128 * 2
        ms = timed(lambda: wan.transpose_blocks(q, send, L, P, rb))
        nb = 2 * q.numel() * 2
        out["ulysses_pack_8"] = {"bytes_per_call": nb, "ms": ms,
                                 "achieved_gbs": nb / (ms / 1e3) / 1e9,
                                 "peak_gbs": peak_gbs,
                                 "frac": nb / (ms / 1e3) / 1e9 / peak_gbs}
        del send
    del q, k
    # AdaLN modulate and gated residual on the fp32 residual stream
    D = H * 128
    x = torch.randn(1, L, D, device=dev, generator=gen)
    sh = torch.randn(1, D, device=dev, generator=gen)
    sc = torch.randn(1, D, device=dev, generator=gen)
    yb = torch.empty(1, L, D, device=dev, dtype=torch.bfloat16)
    ms = timed(lambda: wan.adaln_modulate(x, sh, sc, yb))
    nb = x.numel() * 6
    out["adaln_modulate"] = {"bytes_per_call": nb, "ms": ms,
                             "achieved_gbs": nb / (ms / 1e3) / 1e9,
                             "peak_gbs": peak_gbs,
                             "frac": nb / (ms / 1e3) / 1e9 / peak_gbs}
    ms = timed(lambda: wan.gated_residual(x, yb, sh))
    nb = x.numel() * 10
    out["gated_residual"] = {"bytes_per_call": nb, "ms": ms,
                             "achieved_gbs": nb / (ms / 1e3) / 1e9,
                             "peak_gbs": peak_gbs,
                             "frac": nb / (ms / 1e3) / 1e9 / peak_gbs}
    del x, yb
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    xl = torch.randn(n_lat, device=dev, generator=gen)
    cl = torch.randn(n_lat, device=dev, generator=gen)
    ul = torch.randn(n_lat, device=dev, generator=gen)
    tot = 0.0
    cold_reps = 100
    for i in range(cold_reps + 3):
        flush.fill_(i & 255)
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        wan.fm_step(xl, cl, ul, 4.0, 0.5, 0.49)
        b.record()
        torch.cuda.synchronize()
        if i >= 3:
            tot += a.elapsed_time(b)
    ms = tot / cold_reps
    out["fm_step_latent_cold"] = {"elements": n_lat, "ms": ms,
                                  "calls": cold_reps,
                                  "achieved_gbs": 16.0 * n_lat / (ms / 1e3)
                                  / 1e9, "l2": "flushed before each call"}
    return out


def causal_rooflines(dev, peak_tflops, reps=5):
    """Block-causal (Self Forcing chunk) attention at 480p-165f: 42 x 30 x
    52 = 65,520 tokens, 40 heads, chunks of 3 latent frames (4,680 tokens).
    Times the full-sequence call and the KV-cache step of the last chunk
    (4,680 queries against all 65,520 keys) as the binding runs them by
    default (block_causal_default_pair: the two-tile kernel for the full
    sequence, the CTA-pair kernel for the KV-cache step), and beside them
    the other kernel: the full sequence on the CTA-pair kernel, the
    KV-cache step on the two-tile kernel with the key ranges
    wan_block_causal_attn_splits picks (plus the combining pass) and with
    one range.  The calls are timed in turn, one launch of each per round,
    and each reports its median.  FLOPs count only visible keys:
    4 * 128 * heads * sum over queries of the key limit."""
    import numpy as np
    import torch

    from video_diffusion_transformer_self_b200 import wan
    from video_diffusion_transformer_self_b200.workloads import WORKLOADS

    w = WORKLOADS[4]
    _, g = wan.token_grid(w.frames, w.height, w.width)
    L, H = g.F * g.H * g.W, w.heads
    chunk = 3 * g.H * g.W
    gen = torch.Generator(device=dev)
    gen.manual_seed(5151)
    q = torch.randn(1, L, H, 128, device=dev, generator=gen).to(torch.bfloat16)
    k = torch.randn(1, L, H, 128, device=dev, generator=gen).to(torch.bfloat16)
    v = torch.randn(1, L, H, 128, device=dev, generator=gen).to(torch.bfloat16)
    o = torch.empty_like(q)

    def visible(lq, off):
        a = off + np.arange(lq, dtype=np.int64)
        return float(np.minimum(L, (a // chunk + 1) * chunk).sum())

    # CTA pairs resident at once (clusters of two CTAs share a GPC, so an SM
    # left over in a GPC with an odd number of them runs none): the pair
    # kernel's timings depend on it from box to box
    out = {"workload": "480p-165f", "tokens": L, "heads": H,
           "chunk_tokens": chunk,
           "pair_resident_clusters": wan.attn_pair_resident_clusters(),
           "sm_count": torch.cuda.get_device_properties(
               dev).multi_processor_count}
    ql = q[:, L - chunk:].contiguous()
    n_split = wan.block_causal_splits(1, chunk, L, H, chunk, L - chunk)
    ws = torch.empty(max(1, wan.block_causal_workspace_bytes(
        1, chunk, H, n_split)), dtype=torch.uint8, device=dev)
    # (name, queries, offset, pair kernel or None for the binding's
    # default, key ranges)
    cases = (("full_sequence", q, 0, None, 1),
             ("kv_cache_last_chunk", ql, L - chunk, None, 1),
             ("full_sequence_pair", q, 0, True, 1),
             ("kv_cache_last_chunk_two_tile_key_ranges", ql, L - chunk,
              False, n_split),
             ("kv_cache_last_chunk_two_tile_one_range", ql, L - chunk, False,
              1))
    calls = []
    for name, qq, off, pair, sp in cases:
        oo = o[:, :qq.shape[1]] if off else o

        def call(qq=qq, oo=oo, off=off, pair=pair, sp=sp):
            wan.block_causal_attn(qq, k, v, oo, chunk, off, pair=pair,
                                  split=sp if sp > 1 else None,
                                  workspace=ws if sp > 1 else None)
        for _ in range(2):
            call()
        calls.append(call)
    times = [[] for _ in cases]
    for _ in range(reps):
        for i, call in enumerate(calls):
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize()
            e0.record()
            call()
            e1.record()
            torch.cuda.synchronize()
            times[i].append(e0.elapsed_time(e1))
    for (name, qq, off, pair, sp), t in zip(cases, times):
        if pair is None:
            pair = wan.block_causal_default_pair(1, qq.shape[1], L, H, chunk,
                                                 off)
        ms = float(np.median(t))
        fl = 4.0 * 128 * H * visible(qq.shape[1], off)
        out[name] = {"ms": ms, "tflops": fl / (ms / 1e3) / 1e12,
                     "frac_of_sustained_peak": fl / (ms / 1e3) / 1e12
                     / peak_tflops,
                     "kernel": "attn_pair_kernel" if pair else
                     "attn_fwd_kernel", "key_ranges": sp}
    if wan.device_status() != 0:
        raise RuntimeError("device timeout in the block-causal timings")
    return out


def attn_points(dev, pk, reps=10):
    """Self-attention launch alone at the two token counts of the metric:
    480p-81f (B 2 x 12 heads x 32,760 tokens) and 720p-81f (B 1 x 40 heads
    x 75,600 tokens).  Two-tile kernel with Q / K rotated beforehand ("pre"),
    with the rotation of both fused into its tile stage ("fused"), and with
    Q rotated in its tile stage, K by the pass ("fused_q"; the launch timed
    is the attention alone, the K pass moves half the bytes of the full
    pass); the CTA-pair kernel with Q / K rotated beforehand ("pair_pre") and with Q
    rotated in its tile stage, K by the pass ("pair_fused_q"; the launch
    timed here is the attention alone).  Each form runs 3 warm-up launches,
    then `reps` back-to-back launches with a CUDA event on the launching
    stream between consecutive ones (no idle gap, so each form is timed at
    the clocks its own steady power draw allows), and reports the median of
    those launch times (and their mean).  Q, K and V are each larger than
    L2 at 720p (774 MB) and together above it at 480p (3 x 201 MB).  FLOPs
    4 * B * heads * L^2 * 128."""
    import numpy as np
    import torch

    from video_diffusion_transformer_self_b200 import wan
    from video_diffusion_transformer_self_b200.workloads import by_name

    sustained = float(pk.get("bf16_tflops_sustained", 1400.0))
    burst = float(pk.get("bf16_tflops", 1590.0))
    gen = torch.Generator(device=dev)
    gen.manual_seed(6161)
    stream = torch.cuda.current_stream()
    out = {}
    for name in ("480p-81f", "720p-81f"):
        w = by_name(name)
        _, g = wan.token_grid(w.frames, w.height, w.width)
        L, B, H = g.F * g.H * g.W, w.batch, w.heads
        shape = (B, L, H, 128)
        q = torch.randn(shape, device=dev, generator=gen).to(torch.bfloat16)
        k = torch.randn(shape, device=dev, generator=gen).to(torch.bfloat16)
        v = torch.randn(shape, device=dev, generator=gen).to(torch.bfloat16)
        o = torch.empty_like(q)
        table = wan.rope3d_table(g)
        fl = 4.0 * B * H * L * L * 128
        point = {"tokens": L, "batch": B, "heads": H, "flops": fl}
        wan.rope3d_qk(None, k, g, table)  # k rotated once, for the pair
        calls = {
            "pre": lambda: wan.self_attn(q, k, v, o, g),
            "fused": lambda: wan.self_attn(q, k, v, o, g, table=table),
            "fused_q": lambda: wan.self_attn_rope_q(q, k, v, o, g, table),
            "pair_pre": lambda: wan.self_attn_pair(q, k, v, o, g),
            "pair_fused_q": lambda: wan.self_attn_pair(q, k, v, o, g,
                                                       table_q=table),
        }
        times = {}
        for mode, call in calls.items():
            for _ in range(3):
                call()
            ev = [torch.cuda.Event(enable_timing=True)
                  for _ in range(reps + 1)]
            torch.cuda.synchronize()
            ev[0].record(stream)
            for i in range(reps):
                call()
                ev[i + 1].record(stream)
            torch.cuda.synchronize()
            times[mode] = [ev[i].elapsed_time(ev[i + 1]) for i in range(reps)]
        for mode, t in times.items():
            ms = float(np.median(t))
            tf = fl / (ms / 1e3) / 1e12
            point[mode] = {"median_launch_ms": ms,
                           "mean_launch_ms": float(np.mean(t)),
                           "launches": len(t), "tflops": tf,
                           "frac_of_measured_sustained": tf / sustained,
                           "frac_of_measured_burst": tf / burst,
                           "frac_of_datasheet_2250": tf / 2250.0}
        if wan.device_status() != 0:
            raise RuntimeError("device timeout in the attention points")
        out[name] = point
        del q, k, v, o
    return out


def cross_roofline(B, L, H, Lk, lens, ms, peak_tflops, peak_gbs):
    """Cross-attention launch of the timed step (CUDA events around it).
    FLOPs count the true text lengths, 4 * L * len_b * 128 * H per batch row
    (and, for reference, the padded Lk); bytes are Q read and O written
    (B * L * H * 256 each) plus the len_b valid K and V rows.  Its
    arithmetic intensity (about len_b FLOP per byte) is near the B200 ridge,
    so both fractions are given."""
    fl = sum(4.0 * L * n * 128 * H for n in lens)
    fl_pad = 4.0 * B * L * Lk * 128 * H
    nb = 2.0 * B * L * H * 256 + sum(2.0 * n * H * 256 for n in lens)
    tf = fl / (ms / 1e3) / 1e12
    gbs = nb / (ms / 1e3) / 1e9
    return {"kernel": "attn_fwd_kernel cross-attention", "ms": ms,
            "text_lens": list(lens), "flops": fl, "bytes": nb,
            "tflops": tf, "tflops_padded_lk": fl_pad / (ms / 1e3) / 1e12,
            "frac_of_sustained_tensor_peak": tf / peak_tflops,
            "gbs": gbs, "frac_of_hbm_peak": gbs / peak_gbs,
            "intensity_flop_per_byte": fl / nb}


def run_wan(args, w, rank, world, local_rank):
    import numpy as np
    import torch

    from video_diffusion_transformer_self_b200 import inputs, wan

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    stream = torch.cuda.current_stream()

    lat, g = wan.token_grid(w.frames, w.height, w.width)
    L = g.F * g.H * g.W
    B, H = w.batch, w.heads
    n_lat = int(np.prod(lat)) * B
    sigmas = wan.fm_sigmas(w.steps, w.shift)
    seed_off = rank_seed_offset(rank)

    def sd(role):
        return inputs.seed_for(w.index, role) + seed_off

    shape = (B, L, H, 128)
    ctx_shape = (B, w.text_tokens, H, 128)
    host = {
        "q": inputs.randn_bf16(shape, sd("q")),
        "k": inputs.randn_bf16(shape, sd("k")),
        "v": inputs.randn_bf16(shape, sd("v")),
        "k_ctx": inputs.randn_bf16(ctx_shape, sd("k_ctx")),
        "v_ctx": inputs.randn_bf16(ctx_shape, sd("v_ctx")),
        "x": inputs.randn_f32((n_lat,), sd("x")),
        "v_cond": inputs.randn_f32((n_lat,), sd("v_cond")),
        "v_uncond": inputs.randn_f32((n_lat,), sd("v_uncond")),
    }
    lens = inputs.uniform_int(B, w.text_len_lo, w.text_len_hi,
                              sd("lens")).tolist()
    d = {kk: t.to(dev) for kk, t in host.items()}
    o = torch.empty_like(d["q"])
    oc = torch.empty_like(d["q"])
    table = wan.rope3d_table(g)
    guide = 4.0
    flops_self = 4.0 * B * H * L * L * 128

    ev_pairs = []
    ev_cross = []

    rope_q = args.rope == "fused-q" or (args.rope == "fused"
                                         and args.attn == "pair")

    def rope_pass(ds, strm=None):
        # the stand-alone RoPE pass: Q and K (--rope pre), or K alone when
        # the attention kernel rotates Q in its tile stage
        if args.rope == "pre":
            wan.rope3d_qk(ds["q"], ds["k"], g, table, stream=strm)
        elif rope_q:
            wan.rope3d_qk(None, ds["k"], g, table, stream=strm)

    def attention(ds, out, strm=None):
        if args.attn == "pair":
            wan.self_attn_pair(ds["q"], ds["k"], ds["v"], out, g,
                               table_q=table if rope_q else None,
                               stream=strm)
        elif rope_q:
            wan.self_attn_rope_q(ds["q"], ds["k"], ds["v"], out, g, table,
                                 stream=strm)
        else:
            wan.self_attn(ds["q"], ds["k"], ds["v"], out, g,
                          table=table if args.rope == "fused" else None,
                          stream=strm)

    def step(i, timed):
        s0, s1 = sigmas[i % w.steps], sigmas[i % w.steps + 1]
        rope_pass(d)
        if timed:
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
        attention(d, o)
        if timed:
            e1.record(stream)
            ev_pairs.append((e0, e1))
        wan.cross_attn(o, d["k_ctx"], d["v_ctx"], oc, lens)
        if timed:
            e2 = torch.cuda.Event(enable_timing=True)
            e2.record(stream)
            ev_cross.append((e1, e2))
        wan.fm_step(d["x"], d["v_cond"], d["v_uncond"], guide, s0, s1)

    launches_per_step = 3 + (1 if args.rope == "pre" or rope_q else 0)

    dist = None
    if world > 1:
        import torch.distributed as dist_mod
        dist = dist_mod

    def barrier():
        if dist is not None:
            dist.barrier(device_ids=[local_rank])

    for i in range(args.warmup):
        step(i, False)
    torch.cuda.synchronize()
    if wan.device_status() != 0:
        raise RuntimeError("device timeout during warm-up")

    clocks = ClockSampler(local_rank) if rank == 0 else None
    barrier()
    torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for i in range(args.steps):
        step(i, True)
    t_end.record(stream)
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop() if clocks else None
    ms = t_start.elapsed_time(t_end)
    if wan.device_status() != 0:
        raise RuntimeError("device timeout during the timed steps")
    # self-attention launch time (the RoPE pass of --rope pre excluded)
    attn_ms = [a.elapsed_time(b) for a, b in ev_pairs]
    attn_avg = sum(attn_ms) / len(attn_ms)
    cross_ms = [a.elapsed_time(b) for a, b in ev_cross]
    cross_avg = sum(cross_ms) / len(cross_ms)
    ms, attn_avg, cross_avg = max_over_ranks([ms, attn_avg, cross_avg], dist,
                                             dev)

    # ----- end to end: host buffers in, results out, every step -----
    # Each step copies its inputs from pinned host memory and reads back its
    # results (cross-attention output and the stepped latent).  Two device
    # buffer sets and separate H2D / compute / D2H streams let the copies of
    # step i+1 run under the kernels of step i.
    e2e = None
    if not args.no_e2e:
        pin = {kk: t.pin_memory() for kk, t in host.items()}
        outs_h = [torch.empty(oc.shape, dtype=oc.dtype).pin_memory()
                  for _ in range(2)]
        xs_h = [torch.empty(n_lat, dtype=torch.float32).pin_memory()
                for _ in range(2)]
        sets = [d, {kk: torch.empty_like(t) for kk, t in d.items()}]
        ocs = [oc, torch.empty_like(oc)]
        os_ = [o, torch.empty_like(o)]
        h2d_s = torch.cuda.Stream(device=dev)
        d2h_s = torch.cuda.Stream(device=dev)
        comp = stream
        h2d = sum(t.numel() * t.element_size() for t in pin.values())
        d2h = outs_h[0].numel() * 2 + xs_h[0].numel() * 4

        def run_steps(n_steps, start_ev=None):
            freed = [None, None]    # compute of the last step using set b
            read = [None, None]     # D2H of the last results of set b
            for i in range(n_steps):
                bi = i & 1
                ds = sets[bi]
                with torch.cuda.stream(h2d_s):
                    if freed[bi] is not None:
                        h2d_s.wait_event(freed[bi])
                    if read[bi] is not None:  # x of set b is read back
                        h2d_s.wait_event(read[bi])
                    if i == 0 and start_ev is not None:
                        start_ev.record(h2d_s)
                    for kk, t in pin.items():
                        ds[kk].copy_(t, non_blocking=True)
                    ready = torch.cuda.Event()
                    ready.record(h2d_s)
                comp.wait_event(ready)
                if read[bi] is not None:
                    comp.wait_event(read[bi])
                s0, s1 = sigmas[i % w.steps], sigmas[i % w.steps + 1]
                rope_pass(ds, comp)
                attention(ds, os_[bi], comp)
                wan.cross_attn(os_[bi], ds["k_ctx"], ds["v_ctx"], ocs[bi],
                               lens, stream=comp)
                wan.fm_step(ds["x"], ds["v_cond"], ds["v_uncond"], guide, s0,
                            s1, stream=comp)
                done = torch.cuda.Event()
                done.record(comp)
                freed[bi] = done
                with torch.cuda.stream(d2h_s):
                    d2h_s.wait_event(done)
                    outs_h[bi].copy_(ocs[bi], non_blocking=True)
                    xs_h[bi].copy_(ds["x"], non_blocking=True)
                    rd = torch.cuda.Event()
                    rd.record(d2h_s)
                    read[bi] = rd
            end_ev = torch.cuda.Event(enable_timing=True)
            end_ev.record(d2h_s)
            return end_ev

        run_steps(2)
        torch.cuda.synchronize()
        barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = run_steps(args.steps, start_ev=e0)
        torch.cuda.synchronize()
        barrier()
        e2e_ms = max_over_ranks([e0.elapsed_time(e1)], dist, dev)[0]
        e2e = {"value": job_throughput(world, flops_self, args.steps, e2e_ms),
               "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h,
               "ms_per_step": e2e_ms / args.steps,
               "pipelined": "H2D of step i+1 overlaps the kernels of step i"}

    if rank != 0:
        return
    pk, pk_kind = peaks()
    peak = float(pk.get("bf16_tflops_sustained", 1400.0))
    value = job_throughput(world, flops_self, args.steps, ms)
    achieved = flops_self / (attn_avg / 1e3) / 1e12
    line = {
        "metric": "self-attn TFLOP/s",
        "value": value,
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {
            "workload": w.name, "batch": B, "heads": H, "seq_len": L,
            "grid": [g.F, g.H, g.W], "text_tokens": w.text_tokens,
            "text_lens": lens, "latent": list(lat), "rope": args.rope,
            "attn_kernel": args.attn,
            "parallelism": "replicas" if world > 1 else "single",
            "l2": "inputs larger than L2 (Q/K/V %.0f MB each)"
                  % (B * L * H * 256 / 1e6),
        },
        "frac_of_peak": {
            "dense_bf16_datasheet_2250": value / 2250.0,
            "measured_burst": value / float(pk.get("bf16_tflops", 1590.0)),
            "measured_sustained": value / peak,
        },
        "roofline": {
            "kernel": ("attn_pair_kernel (CTA pairs)" if args.attn == "pair"
                       else "attn_fwd_kernel (two tiles per CTA)")
            + " self-attention" + {"pre": "", "fused": " with fused RoPE",
                                   "fused-q": " with Q rotated in the tile "
                                   "stage"}[args.rope],
            "bound": "tensor", "achieved": achieved, "peak": peak,
            "unit": "TFLOP/s", "frac": achieved / peak,
            "traffic": ATTN_DRAM_PER_ALG_BYTE * 4 * B * L * H * 256,
            "traffic_source": "ncu dram read+write of the 480p-81f launch, "
                              "scaled by bytes processed",
            "peak_kind": pk_kind + " sustained bf16 (kernel timed inside a "
                                   "long step)",
            "avg_launch_ms": attn_avg,
        },
        "cross_attn": cross_roofline(B, L, H, w.text_tokens, lens, cross_avg,
                                     peak, float(pk.get("hbm_gbs", 6650.0))),
        "gpu_launches": launches_per_step * args.steps,
        "e2e": e2e,
        "clocks": clk,
    }
    if not args.no_hbm and world == 1:
        line["hbm_kernels"] = hbm_rooflines(
            dev, g, L, H, n_lat, float(pk.get("hbm_gbs", 6650.0)),
            n=args.hbm_elems)
    if not args.no_causal and world == 1:
        line["block_causal"] = causal_rooflines(dev, peak)
    if not args.no_points and world == 1:
        line["metric_points"] = attn_points(dev, pk)
    if not args.no_cpu_baseline and world == 1:
        dt, fl, text = cpu_oracle_sample(w, args.cpu_rows)
        line["cpu_baseline"] = {"value": fl / dt / 1e12, "unit": "TFLOP/s",
                                "cores": blas_threads(), "kind": "oracle",
                                "sample": text, "seconds": dt}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------ Ulysses ---

def ulysses_plan(L, world, rank):
    """Sequence shard of one rank: the token count padded to a multiple of
    the rank count (Wan2.2 source reading, ch. 8 "Ulysses"), Ls tokens per
    rank, rank r holding tokens r * Ls .. (r + 1) * Ls - 1."""
    from video_diffusion_transformer_self_b200 import ulysses
    Lpad = ulysses.padded_len(L, world)
    Ls = Lpad // world
    return {"Lpad": Lpad, "Ls": Ls, "first": rank * Ls,
            "end": (rank + 1) * Ls}


def ulysses_value(B, H, L, steps, max_ms):
    """Whole-job TFLOP/s of the sharded problem: the FLOPs of ONE full
    self-attention (4 * B * heads * L^2 * 128) per step, over the slowest
    rank's time -- strong scaling, the ranks split one problem."""
    return 4.0 * B * H * L * L * 128 * steps / (max_ms / 1e3) / 1e12


def ulysses_steps(q, k, v, g, table, rope, steps, group=None, mark=None):
    """`steps` Ulysses self-attentions of this rank's [B, Ls, H, 128]
    shards; mark(tag) (if given) is called with "start", "exchanged",
    "attended" and "end" around the phases.  Returns the last output."""
    from video_diffusion_transformer_self_b200 import ulysses
    o = None
    for _ in range(steps):
        if mark:
            mark("start")
        o = ulysses.ulysses_self_attn(q, k, v, g, table, group=group,
                                      rope=rope, marks=mark)
        if mark:
            mark("end")
    return o


def run_ulysses(args, w, rank, world, local_rank):
    """One 720p-81f (or --workload) self-attention split over the ranks by
    Ulysses: each rank holds a sequence shard of Q, K, V (all heads), three
    all-to-alls give it the whole sequence of heads / P heads, it rotates
    them (--rope pre) or attends with the rotation fused, and one all-to-all
    returns its output shard.  The exchanges (pack, NCCL all-to-all,
    unpack) and the attention are timed separately with CUDA events."""
    import torch

    from video_diffusion_transformer_self_b200 import wan

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    stream = torch.cuda.current_stream()
    _, g = wan.token_grid(w.frames, w.height, w.width)
    L, B, H = g.F * g.H * g.W, w.batch, w.heads
    if H % world:
        raise SystemExit("heads (%d) do not divide by %d ranks" % (H, world))
    plan = ulysses_plan(L, world, rank)
    gen = torch.Generator(device=dev)
    gen.manual_seed(7070 + rank)
    shape = (B, plan["Ls"], H, 128)
    q, k, v = (torch.randn(shape, device=dev, generator=gen)
               .to(torch.bfloat16) for _ in range(3))
    table = wan.rope3d_table(g)
    dist = None
    if world > 1:
        import torch.distributed as dist_mod
        dist = dist_mod

    def barrier():
        if dist is not None:
            dist.barrier(device_ids=[local_rank])

    events = {}

    def mark(tag):
        e = torch.cuda.Event(enable_timing=True)
        e.record(stream)
        events.setdefault(tag, []).append(e)

    ulysses_steps(q, k, v, g, table, args.rope, args.warmup)
    torch.cuda.synchronize()
    clocks = ClockSampler(local_rank) if rank == 0 else None
    barrier()
    torch.cuda.synchronize()
    ulysses_steps(q, k, v, g, table, args.rope, args.steps, mark=mark)
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop() if clocks else None
    if wan.device_status() != 0:
        raise RuntimeError("device timeout during the timed steps")
    st, ex, at, en = (events[t] for t in ("start", "exchanged", "attended",
                                           "end"))
    total = st[0].elapsed_time(en[-1])
    exch = sum(a.elapsed_time(b) for a, b in zip(st, ex)) + \
        sum(a.elapsed_time(b) for a, b in zip(at, en))
    attn = sum(a.elapsed_time(b) for a, b in zip(ex, at))
    total, exch, attn = max_over_ranks([total, exch, attn], dist, dev)

    # end to end: every step uploads this rank's shards from pinned host
    # memory and reads its output shard back
    e2e = None
    if not args.no_e2e:
        hq, hk, hv = (t.cpu().pin_memory() for t in (q, k, v))
        ho = torch.empty(shape, dtype=torch.bfloat16).pin_memory()
        dq, dk, dv = (torch.empty_like(t) for t in (q, k, v))

        def e2e_steps(n):
            for _ in range(n):
                for d_, h_ in ((dq, hq), (dk, hk), (dv, hv)):
                    d_.copy_(h_, non_blocking=True)
                o = ulysses_steps(dq, dk, dv, g, table, args.rope, 1)
                ho.copy_(o, non_blocking=True)

        e2e_steps(1)
        torch.cuda.synchronize()
        barrier()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        e2e_steps(args.steps)
        b.record(stream)
        torch.cuda.synchronize()
        barrier()
        e2e_ms = max_over_ranks([a.elapsed_time(b)], dist, dev)[0]
        nb = 3 * q.numel() * 2
        e2e = {"value": ulysses_value(B, H, L, args.steps, e2e_ms),
               "unit": "TFLOP/s", "h2d_bytes_per_step": nb,
               "d2h_bytes_per_step": q.numel() * 2,
               "ms_per_step": e2e_ms / args.steps,
               "pipelined": "no (copies, exchanges and kernels in order)"}
    if rank != 0:
        return
    pk, pk_kind = peaks()
    peak = float(pk.get("bf16_tflops_sustained", 1400.0))
    value = ulysses_value(B, H, L, args.steps, total)
    fl_rank = 4.0 * B * (H // world) * L * L * 128
    # library launches per step: the transpose kernel packs q, k, v (and
    # unpacks them when B > 1) and unpacks the output (packing it too when
    # B > 1); then the RoPE pass (--rope pre) and the attention kernel
    moves = (3 + 1 + (4 if B > 1 else 0)) if world > 1 else 0
    per_step = moves + 1 + (1 if args.rope == "pre" else 0)
    line = {
        "metric": "self-attn TFLOP/s",
        "value": value,
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": total / args.steps,
        "higher_is_better": True,
        "scaling": "strong",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {
            "workload": w.name, "batch": B, "heads": H, "seq_len": L,
            "grid": [g.F, g.H, g.W], "rope": args.rope,
            "parallelism": "ulysses%d" % world, "tokens_per_rank":
            plan["Ls"], "padded_tokens": plan["Lpad"],
            "l2": "inputs larger than L2 at 720p-81f",
        },
        "ulysses": {
            "exchange_ms_per_step": exch / args.steps,
            "attention_ms_per_step": attn / args.steps,
            "exchange_bytes_per_rank_per_step":
                4 * B * plan["Ls"] * H * 256 * (world - 1) / world,
            "attention_tflops_per_rank": fl_rank / (attn / args.steps / 1e3)
                / 1e12,
        },
        "roofline": {
            "kernel": "attn_fwd_kernel self-attention on heads / P",
            "bound": "tensor",
            "achieved": fl_rank / (attn / args.steps / 1e3) / 1e12,
            "peak": peak, "unit": "TFLOP/s",
            "frac": fl_rank / (attn / args.steps / 1e3) / 1e12 / peak,
            "traffic": None, "peak_kind": pk_kind + " sustained bf16",
        },
        "gpu_launches": per_step * args.steps,
        "e2e": e2e,
        "clocks": clk,
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    from video_diffusion_transformer_self_b200.workloads import by_name
    w = by_name(args.workload)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, w, rank, world)
        return
    from video_diffusion_transformer_self_b200 import build
    if rank == 0 or world == 1:
        build.build()
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        if args.parallel == "ulysses":
            # keep NCCL's communicator lines (transport, NVLS use) in the log
            os.environ.setdefault("NCCL_DEBUG", "INFO")
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl",
                                timeout=datetime.timedelta(seconds=120))
        dist.barrier(device_ids=[local_rank])
    try:
        if args.parallel == "ulysses":
            run_ulysses(args, w, rank, world, local_rank)
        else:
            run_wan(args, w, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
