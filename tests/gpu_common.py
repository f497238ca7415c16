"""Shared helpers of the GPU parity tests (comparison metrics, device
copies).  The expected values always come from ``oracle/``; the inputs from
the seeded generators in ``video_diffusion_transformer_self_b200.inputs``."""

import math

import numpy as np
import torch

# Tolerances stated for the hot path: bf16 attention and the fp32 step.
ATTN_MAX_ABS = 2e-2
ATTN_REL_FRO = 5e-3
STEP_REL = 1e-6


def f64(t):
    """Exact widening of a CPU/GPU tensor to a float64 numpy array."""
    return t.detach().float().cpu().numpy().astype(np.float64)


def rel_fro(got, want):
    return float(np.linalg.norm(got - want) / np.linalg.norm(want))


def max_abs(got, want):
    return float(np.max(np.abs(got - want)))


def assert_attn_close(got, want, what=""):
    ma, rf = max_abs(got, want), rel_fro(got, want)
    assert np.all(np.isfinite(got)), what + ": non-finite output"
    assert ma <= ATTN_MAX_ABS and rf <= ATTN_REL_FRO, \
        "%s: max_abs %.3g (<= %.3g), rel_fro %.3g (<= %.3g)" % (
            what, ma, ATTN_MAX_ABS, rf, ATTN_REL_FRO)
    return ma, rf


def cuda(t):
    return t.to("cuda").contiguous()


def scale_for(head_dim=128):
    return 1.0 / math.sqrt(head_dim)


def guarded_empty_like(t, guard=4096, fill=float("nan")):
    """Output tensor view inside a buffer with NaN guard bands either side.

    Returns (view, buffer, guard); ``check_guards`` verifies that nothing was
    written outside the view.
    """
    n = t.numel()
    buf = torch.full((n + 2 * guard,), fill, dtype=t.dtype, device="cuda")
    view = buf[guard:guard + n].view(t.shape)
    return view, buf, guard


def check_guards(buf, guard):
    head = buf[:guard].float()
    tail = buf[-guard:].float()
    assert torch.isnan(head).all() and torch.isnan(tail).all(), \
        "write outside the output tensor"


def oracle_threads():
    """Worker threads for oracle evaluations over independent heads."""
    import os
    try:
        n = len(os.sched_getaffinity(0))
    except AttributeError:
        n = os.cpu_count() or 1
    return max(1, min(int(os.environ.get("WAN_ORACLE_THREADS", n)), 32))


def map_threads(fn, items):
    """list(map(fn, items)) on a thread pool.  numpy's BLAS calls and
    float64 ufunc loops release the GIL, so independent heads run in
    parallel; BLAS is held to one thread per call while the pool runs (no
    process pool: nothing is forked after the CUDA context exists)."""
    from concurrent.futures import ThreadPoolExecutor

    from threadpoolctl import threadpool_limits
    with threadpool_limits(limits=1, user_api="blas"):
        with ThreadPoolExecutor(oracle_threads()) as ex:
            return list(ex.map(fn, items))


def head_metrics(label, got, want):
    """(label, max-abs error, relative Frobenius error, all finite) of one
    (batch, head) comparison."""
    return (label, max_abs(got, want), rel_fro(got, want),
            bool(np.all(np.isfinite(got))))


def assert_heads_close(results, what):
    """results: list of head_metrics(...) per (batch, head).  Every pair
    must meet the attention tolerance; the assertion text lists the
    max-abs and relative-Frobenius errors of every pair and the worst."""
    worst_ma, worst_rf, lines, bad = 0.0, 0.0, [], []
    for label, ma, rf, finite in results:
        worst_ma, worst_rf = max(worst_ma, ma), max(worst_rf, rf)
        ok = finite and ma <= ATTN_MAX_ABS and rf <= ATTN_REL_FRO
        lines.append("%s max_abs %.3g rel_fro %.3g%s"
                     % (label, ma, rf, "" if ok else "  <-- FAIL"))
        if not ok:
            bad.append(label)
    assert not bad, "%s: %d of %d (b, h) over tolerance (max_abs <= %.3g, " \
        "rel_fro <= %.3g); worst max_abs %.3g rel_fro %.3g\n%s" % (
            what, len(bad), len(results), ATTN_MAX_ABS, ATTN_REL_FRO,
            worst_ma, worst_rf, "\n".join(lines))
    return worst_ma, worst_rf
