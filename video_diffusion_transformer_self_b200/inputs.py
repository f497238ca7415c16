"""Seeded synthetic inputs shared by the oracle tests, the GPU tests and the
benchmark.

This module holds no arithmetic of the method: it only draws seeded random
tensors on the CPU (``torch.Generator('cpu')``), so that every consumer sees
bit-identical inputs.  bf16 tensors are drawn as fp32 N(0, 1) and rounded to
bf16 once; widening them back to float64 is exact.

Seed convention: ``1000 + 100 * workload_index + role``.
"""

import torch

ROLE = {
    "q": 0, "k": 1, "v": 2, "k_ctx": 3, "v_ctx": 4, "lens": 5,
    "x": 6, "v_cond": 7, "v_uncond": 8, "x0": 9, "rows": 10,
    "x_corr": 11, "m_prev1": 12, "m_prev2": 13,
}


def seed_for(index, role):
    """Seed of one input tensor of workload ``index``."""
    return 1000 + 100 * int(index) + ROLE[role]


def _gen(seed):
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def randn_f32(shape, seed, scale=1.0):
    """fp32 N(0, scale^2) tensor on the CPU."""
    t = torch.randn(tuple(shape), generator=_gen(seed), dtype=torch.float32)
    if scale != 1.0:
        t.mul_(scale)
    return t


def randn_bf16(shape, seed, scale=1.0):
    """bf16 tensor: fp32 N(0, scale^2) rounded once to bf16."""
    return randn_f32(shape, seed, scale).to(torch.bfloat16)


def uniform_int(n, lo, hi, seed):
    """int32 tensor of n integers uniform in [lo, hi] (inclusive)."""
    return torch.randint(lo, hi + 1, (n,), generator=_gen(seed),
                         dtype=torch.int64).to(torch.int32)


def sample_rows(n_total, n_rows, seed):
    """Sorted distinct row indices (int64) for sampled comparisons.

    Always includes the first and last row so that the ragged tail tile is
    covered.
    """
    if n_rows >= n_total:
        return torch.arange(n_total, dtype=torch.int64)
    perm = torch.randperm(n_total, generator=_gen(seed))[:n_rows]
    rows = torch.unique(torch.cat([perm, torch.tensor([0, n_total - 1])]))
    return rows.sort().values


def poison_tail(t, lens, value=float("nan")):
    """Overwrite rows j >= lens[b] of a [B, Lk, ...] tensor with ``value``.

    Used to show that padded text keys/values never reach the output.
    """
    t = t.clone()
    for b in range(t.shape[0]):
        t[b, int(lens[b]):] = value
    return t
