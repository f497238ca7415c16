"""Seeded random shapes for every attention entry point, each compared in
full with the fp64 oracle: odd token grids (ragged tiles and key blocks,
single tokens), batch rows and head counts, per-row text lengths with
NaN-poisoned padding, block-causal chunks and KV-cache offsets on both
kernels, and key ranges.  The cases are drawn once, from a fixed seed, when
the module is collected; every draw satisfies the calls' documented
argument rules."""

import numpy as np
import pytest
import torch

from gpu_common import (assert_attn_close, check_guards, cuda, f64,
                        guarded_empty_like, scale_for)
from oracle import attention as oattn
from oracle import rope as orope
from video_diffusion_transformer_self_b200 import build, inputs, wan

pytestmark = pytest.mark.gpu

_RNG = np.random.default_rng(20261203)


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    wan.lib()


def _bf16(shape, seed):
    return inputs.randn_bf16(shape, seed)


# ------------------------------------------------------ self-attention --

SELF_MODES = ("none", "fused", "pre", "rope_q", "pair", "pair_rope_q")


def _self_cases(n):
    cases = []
    for i in range(n):
        F = int(_RNG.integers(1, 4))
        H = int(_RNG.integers(1, 10))
        W = int(_RNG.integers(1, 26))
        B = int(_RNG.integers(1, 3))
        heads = int(_RNG.integers(1, 4))
        mode = SELF_MODES[i % len(SELF_MODES)]
        cases.append(((F, H, W), B, heads, mode, 7000 + 10 * i))
    return cases


@pytest.mark.parametrize(
    "grid,B,heads,mode,seed", _self_cases(36),
    ids=lambda c: "-".join(map(str, c)) if isinstance(c, tuple) else str(c))
def test_self_attention_random(grid, B, heads, mode, seed):
    L = grid[0] * grid[1] * grid[2]
    q = _bf16((B, L, heads, 128), seed)
    k = _bf16((B, L, heads, 128), seed + 1)
    v = _bf16((B, L, heads, 128), seed + 2)
    g = wan.grid(*grid)
    qg, kg, vg = cuda(q), cuda(k), cuda(v)
    o, buf, guard = guarded_empty_like(qg)
    rope = mode not in ("none", "pair")
    table = wan.rope3d_table(g) if rope else None
    if mode == "none":
        wan.self_attn(qg, kg, vg, o, g)
    elif mode == "fused":
        wan.self_attn(qg, kg, vg, o, g, table=table)
    elif mode == "pre":
        wan.rope3d_qk(qg, kg, g, table)
        wan.self_attn(qg, kg, vg, o, g)
    elif mode == "rope_q":
        wan.rope3d_qk(None, kg, g, table)
        wan.self_attn_rope_q(qg, kg, vg, o, g, table)
    elif mode == "pair":
        wan.self_attn_pair(qg, kg, vg, o, g)
    else:  # pair_rope_q
        wan.rope3d_qk(None, kg, g, table)
        wan.self_attn_pair(qg, kg, vg, o, g, table_q=table)
    torch.cuda.synchronize()
    assert wan.device_status() == 0
    check_guards(buf, guard)
    qd, kd, vd = f64(q), f64(k), f64(v)
    if rope:
        qd, kd = orope.rope3d(qd, grid), orope.rope3d(kd, grid)
    want = oattn.attention(qd, kd, vd, scale_for())
    assert_attn_close(f64(o), want, "self %s grid %s B %d heads %d"
                      % (mode, grid, B, heads))


# ----------------------------------------------------- cross-attention --

def _cross_cases(n):
    cases = []
    for i in range(n):
        B = int(_RNG.integers(1, 4))
        Lq = int(_RNG.integers(1, 701))
        Lk = int(_RNG.choice([16, 77, 128, 129, 300, 512]))
        heads = int(_RNG.integers(1, 3))
        lens = tuple(int(x) for x in _RNG.integers(1, Lk + 1, size=B))
        cases.append((B, Lq, Lk, heads, lens, 8000 + 10 * i))
    return cases


@pytest.mark.parametrize("B,Lq,Lk,heads,lens,seed", _cross_cases(24))
def test_cross_attention_random(B, Lq, Lk, heads, lens, seed):
    q = _bf16((B, Lq, heads, 128), seed)
    kc = _bf16((B, Lk, heads, 128), seed + 1)
    vc = _bf16((B, Lk, heads, 128), seed + 2)
    # padding past each text length holds NaN: it must never reach O
    kp, vp = inputs.poison_tail(kc, lens), inputs.poison_tail(vc, lens)
    qg = cuda(q)
    o, buf, guard = guarded_empty_like(qg)
    wan.cross_attn(qg, cuda(kp), cuda(vp), o, list(lens))
    torch.cuda.synchronize()
    assert wan.device_status() == 0
    check_guards(buf, guard)
    want = oattn.attention(f64(q), f64(kc), f64(vc), scale_for(),
                           kv_lens=list(lens))
    assert_attn_close(f64(o), want, "cross B %d Lq %d Lk %d lens %s"
                      % (B, Lq, Lk, lens))


# -------------------------------------------------------- block-causal --

def _first_item_blocks(Lq, Lk, chunk, q_offset):
    # key blocks of the lightest item (the first 256 queries)
    last = min(256, Lq) - 1 + q_offset
    kv = min(Lk, (last // chunk + 1) * chunk)
    return (kv + 127) // 128


def _causal_cases(n):
    cases = []
    for i in range(n):
        Lk = int(_RNG.integers(2, 1201))
        chunk = int(_RNG.integers(1, 401))
        if i % 2 == 0:
            Lq, q_offset = Lk, 0                      # full sequence
        else:
            Lq = int(_RNG.integers(1, Lk + 1))        # KV-cache step
            q_offset = Lk - Lq
        pair = bool(i % 4 in (1, 2))
        n_split = int(_RNG.integers(1, 4))
        if _first_item_blocks(Lq, Lk, chunk, q_offset) < n_split:
            n_split = 1
        B = int(_RNG.integers(1, 3))
        heads = int(_RNG.integers(1, 3))
        cases.append((B, Lq, Lk, heads, chunk, q_offset, pair, n_split,
                      9000 + 10 * i))
    return cases


@pytest.mark.parametrize("B,Lq,Lk,heads,chunk,q_offset,pair,n_split,seed",
                         _causal_cases(40))
def test_block_causal_random(B, Lq, Lk, heads, chunk, q_offset, pair,
                             n_split, seed):
    q = _bf16((B, Lq, heads, 128), seed)
    k = _bf16((B, Lk, heads, 128), seed + 1)
    v = _bf16((B, Lk, heads, 128), seed + 2)
    qg = cuda(q)
    o, buf, guard = guarded_empty_like(qg)
    ws = None
    if n_split > 1:
        ws = torch.full((wan.block_causal_workspace_bytes(B, Lq, heads,
                                                          n_split),),
                        255, dtype=torch.uint8, device="cuda")
    wan.block_causal_attn(qg, cuda(k), cuda(v), o, chunk, q_offset,
                          pair=pair, split=n_split if n_split > 1 else None,
                          workspace=ws)
    torch.cuda.synchronize()
    assert wan.device_status() == 0
    check_guards(buf, guard)
    want = oattn.block_causal_attention(f64(q), f64(k), f64(v), scale_for(),
                                        chunk, q_offset)
    assert_attn_close(f64(o), want, "block-causal %s" % ((
        B, Lq, Lk, heads, chunk, q_offset, pair, n_split),))


# ---------------------------------------------------------------- RoPE --

def _rope_cases(n):
    cases = []
    for i in range(n):
        # token grids up to the RoPE table's side limit on one axis at a
        # time, a few thousand tokens in all
        F = int(_RNG.integers(1, 30))
        H = int(_RNG.integers(1, 40))
        W = int(_RNG.integers(1, max(2, 4000 // (F * H))))
        if i % 4 == 3:
            F, H, W = 1, 1, int(_RNG.integers(900, 1025))  # long width axis
        B = int(_RNG.integers(1, 3))
        heads = int(_RNG.integers(1, 17))
        cases.append(((F, H, W), B, heads, 9500 + 10 * i))
    return cases


@pytest.mark.parametrize(
    "grid,B,heads,seed", _rope_cases(16),
    ids=lambda c: "-".join(map(str, c)) if isinstance(c, tuple) else str(c))
def test_rope_random(grid, B, heads, seed):
    L = grid[0] * grid[1] * grid[2]
    q = _bf16((B, L, heads, 128), seed)
    k = _bf16((B, L, heads, 128), seed + 1)
    g = wan.grid(*grid)
    table = wan.rope3d_table(g)
    qg, kg = cuda(q), cuda(k)
    wan.rope3d_qk(qg, kg, g, table)
    torch.cuda.synchronize()
    assert wan.device_status() == 0
    for got, x in ((qg, q), (kg, k)):
        xd = x.double().numpy()
        want = orope.rope3d(xd, grid)
        # bf16 output: half an ulp is <= 2^-8 of the value; fp32 arithmetic
        # and the fp32 table add ~1e-6 of the pair's norm
        pair = np.repeat(np.sqrt(xd[..., 0::2] ** 2 + xd[..., 1::2] ** 2), 2,
                         axis=-1)
        bound = 2.0 ** -8 * np.abs(want) + 1e-6 * pair + 1e-30
        err = np.abs(got.double().cpu().numpy() - want)
        assert np.all(err <= bound), (grid, float(np.max(err / bound)))
