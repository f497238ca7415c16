"""GPU parity of wan_self_attn / wan_cross_attn against the fp64 oracle on
configurations the oracle finishes in seconds (several tiles, ragged tails,
single-token and single-key edge cases, structured inputs)."""

import numpy as np
import pytest
import torch

from gpu_common import (assert_attn_close, check_guards, cuda, f64,
                        guarded_empty_like, scale_for)
from oracle import attention as oattn
from oracle import rope as orope
from video_diffusion_transformer_self_b200 import build, inputs, wan

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    wan.lib()


def _qkv(B, L, H, seed, q_scale=1.0):
    q = inputs.randn_bf16((B, L, H, 128), seed, q_scale)
    k = inputs.randn_bf16((B, L, H, 128), seed + 1)
    v = inputs.randn_bf16((B, L, H, 128), seed + 2)
    return q, k, v


def _run_self(q, k, v, grid, mode):
    """mode: 'fused' (table in the kernel), 'pre' (wan_rope3d_qk first),
    'rope_q' (k by the pass, q in the kernel), 'none' (no RoPE)."""
    g = wan.grid(*grid)
    qg, kg, vg = cuda(q), cuda(k), cuda(v)
    o, buf, guard = guarded_empty_like(qg)
    table = wan.rope3d_table(g) if mode != "none" else None
    if mode == "pre":
        wan.rope3d_qk(qg, kg, g, table)
        wan.self_attn(qg, kg, vg, o, g)
    elif mode == "rope_q":
        # k by the pass, q in the kernel's tile stage (q stays unrotated)
        wan.rope3d_qk(None, kg, g, table)
        wan.self_attn_rope_q(qg, kg, vg, o, g, table)
        torch.cuda.synchronize()
        assert torch.equal(qg.cpu(), q)
    else:
        wan.self_attn(qg, kg, vg, o, g, table=table if mode == "fused"
                      else None)
    torch.cuda.synchronize()
    assert wan.device_status() == 0
    check_guards(buf, guard)
    return f64(o)


def _oracle_self(q, k, v, grid, rope=True):
    qd, kd, vd = f64(q), f64(k), f64(v)
    if rope:
        qd, kd = orope.rope3d(qd, grid), orope.rope3d(kd, grid)
    return oattn.attention(qd, kd, vd, scale_for())


SELF_CASES = [
    ((2, 4, 4), 1, 2),      # tiny: 32 tokens, less than one tile
    ((3, 7, 13), 2, 3),     # 273 tokens: 3 tiles, ragged tail of 17
    ((2, 8, 16), 1, 2),     # exactly 2 tiles
    ((1, 1, 1), 1, 2),      # single token
    ((1, 3, 43), 1, 1),     # 129 tokens: one full tile + 1
    ((1, 1, 127), 1, 2),    # 127 tokens: one tile short of a row
    ((2, 12, 16), 1, 1),    # 384 tokens: 3 tiles, second CTA half empty
    ((1, 5, 77), 2, 1),     # 385 tokens: 4 tiles, last holds 1 row
]


@pytest.mark.parametrize("grid,B,H", SELF_CASES)
@pytest.mark.parametrize("mode", ["fused", "pre", "rope_q", "none"])
def test_self_attn_small(grid, B, H, mode):
    L = grid[0] * grid[1] * grid[2]
    q, k, v = _qkv(B, L, H, 100 + L)
    got = _run_self(q, k, v, grid, mode)
    want = _oracle_self(q, k, v, grid, rope=(mode != "none"))
    assert_attn_close(got, want, "self %s %s" % (grid, mode))


@pytest.mark.parametrize("mode", ["fused", "pre", "rope_q"])
def test_self_attn_480p_17f(mode):
    # 17 frames at 480p: 5 x 30 x 52 = 7,800 tokens, 12 heads (full compare)
    grid, B, H = (5, 30, 52), 1, 12
    L = 7800
    q = inputs.randn_bf16((B, L, H, 128), inputs.seed_for(1, "q"))
    k = inputs.randn_bf16((B, L, H, 128), inputs.seed_for(1, "k"))
    v = inputs.randn_bf16((B, L, H, 128), inputs.seed_for(1, "v"))
    got = _run_self(q, k, v, grid, mode)
    want = _oracle_self(q, k, v, grid)
    assert_attn_close(got, want, "self 7800 " + mode)


def test_self_attn_single_token_returns_v():
    q, k, v = _qkv(1, 1, 3, 7)
    got = _run_self(q, k, v, (1, 1, 1), "fused")
    # one key: softmax weight 1, O = V rounded to bf16 (V is bf16 already)
    assert np.array_equal(got, f64(v))


def test_self_attn_identical_keys_mean_v():
    B, L, H = 1, 300, 2
    q, _, v = _qkv(B, L, H, 9)
    k = inputs.randn_bf16((B, 1, H, 128), 10).expand(B, L, H, 128).contiguous()
    got = _run_self(q, k, v, (3, 10, 10), "none")
    want = np.broadcast_to(f64(v).mean(axis=1, keepdims=True), got.shape)
    assert_attn_close(got, want, "identical keys")


@pytest.mark.parametrize("L", [256, 200, 300])
def test_self_attn_constant_negative_scores_exact(L):
    # Every score equal and negative, every V row equal: softmax weights are
    # uniform, O must be that V row bit for bit.  P = 2^(s - max) is then
    # exactly 1 in every lane, so any error in the running row max (it must
    # equal the negative score, not 0) shows up as a bf16 rounding change.
    B, H = 1, 2
    k0 = inputs.randn_bf16((1, 1, H, 128), 31)
    k = k0.expand(B, L, H, 128).contiguous()
    q = (-k0).expand(B, L, H, 128).contiguous()
    v = inputs.randn_bf16((1, 1, H, 128), 32).expand(B, L, H, 128).contiguous()
    got = _run_self(q, k, v, (1, 1, L), "none")
    assert np.array_equal(got, f64(v))


def test_self_attn_peaked_softmax():
    # Q x 8: scores spread ~8, softmax far from flat -- a kernel that returned
    # mean(V) or mixed rows up fails here.  Unrotated path: the rotated q, k
    # of a RoPE path are rounded to bf16 before the MMA, which alone exceeds
    # the tolerance at this score scale.
    grid, B, H = (3, 7, 13), 1, 2
    q, k, v = _qkv(B, 273, H, 11, q_scale=8.0)
    got = _run_self(q, k, v, grid, "none")
    want = _oracle_self(q, k, v, grid, rope=False)
    assert_attn_close(got, want, "peaked")
    flat = np.broadcast_to(f64(v).mean(axis=1, keepdims=True), got.shape)
    assert np.linalg.norm(flat - want) / np.linalg.norm(want) > 0.5


# ------------------------------------------------------------ cross-attn --

def _run_cross(q, kc, vc, lens):
    qg, kg, vg = cuda(q), cuda(kc), cuda(vc)
    o, buf, guard = guarded_empty_like(qg)
    wan.cross_attn(qg, kg, vg, o, lens)
    torch.cuda.synchronize()
    assert wan.device_status() == 0
    check_guards(buf, guard)
    return f64(o)


def _cross_inputs(B, Lq, Lk, H, seed, lens, poison=True):
    q = inputs.randn_bf16((B, Lq, H, 128), seed)
    kc = inputs.randn_bf16((B, Lk, H, 128), seed + 1)
    vc = inputs.randn_bf16((B, Lk, H, 128), seed + 2)
    if poison:
        kc = inputs.poison_tail(kc, lens)
        vc = inputs.poison_tail(vc, lens)
    return q, kc, vc


def _oracle_cross(q, kc, vc, lens):
    return oattn.attention(f64(q), f64(kc), f64(vc), scale_for(),
                           kv_lens=lens)


@pytest.mark.parametrize("B,Lq,Lk,H,lens", [
    (1, 32, 16, 2, [11]),              # tiny case: 16 text tokens, length 11
    (3, 300, 512, 2, [1, 512, 129]),   # single key, full length, ragged
    (2, 129, 200, 1, [128, 200]),      # exactly one block; ragged 2nd block
    (1, 7, 5, 3, [5]),
    (3, 19993, 512, 4, [37, 512, 300]),  # 948 items: each persistent CTA
                                         # reuses its output staging buffer
])
def test_cross_attn_small(B, Lq, Lk, H, lens):
    q, kc, vc = _cross_inputs(B, Lq, Lk, H, 300 + Lq, lens)
    got = _run_cross(q, kc, vc, lens)
    want = _oracle_cross(q, kc, vc, lens)
    assert_attn_close(got, want, "cross %s" % (lens,))


def test_cross_attn_480p_17f():
    B, Lq, Lk, H = 1, 7800, 512, 12
    lens = inputs.uniform_int(B, 32, 512, inputs.seed_for(1, "lens")).tolist()
    q = inputs.randn_bf16((B, Lq, H, 128), inputs.seed_for(1, "q"))
    kc = inputs.poison_tail(
        inputs.randn_bf16((B, Lk, H, 128), inputs.seed_for(1, "k_ctx")), lens)
    vc = inputs.poison_tail(
        inputs.randn_bf16((B, Lk, H, 128), inputs.seed_for(1, "v_ctx")), lens)
    got = _run_cross(q, kc, vc, lens)
    want = _oracle_cross(q, kc, vc, lens)
    assert_attn_close(got, want, "cross 7800")


def test_cross_attn_zero_query_is_mean_of_valid_rows():
    B, Lq, Lk, H = 2, 130, 300, 2
    lens = [37, 300]
    _, kc, vc = _cross_inputs(B, Lq, Lk, H, 55, lens)
    q = torch.zeros((B, Lq, H, 128), dtype=torch.bfloat16)
    got = _run_cross(q, kc, vc, lens)
    for b, n in enumerate(lens):
        want = np.broadcast_to(f64(vc[b, :n]).mean(axis=0), got[b].shape)
        assert_attn_close(got[b], want, "zero query b=%d" % b)


def test_cross_attn_single_valid_key_returns_its_row():
    B, Lq, Lk, H = 1, 140, 64, 2
    q, kc, vc = _cross_inputs(B, Lq, Lk, H, 66, [1])
    got = _run_cross(q, kc, vc, [1])
    assert np.array_equal(got, np.broadcast_to(f64(vc[:, :1]), got.shape))


def test_cross_attn_peaked():
    B, Lq, Lk, H = 1, 200, 512, 2
    lens = [300]
    q = inputs.randn_bf16((B, Lq, H, 128), 77, 8.0)
    kc = inputs.poison_tail(inputs.randn_bf16((B, Lk, H, 128), 78), lens)
    vc = inputs.poison_tail(inputs.randn_bf16((B, Lk, H, 128), 79), lens)
    got = _run_cross(q, kc, vc, lens)
    assert_attn_close(got, _oracle_cross(q, kc, vc, lens), "cross peaked")
