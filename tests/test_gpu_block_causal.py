"""GPU parity of wan_block_causal_attn (chunk-wise causal attention with a
KV cache) against the fp64 oracle."""

import numpy as np
import pytest
import torch

from gpu_common import (assert_attn_close, assert_heads_close, check_guards,
                        cuda, f64, guarded_empty_like, head_metrics,
                        map_threads, scale_for)
from oracle import attention as oattn
from video_diffusion_transformer_self_b200 import build, inputs, wan

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    wan.lib()


def _run(q, k, v, chunk, q_offset=0, pair=False):
    qg, kg, vg = cuda(q), cuda(k), cuda(v)
    o, buf, guard = guarded_empty_like(qg)
    wan.block_causal_attn(qg, kg, vg, o, chunk, q_offset, pair=pair)
    torch.cuda.synchronize()
    assert wan.device_status() == 0
    check_guards(buf, guard)
    return f64(o)


def _qkv(B, Lq, Lk, H, seed):
    q = inputs.randn_bf16((B, Lq, H, 128), seed)
    k = inputs.randn_bf16((B, Lk, H, 128), seed + 1)
    v = inputs.randn_bf16((B, Lk, H, 128), seed + 2)
    return q, k, v


@pytest.mark.parametrize("pair", [False, True], ids=["tiles", "pair"])
@pytest.mark.parametrize("B,L,H,chunk", [
    (1, 300, 2, 50),     # chunks inside tiles, several per CTA
    (2, 700, 1, 128),    # chunk = one key block
    (1, 520, 2, 200),    # chunk boundaries mid-block
    (1, 257, 1, 1),      # token-causal
    (1, 333, 2, 333),    # one chunk = full attention
    (1, 1000, 1, 2000),  # chunk longer than the sequence
])
def test_full_sequence(B, L, H, chunk, pair):
    q, k, v = _qkv(B, L, L, H, 500 + L)
    got = _run(q, k, v, chunk, pair=pair)
    want = oattn.block_causal_attention(f64(q), f64(k), f64(v), scale_for(),
                                        chunk)
    assert_attn_close(got, want, "block-causal L=%d chunk=%d" % (L, chunk))


@pytest.mark.parametrize("pair", [False, True], ids=["tiles", "pair"])
@pytest.mark.parametrize("chunk,n_chunks", [(120, 5), (1560, 3)])
def test_kv_cache_chunk_step(chunk, n_chunks, pair):
    # the last chunk's queries against the cached prefix + itself
    L = chunk * n_chunks
    q, k, v = _qkv(1, L, L, 2, 900 + chunk)
    off = L - chunk
    got = _run(q[:, off:].contiguous(), k, v, chunk, q_offset=off, pair=pair)
    want = oattn.block_causal_attention(f64(q[:, off:]), f64(k), f64(v),
                                        scale_for(), chunk, q_offset=off)
    assert_attn_close(got, want, "kv-cache chunk %d" % chunk)


@pytest.mark.parametrize("Lq,Lk,chunk,expect_pair", [
    (256, 4096, 256, True),    # KV-cache step: equal items, the two-tile
                               # kernel would cut them into key ranges
    (600, 600, 120, False),    # full sequence: unequal items
])
def test_default_kernel(Lq, Lk, chunk, expect_pair):
    # pair=None (the default) runs the kernel block_causal_default_pair
    # names: bit-identical to asking for it
    off = Lk - Lq
    assert wan.block_causal_default_pair(1, Lq, Lk, 2, chunk, off) \
        == expect_pair
    q, k, v = _qkv(1, Lq, Lk, 2, 4242 + Lk)
    qg, kg, vg = cuda(q), cuda(k), cuda(v)
    outs = {}
    for name, kw in (("default", {}), ("named", {"pair": expect_pair}),
                     ("split2", {"split": 2}),
                     ("named2", {"pair": expect_pair, "split": 2})):
        o = torch.empty_like(qg)
        wan.block_causal_attn(qg, kg, vg, o, chunk, off, **kw)
        outs[name] = o
    torch.cuda.synchronize()
    assert wan.device_status() == 0
    assert torch.equal(outs["default"], outs["named"])
    assert torch.equal(outs["split2"], outs["named2"])


@pytest.mark.parametrize("L,chunk,q_offset,Lq,n_split", [
    (600, 120, 480, 120, 2),     # KV-cache step, equal items
    (600, 120, 480, 120, 3),
    (1000, 100, 700, 300, 4),    # KV-cache step over 3 chunks, 2 tiles
    (700, 128, 0, 700, 2),       # full sequence: early rows see no key of
                                 # the second range (row max stays -inf)
    (520, 200, 0, 520, 2),       # chunk boundaries mid-block
])
@pytest.mark.parametrize("pair", [False, True], ids=["tiles", "pair"])
def test_split_key_ranges(L, chunk, q_offset, Lq, n_split, pair):
    q, k, v = _qkv(2, L, L, 2, 1300 + L + n_split)
    ql = q[:, q_offset:q_offset + Lq].contiguous()
    qg, kg, vg = cuda(ql), cuda(k), cuda(v)
    o, buf, guard = guarded_empty_like(qg)
    ws = torch.full((wan.block_causal_workspace_bytes(2, Lq, 2, n_split),),
                    255, dtype=torch.uint8, device="cuda")  # NaN-patterned
    wan.block_causal_attn(qg, kg, vg, o, chunk, q_offset, split=n_split,
                          workspace=ws, pair=pair)
    torch.cuda.synchronize()
    assert wan.device_status() == 0
    check_guards(buf, guard)
    want = oattn.block_causal_attention(f64(ql), f64(k), f64(v), scale_for(),
                                        chunk, q_offset)
    got = f64(o)
    assert_attn_close(got, want, "split %d L=%d" % (n_split, L))
    # the same as one key range, up to fp32 summation order
    one = _run(ql, k, v, chunk, q_offset)
    assert np.max(np.abs(got - one)) <= 1e-2


@pytest.mark.parametrize("pair", [False, True], ids=["tiles", "pair"])
def test_first_chunk_ignores_later_keys(pair):
    chunk, L = 96, 400
    q, k, v = _qkv(1, L, L, 1, 77)
    k2 = (k.float() + 5.0).to(torch.bfloat16)
    v2 = (v.float() - 3.0).to(torch.bfloat16)
    k2[:, :chunk] = k[:, :chunk]
    v2[:, :chunk] = v[:, :chunk]
    a = _run(q[:, :chunk].contiguous(), k, v, chunk, pair=pair)
    b = _run(q[:, :chunk].contiguous(), k2, v2, chunk, pair=pair)
    # keys past the first chunk get weight exactly 0 (they may share a
    # loaded key block with visible keys): changing them changes no bit
    assert np.array_equal(a, b)


@pytest.mark.parametrize("pair", [False, True], ids=["tiles", "pair"])
def test_480p_17f_frame_chunks(pair):
    # 7,800 tokens, chunk = one latent frame (1,560 tokens), 12 heads
    L, H, chunk = 7800, 12, 1560
    q, k, v = _qkv(1, L, L, H, inputs.seed_for(1, "q"))
    got = _run(q, k, v, chunk, pair=pair)
    want = oattn.block_causal_attention(f64(q), f64(k), f64(v), scale_for(),
                                        chunk)
    assert_attn_close(got, want, "block-causal 7800")


# ---- the launch configuration bench.py times: 480p-165f, 42 x 30 x 52 =
# 65,520 tokens, 40 heads, chunks of 3 latent frames (4,680 tokens).  The
# oracle evaluates 4,096 seeded sampled rows of every head (heads are
# independent and run on a thread pool), always including rows on both
# sides of chunk boundaries.
FULL_L, FULL_H, FULL_CHUNK = 65520, 40, 4680
N_ROWS = 4096


def _full_qkv():
    return _qkv(1, FULL_L, FULL_L, FULL_H, 900)


def _rows(n_total, seed, extra=()):
    rows = inputs.sample_rows(n_total, N_ROWS - len(extra), seed).numpy()
    return np.unique(np.concatenate([rows, np.asarray(extra, np.int64)]))


def _per_head(got, q, k, v, rows, q_offset, what):
    def one(h):
        want = oattn.block_causal_attention(
            f64(q[:, :, h:h + 1]), f64(k[:, :, h:h + 1]),
            f64(v[:, :, h:h + 1]), scale_for(128), FULL_CHUNK, q_offset,
            rows, row_block=128)
        return head_metrics("%s h%d (%d rows)" % (what, h, len(rows)),
                            got[:, rows, h:h + 1], want)
    assert_heads_close(map_threads(one, range(FULL_H)), what)


@pytest.mark.parametrize("pair", [False, True], ids=["tiles", "pair"])
def test_full_sequence_480p_165f_sampled(pair):
    q, k, v = _full_qkv()
    got = _run(q, k, v, FULL_CHUNK, pair=pair)
    # rows on both sides of chunk boundaries and in the first chunk
    rows = _rows(FULL_L, 91, [1, 4679, 4680, 32759, 32760, 60839, 60840])
    _per_head(got, q, k, v, rows, 0, "480p-165f full")


@pytest.mark.parametrize("pair", [False, True], ids=["tiles", "pair"])
def test_kv_cache_last_chunk_480p_165f_sampled(pair):
    q, k, v = _full_qkv()
    q0 = FULL_L - FULL_CHUNK
    ql = q[:, q0:].contiguous()
    got = _run(ql, k, v, FULL_CHUNK, q0, pair=pair)
    rows = _rows(FULL_CHUNK, 92, [1, FULL_CHUNK - 2])
    _per_head(got, ql, k, v, rows, q0, "480p-165f KV step")


@pytest.mark.parametrize("pair", [False, True], ids=["tiles", "pair"])
def test_kv_cache_last_chunk_480p_165f_split_sampled(pair):
    # two-tile kernel: the key ranges its policy picks for this device (3 on
    # 148 SMs, as 760 equal items would fill 5.1 waves); CTA-pair kernel:
    # 2 ranges (its policy keeps one here, as splitting measured slower);
    # combining pass after
    q, k, v = _full_qkv()
    q0 = FULL_L - FULL_CHUNK
    ql = q[:, q0:].contiguous()
    n = wan.block_causal_splits(1, FULL_CHUNK, FULL_L, FULL_H, FULL_CHUNK, q0,
                                pair=pair)
    if pair:
        n = 2
    assert n > 1
    qg, kg, vg = cuda(ql), cuda(k), cuda(v)
    o = torch.empty_like(qg)
    wan.block_causal_attn(qg, kg, vg, o, FULL_CHUNK, q0, split=n, pair=pair)
    torch.cuda.synchronize()
    assert wan.device_status() == 0
    got = f64(o)
    rows = _rows(FULL_CHUNK, 92, [1, FULL_CHUNK - 2])
    _per_head(got, ql, k, v, rows, q0, "480p-165f KV step")
