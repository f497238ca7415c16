"""Pins of the oracle's attention: closed forms, brute force, library."""

import math

import numpy as np
import pytest
import torch

from oracle import attention


def _rng(seed):
    return np.random.default_rng(seed)


def _brute(q, k, v, scale, kv_len):
    """Pure-Python triple loop, independent of numpy, for tiny inputs."""
    out = []
    for qi in q:
        s = [scale * sum(a * b for a, b in zip(qi, k[j]))
             for j in range(kv_len)]
        m = max(s)
        p = [math.exp(x - m) for x in s]
        z = sum(p)
        out.append([sum(p[j] * v[j][c] for j in range(kv_len)) / z
                    for c in range(len(v[0]))])
    return np.array(out)


@pytest.mark.parametrize("lq,lk,d,kv_len", [(5, 7, 4, 7), (3, 9, 6, 4),
                                            (1, 1, 8, 1)])
def test_brute_force(lq, lk, d, kv_len):
    r = _rng(lq * 100 + lk)
    q = r.standard_normal((lq, d))
    k = r.standard_normal((lk, d))
    v = r.standard_normal((lk, d))
    want = _brute(q.tolist(), k.tolist(), v.tolist(), 0.7, kv_len)
    got = attention.attend(q, k, v, 0.7, kv_len)
    assert np.max(np.abs(got - want)) < 1e-13


def test_matches_torch_sdpa_fp64():
    # Special case reducing to a library routine: torch's fp64 SDPA.
    r = _rng(7)
    B, L, H, D, LK = 2, 33, 3, 16, 20
    q = r.standard_normal((B, L, H, D))
    k = r.standard_normal((B, LK, H, D))
    v = r.standard_normal((B, LK, H, D))
    lens = [5, 20]
    got = attention.attention(q, k, v, 1 / math.sqrt(D), kv_lens=lens)
    tq = torch.from_numpy(q).permute(0, 2, 1, 3)
    tk = torch.from_numpy(k).permute(0, 2, 1, 3)
    tv = torch.from_numpy(v).permute(0, 2, 1, 3)
    mask = torch.zeros(B, 1, 1, LK, dtype=torch.bool)
    for b, n in enumerate(lens):
        mask[b, ..., :n] = True
    ref = torch.nn.functional.scaled_dot_product_attention(
        tq, tk, tv, attn_mask=mask).permute(0, 2, 1, 3).numpy()
    assert np.max(np.abs(got - ref)) < 1e-12


def test_rows_sum_to_one():
    s = _rng(8).standard_normal((10, 50)) * 5
    p = attention.softmax_rows(s)
    assert np.max(np.abs(p.sum(axis=1) - 1)) < 1e-14
    assert np.all(p > 0)


def test_single_key_returns_its_value_row():
    r = _rng(9)
    q = r.standard_normal((4, 128))
    k = r.standard_normal((1, 128))
    v = r.standard_normal((1, 128))
    o = attention.attend(q, k, v, 1 / math.sqrt(128))
    assert np.array_equal(o, np.repeat(v, 4, axis=0))
    # and with kv_len = 1 out of many keys
    k2 = np.concatenate([k, r.standard_normal((9, 128))])
    v2 = np.concatenate([v, r.standard_normal((9, 128))])
    o2 = attention.attend(q, k2, v2, 1 / math.sqrt(128), kv_len=1)
    assert np.array_equal(o2, np.repeat(v, 4, axis=0))


def test_identical_keys_give_mean_value():
    r = _rng(10)
    q = r.standard_normal((6, 32))
    k = np.repeat(r.standard_normal((1, 32)), 11, axis=0)
    v = r.standard_normal((11, 32))
    o = attention.attend(q, k, v, 0.3)
    assert np.max(np.abs(o - v.mean(axis=0))) < 1e-14


def test_zero_query_gives_mean_of_valid_rows():
    r = _rng(11)
    q = np.zeros((3, 16))
    k = r.standard_normal((12, 16))
    v = r.standard_normal((12, 16))
    o = attention.attend(q, k, v, 0.25, kv_len=5)
    assert np.max(np.abs(o - v[:5].mean(axis=0))) < 1e-14


def test_full_length_equals_unmasked_and_nan_padding_ignored():
    r = _rng(12)
    B, L, H, D, LK = 2, 9, 2, 8, 12
    q = r.standard_normal((B, L, H, D))
    k = r.standard_normal((B, LK, H, D))
    v = r.standard_normal((B, LK, H, D))
    full = attention.attention(q, k, v, 0.35)
    assert np.array_equal(attention.attention(q, k, v, 0.35,
                                              kv_lens=[LK, LK]), full)
    lens = [3, 7]
    masked = attention.attention(q, k, v, 0.35, kv_lens=lens)
    kp, vp = k.copy(), v.copy()
    for b, n in enumerate(lens):
        kp[b, n:] = np.nan
        vp[b, n:] = np.nan
    assert np.array_equal(attention.attention(q, kp, vp, 0.35, kv_lens=lens),
                          masked)


def test_peaked_query_selects_matching_key():
    # Scaling q along one key's direction drives the softmax to one-hot.
    r = _rng(13)
    k = r.standard_normal((20, 64))
    k /= np.linalg.norm(k, axis=1, keepdims=True)
    v = r.standard_normal((20, 64))
    q = 400.0 * k[7:8]
    o = attention.attend(q, k, v, 1.0)
    assert np.max(np.abs(o[0] - v[7])) < 1e-6


def test_sampled_rows_equal_full_rows():
    r = _rng(14)
    q = r.standard_normal((1, 40, 2, 8))
    k = r.standard_normal((1, 40, 2, 8))
    v = r.standard_normal((1, 40, 2, 8))
    rows = np.array([0, 5, 39])
    full = attention.attention(q, k, v, 0.5)
    part = attention.attention(q, k, v, 0.5, rows=rows, row_block=2)
    # the library matmul may sum in another order for another shape
    assert np.max(np.abs(part - full[:, rows])) < 1e-14


def test_planted_transpose_mistake_is_caught(monkeypatch):
    # Passing the wrong operand (k as the values) must fail brute force.
    r = _rng(15)
    q, k, v = (r.standard_normal((5, 5)) for _ in range(3))
    good = _brute(q.tolist(), k.tolist(), v.tolist(), 0.5, 5)
    orig = attention.attend

    def wrong(q, k, v, scale, kv_len=None):
        return orig(q, k, k, scale, kv_len)
    monkeypatch.setattr(attention, "attend", wrong)
    assert np.max(np.abs(attention.attend(q, k, v, 0.5) - good)) > 1e-3


# ------------------------------------------------------------ block-causal --

def test_block_causal_one_chunk_is_full_attention():
    r = _rng(21)
    q, k, v = (r.standard_normal((1, 24, 2, 8)) for _ in range(3))
    full = attention.attention(q, k, v, 0.4)
    bc = attention.block_causal_attention(q, k, v, 0.4, chunk_tokens=24)
    assert np.max(np.abs(bc - full)) < 1e-13
    bc2 = attention.block_causal_attention(q, k, v, 0.4, chunk_tokens=1000)
    assert np.max(np.abs(bc2 - full)) < 1e-13


def test_block_causal_chunk_one_is_token_causal_sdpa():
    # chunk of one token = ordinary causal attention (library routine)
    r = _rng(22)
    q, k, v = (r.standard_normal((2, 17, 3, 8)) for _ in range(3))
    got = attention.block_causal_attention(q, k, v, 1 / math.sqrt(8), 1)
    t = [torch.from_numpy(x).permute(0, 2, 1, 3) for x in (q, k, v)]
    ref = torch.nn.functional.scaled_dot_product_attention(
        *t, is_causal=True).permute(0, 2, 1, 3).numpy()
    assert np.max(np.abs(got - ref)) < 1e-12


def test_block_causal_matches_explicit_mask_sdpa():
    r = _rng(23)
    L, chunk = 20, 6
    q, k, v = (r.standard_normal((1, L, 2, 8)) for _ in range(3))
    got = attention.block_causal_attention(q, k, v, 0.3, chunk)
    mask = torch.zeros(L, L, dtype=torch.bool)
    for a in range(L):
        mask[a, :min(L, (a // chunk + 1) * chunk)] = True
    t = [torch.from_numpy(x).permute(0, 2, 1, 3) for x in (q, k, v)]
    ref = torch.nn.functional.scaled_dot_product_attention(
        *t, attn_mask=mask, scale=0.3).permute(0, 2, 1, 3).numpy()
    assert np.max(np.abs(got - ref)) < 1e-12


def test_block_causal_kv_cache_form_equals_full_rows():
    # queries of the last chunk against cached keys = rows of the full run
    r = _rng(24)
    L, chunk = 30, 7
    q, k, v = (r.standard_normal((1, L, 1, 8)) for _ in range(3))
    full = attention.block_causal_attention(q, k, v, 0.5, chunk)
    off = 21  # queries of positions 21..29 (chunks 3 and 4)
    part = attention.block_causal_attention(q[:, off:], k, v, 0.5, chunk,
                                            q_offset=off)
    assert np.max(np.abs(part - full[:, off:])) < 1e-13
    # the first chunk never sees later keys: changing them changes nothing
    k2, v2 = k.copy(), v.copy()
    k2[:, chunk:] += 5.0
    v2[:, chunk:] -= 3.0
    again = attention.block_causal_attention(q, k2, v2, 0.5, chunk)
    assert np.array_equal(again[:, :chunk], full[:, :chunk])


def test_block_causal_limits_and_rejects():
    lim = attention.block_causal_limits(5, 9, 4, q_offset=4)
    assert list(lim) == [8, 8, 8, 8, 9]
    with pytest.raises(ValueError):
        attention.block_causal_limits(5, 8, 4, q_offset=4)
    with pytest.raises(ValueError):
        attention.block_causal_limits(5, 9, 0)


def test_block_causal_grouped_rows_equal_row_by_row():
    # the grouped evaluation (rows sharing a key limit together, in groups
    # smaller than a chunk) against the plain row-by-row definition, on
    # sampled rows and a KV-cache offset
    rng = np.random.default_rng(17)
    q = rng.standard_normal((2, 90, 3, 8))
    k = rng.standard_normal((2, 130, 3, 8))
    v = rng.standard_normal((2, 130, 3, 8))
    rows = np.array([0, 1, 5, 19, 20, 21, 44, 60, 89])
    got = attention.block_causal_attention(q, k, v, 0.35, 20, q_offset=40,
                                           rows=rows, row_block=2)
    lim = attention.block_causal_limits(90, 130, 20, 40)
    for b in range(2):
        for h in range(3):
            want = attention.attend_limited(q[b, rows, h], k[b, :, h],
                                            v[b, :, h], 0.35, lim[rows])
            np.testing.assert_allclose(got[b, :, h], want, rtol=1e-13,
                                       atol=1e-13)
