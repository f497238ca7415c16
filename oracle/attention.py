"""Softmax attention in fp64 (oracle; test infrastructure only).

Self-attention: Wan2.2 source reading, ch. 4, section "Full forward of one
block" -- full 3D joint attention, every token of every frame attends to
every other token with no mask (the intro of ch. 4 chooses full joint
attention over factorised attention); ch. 8 "What is 75600^2" counts its two
matrix products QK^T and AV.

Cross-attention: Wan2.2 source reading, ch. 3 "Where did the prompt go" --
video tokens are the queries, the text context gives keys/values, and each
prompt is trimmed to its true length ``u[:v]`` with
``seq_lens = mask.gt(0).sum(dim=1)``; the forward passes ``context_lens`` on
to ``cross_attn``.  Wan paper explainer, section "Text encoder": the
cross-attention is ``softmax(Q K_text^T / sqrt(d_k)) V_text``.

Definition evaluated here, for each batch row b and head h:

    s_ij = (q_i . k_j) * scale,   j < kv_len
    m_i  = max_j s_ij
    p_ij = exp(s_ij - m_i)
    o_i  = sum_j p_ij v_j / sum_j p_ij

in float64 with no intermediate rounding beyond fp64's own.  Keys at or
beyond kv_len take no part (their contents never enter the arithmetic).
Rows are independent, so evaluating a subset of query rows (``rows=``) or
evaluating rows in groups to bound memory changes no row's definition; the
library matmul may only sum in another order (fp64 rounding level).
"""

import numpy as np


def softmax_rows(s):
    """Row softmax of a float64 score matrix (max-subtracted exp / sum)."""
    m = s.max(axis=1, keepdims=True)
    p = np.exp(s - m)
    return p / p.sum(axis=1, keepdims=True)


def attend(q, k, v, scale, kv_len=None):
    """One (batch, head) slice: q [Lq, d], k/v [Lk, d] -> o [Lq, d] fp64."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    if kv_len is not None:
        if not 1 <= kv_len <= k.shape[0]:
            raise ValueError("kv_len out of range")
        k = k[:kv_len]
        v = v[:kv_len]
    s = (q @ k.T) * scale
    return softmax_rows(s) @ v


def attention(q, k, v, scale, kv_lens=None, rows=None, row_block=512):
    """Batched attention over [B, L, heads, d] tensors.

    q: [B, Lq, heads, d]; k, v: [B, Lk, heads, d]; kv_lens: per-batch valid
    key count (None = all Lk keys); rows: optional 1-D array of query indices
    to evaluate (default all).  Returns [B, len(rows), heads, d] float64.
    """
    q = np.asarray(q)
    k = np.asarray(k)
    v = np.asarray(v)
    b_, lq, nh, d = q.shape
    rows = np.arange(lq) if rows is None else np.asarray(rows)
    out = np.empty((b_, rows.shape[0], nh, d), dtype=np.float64)
    for b in range(b_):
        kv_len = None if kv_lens is None else int(kv_lens[b])
        for h in range(nh):
            kh = k[b, :, h, :].astype(np.float64)
            vh = v[b, :, h, :].astype(np.float64)
            for r0 in range(0, rows.shape[0], row_block):
                sel = rows[r0:r0 + row_block]
                qh = q[b, sel, h, :].astype(np.float64)
                out[b, r0:r0 + row_block, h, :] = attend(qh, kh, vh, scale,
                                                         kv_len)
    return out


# --------------------------------------------------------- block-causal --
#
# Long-video survey, section "Route 3 · Self Forcing": bidirectional full
# attention is replaced by causal attention over chunks of frames so that a
# finished chunk can be decoded and streamed; each new chunk attends to the
# chunks before it through a KV cache (the KV cache can also be capped).
#
# Reading: a query at absolute token position a (frame-major order) belongs
# to chunk floor(a / chunk_tokens) and sees every key j with
#     j < (floor(a / chunk_tokens) + 1) * chunk_tokens,
# i.e. all tokens of its own chunk and of every earlier chunk.  In the KV
# cache form the queries of one chunk sit at absolute positions
# q_offset .. q_offset + Lq - 1 and the keys are the cached prefix followed
# by that chunk.

def block_causal_limits(lq, lk, chunk_tokens, q_offset=0):
    """Per-query key limit (exclusive) of the block-causal mask."""
    if chunk_tokens < 1 or q_offset < 0 or q_offset + lq > lk:
        raise ValueError("bad block-causal geometry")
    a = q_offset + np.arange(lq)
    return np.minimum(lk, (a // chunk_tokens + 1) * chunk_tokens)


def attend_limited(q, k, v, scale, limits):
    """One (batch, head) slice with a per-row key limit, fp64.

    Row i uses keys 0 .. limits[i]-1 only (the definition above, evaluated
    row by row).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    out = np.empty((q.shape[0], v.shape[1]), dtype=np.float64)
    for i, n in enumerate(limits):
        s = (q[i] @ k[:n].T) * scale
        p = np.exp(s - s.max())
        out[i] = (p @ v[:n]) / p.sum()
    return out


def block_causal_attention(q, k, v, scale, chunk_tokens, q_offset=0,
                           rows=None, row_block=512):
    """Block-causal attention over [B, L, heads, d] tensors (fp64).

    Every query of one chunk has the same key limit, so the rows sharing a
    limit n are evaluated together as plain attention over keys 0 .. n-1
    (``attend``), in groups of at most ``row_block`` rows; each row is the
    same definition as ``attend_limited`` gives it.
    """
    q = np.asarray(q)
    b_, lq, nh, d = q.shape
    lk = np.asarray(k).shape[1]
    lim = block_causal_limits(lq, lk, chunk_tokens, q_offset)
    rows = np.arange(lq) if rows is None else np.asarray(rows)
    lim_r = lim[rows]
    out = np.empty((b_, rows.shape[0], nh, d), dtype=np.float64)
    for b in range(b_):
        for h in range(nh):
            kh = np.asarray(k[b, :, h, :], dtype=np.float64)
            vh = np.asarray(v[b, :, h, :], dtype=np.float64)
            for n in np.unique(lim_r):
                idx = np.nonzero(lim_r == n)[0]
                for r0 in range(0, idx.shape[0], row_block):
                    sel = idx[r0:r0 + row_block]
                    out[b, sel, h, :] = attend(q[b, rows[sel], h, :],
                                               kh[:n], vh[:n], scale)
    return out
