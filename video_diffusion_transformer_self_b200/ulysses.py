"""Ulysses sequence-parallel self-attention across the ranks of a process
group.

Wan2.2 source reading, ch. 8 "Ulysses": attention needs every token, so the
sequence cannot simply be cut; instead each rank trades its sequence shard
of all heads for the whole sequence of heads / P heads with one all-to-all
(scatter one dimension, gather another), runs attention on those heads, and
trades the output back -- two exchanges per attention (four all-to-alls:
q, k, v and the output).  The head count must divide by the rank count, and
the token count is padded up to a multiple of it (75,601 tokens -> 75,608 on
8 ranks) so that every rank holds an equal slice.

Reading: padded tokens take no part in the attention (they are past the
token grid the kernel is given) and their outputs are unspecified; padding
is supported with batch 1, the pages' setting.

Every layout move runs in the library's transpose kernel
(``wan.transpose_blocks``), the exchange is the process group's
all-to-all (NCCL between GPUs), and the attention is ``wan.self_attn``.
Each exchange is split into pack / all-to-all / unpack so that the same
code can be driven rank by rank (tests emulate several ranks on one GPU).
"""

import torch
import torch.distributed as dist

from . import wan


def padded_len(L, world):
    """Tokens per rank times ranks: L rounded up to a multiple of world."""
    return -(-int(L) // int(world)) * int(world)


def _swap(inp, out, a, b, row_bytes):
    wan.transpose_blocks(inp, out, a, b, row_bytes)


def _attention(q, k, v, o, g, table, softmax_scale):
    wan.self_attn(q, k, v, o, g, table=table, softmax_scale=softmax_scale)


def _rope(q, k, g, table):
    wan.rope3d_qk(q, k, g, table)


def _world(group):
    return dist.get_world_size(group) if dist.is_initialized() else 1


# ------------------------------------------------------ sequence -> head --

def pack_seq_to_head(x, P):
    """[B, Ls, H, d] -> send buffer [P, B, Ls, H / P, d] (chunk p for rank p)."""
    B, Ls, H, d = x.shape
    if H % P:
        raise ValueError("heads (%d) must divide by the rank count (%d)"
                         % (H, P))
    Hp = H // P
    send = torch.empty((P, B, Ls, Hp, d), dtype=x.dtype, device=x.device)
    _swap(x, send, B * Ls, P, Hp * d * x.element_size())
    return send


def unpack_seq_to_head(recv):
    """recv [P (source rank), B, Ls, Hp, d] -> [B, P * Ls, Hp, d]."""
    P, B, Ls, Hp, d = recv.shape
    if B == 1:
        return recv.view(1, P * Ls, Hp, d)
    out = torch.empty((B, P, Ls, Hp, d), dtype=recv.dtype, device=recv.device)
    _swap(recv, out, P, B, Ls * Hp * d * recv.element_size())
    return out.view(B, P * Ls, Hp, d)


def seq_to_head(x, group=None):
    """Sequence shard [B, Ls, H, d] -> head shard [B, P * Ls, H / P, d]."""
    P = _world(group)
    if P == 1:
        return x
    send = pack_seq_to_head(x, P)
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv, send, group=group)
    return unpack_seq_to_head(recv)


# ------------------------------------------------------ head -> sequence --

def pack_head_to_seq(y, P):
    """[B, P * Ls, Hp, d] -> send buffer [P, B, Ls, Hp, d] (shard p to rank p)."""
    B, L, Hp, d = y.shape
    if L % P:
        raise ValueError("sequence (%d) must divide by the rank count (%d)"
                         % (L, P))
    Ls = L // P
    if B == 1:
        return y.view(P, 1, Ls, Hp, d)
    send = torch.empty((P, B, Ls, Hp, d), dtype=y.dtype, device=y.device)
    _swap(y, send, B, P, Ls * Hp * d * y.element_size())
    return send


def unpack_head_to_seq(recv):
    """recv [P (source rank = head group), B, Ls, Hp, d] -> [B, Ls, P * Hp, d]."""
    P, B, Ls, Hp, d = recv.shape
    out = torch.empty((B, Ls, P, Hp, d), dtype=recv.dtype, device=recv.device)
    _swap(recv, out, P, B * Ls, Hp * d * recv.element_size())
    return out.view(B, Ls, P * Hp, d)


def head_to_seq(y, group=None):
    """Head shard [B, P * Ls, Hp, d] -> sequence shard [B, Ls, P * Hp, d]."""
    P = _world(group)
    if P == 1:
        return y
    send = pack_head_to_seq(y, P)
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv, send, group=group)
    return unpack_head_to_seq(recv)


# ------------------------------------------------------------ attention --

def head_attention(qh, kh, vh, g, table=None, softmax_scale=None,
                   rope="fused"):
    """Attention of head-sharded [B, Lpad, Hp, d] tensors over the grid g's
    L = F * H * W tokens; rows past L (padding) are left unspecified.

    With a table, rope="fused" rotates q and k inside the attention kernel's
    tile stage; rope="pre" first rotates the received q and k in place with
    the stand-alone RoPE pass (each holds the whole sequence of its heads,
    so every token's (f, h, w) is known) and then attends without a table.
    """
    if rope not in ("fused", "pre"):
        raise ValueError("rope must be 'fused' or 'pre'")
    B, Lpad = qh.shape[0], qh.shape[1]
    L = g.F * g.H * g.W
    oh = torch.empty_like(qh)
    if Lpad != L and B != 1:
        raise ValueError("sequence padding needs batch 1")
    q_, k_, v_, o_ = ((qh, kh, vh, oh) if Lpad == L else
                      (qh[:, :L], kh[:, :L], vh[:, :L], oh[:, :L]))
    if table is not None and rope == "pre":
        _rope(q_, k_, g, table)
        table = None
    _attention(q_, k_, v_, o_, g, table, softmax_scale)
    return oh


def ulysses_self_attn(q, k, v, g, table=None, softmax_scale=None,
                      group=None, rope="fused", marks=None):
    """Self-attention over the token grid g from sequence shards.

    q, k, v: [B, Ls, H, 128] bf16 on this rank's GPU, rank r holding tokens
    r * Ls .. (r + 1) * Ls - 1 of the sequence padded to P * Ls =
    padded_len(F * H * W, P).  Returns this rank's [B, Ls, H, 128] output.
    rope: see head_attention.  marks: optional callable, called with
    "exchanged" after the three inbound exchanges and with "attended" after
    the attention (used to time the two phases).
    """
    P = _world(group)
    L = g.F * g.H * g.W
    Ls = q.shape[1]
    if P * Ls != padded_len(L, P):
        raise ValueError("shard length %d does not match %d tokens on %d "
                         "ranks" % (Ls, L, P))
    qh = seq_to_head(q, group)
    kh = seq_to_head(k, group)
    vh = seq_to_head(v, group)
    if marks is not None:
        marks("exchanged")
    oh = head_attention(qh, kh, vh, g, table, softmax_scale, rope)
    if marks is not None:
        marks("attended")
    return head_to_seq(oh, group)
