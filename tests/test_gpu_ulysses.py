"""GPU checks of the Ulysses path: the library's block transpose against
numpy (bit-exact), and P ranks emulated on one GPU -- every rank's pack,
head attention and unpack run the real kernels, only the all-to-all is a
local permutation of the send buffers.  The gathered result is compared
with the fp64 oracle on the whole, unsharded problem (at the attention
tolerance), and with wan.self_attn on the whole sequence: attention heads
are independent, so that must be bit-identical."""

import numpy as np
import pytest
import torch

from gpu_common import assert_attn_close, cuda, f64, scale_for
from oracle import attention as oattn
from oracle import rope as orope
from video_diffusion_transformer_self_b200 import build, inputs, ulysses, wan

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    wan.lib()


@pytest.mark.parametrize("a,b,row", [(1, 1, 16), (3, 5, 16), (7, 2, 48),
                                     (64, 8, 1280), (2, 3, 4096),
                                     (1000, 4, 256), (5, 1, 32), (1, 6, 64)])
def test_transpose_blocks_bit_exact(a, b, row):
    g = torch.Generator().manual_seed(a * 1000 + b * 10 + row)
    src = torch.randint(0, 256, (a * b * row,), dtype=torch.uint8,
                        generator=g)
    out = torch.full((a * b * row,), 7, dtype=torch.uint8, device="cuda")
    wan.transpose_blocks(cuda(src), out, a, b, row)
    torch.cuda.synchronize()
    want = src.numpy().reshape(a, b, row).transpose(1, 0, 2).reshape(-1)
    assert np.array_equal(out.cpu().numpy(), want)


def _exchange(sends):
    """all-to-all: rank dst receives chunk dst of every source, in source
    order."""
    P = len(sends)
    return [torch.stack([sends[src][dst] for src in range(P)])
            for dst in range(P)]


@pytest.mark.parametrize("P,B,grid,H,rope", [
    (2, 1, (2, 6, 10), 40, "fused"),
    (4, 2, (2, 6, 10), 40, "fused"),
    (5, 1, (2, 6, 10), 40, None),
    (8, 1, (3, 5, 7), 40, "fused"),  # 105 tokens padded to 112
    (8, 1, (21, 6, 8), 8, "fused"),  # 1,008 tokens: several key blocks
    (4, 1, (21, 6, 8), 8, "pre"),    # rotation after the exchange
    (8, 1, (3, 5, 7), 40, "pre"),    # ... with padding
])
def test_emulated_ranks_equal_unsharded(P, B, grid, H, rope):
    g = wan.grid(*grid)
    L = grid[0] * grid[1] * grid[2]
    Lpad = ulysses.padded_len(L, P)
    Ls = Lpad // P
    seed = P * 10 + B
    full = [inputs.randn_bf16((B, Lpad, H, 128), inputs.seed_for(seed, r))
            for r in ("q", "k", "v")]
    table = wan.rope3d_table(g) if rope else None
    want = torch.empty((B, L, H, 128), dtype=torch.bfloat16, device="cuda")
    qw, kw, vw = [cuda(t[:, :L]) for t in full]
    if rope == "pre":
        wan.rope3d_qk(qw, kw, g, table)
        wan.self_attn(qw, kw, vw, want, g)
    else:
        wan.self_attn(qw, kw, vw, want, g, table=table)
    # rank r holds tokens r * Ls .. (r + 1) * Ls - 1 of every tensor
    shards = [[cuda(t[:, r * Ls:(r + 1) * Ls]) for t in full]
              for r in range(P)]
    heads = []
    for which in range(3):
        sends = [ulysses.pack_seq_to_head(shards[r][which], P)
                 for r in range(P)]
        heads.append([ulysses.unpack_seq_to_head(recv)
                      for recv in _exchange(sends)])
    outs_h = [ulysses.head_attention(heads[0][r], heads[1][r], heads[2][r],
                                     g, table, rope=rope or "fused")
              for r in range(P)]
    sends = [ulysses.pack_head_to_seq(oh, P) for oh in outs_h]
    outs = [ulysses.unpack_head_to_seq(recv) for recv in _exchange(sends)]
    torch.cuda.synchronize()
    assert wan.device_status() == 0
    got = torch.cat(outs, dim=1)[:, :L]
    assert got.shape == want.shape
    # the fp64 oracle on the whole, unsharded problem
    qd, kd, vd = (f64(t[:, :L]) for t in full)
    if rope:
        qd, kd = orope.rope3d(qd, grid), orope.rope3d(kd, grid)
    assert_attn_close(f64(got), oattn.attention(qd, kd, vd, scale_for()),
                      "Ulysses P=%d B=%d %s" % (P, B, rope))
    # and bit-identical to the unsharded kernel: heads are independent
    assert torch.equal(got, want)
