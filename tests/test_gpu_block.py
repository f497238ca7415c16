"""GPU parity of the block prologue / epilogue kernels (AdaLN modulate,
QK-Norm + RoPE, gated residual) against the fp64 oracle."""

import numpy as np
import pytest
import torch

from gpu_common import cuda
from oracle import block as oblock
from video_diffusion_transformer_self_b200 import build, inputs, wan

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    wan.lib()


def _bf16_bound(got, want, extra):
    # bf16 output: half an ulp is <= 2^-8 of the value, plus fp32 slack
    err = np.abs(got - want)
    bound = 2.0 ** -8 * np.abs(want) + extra
    assert np.all(err <= bound), float(np.max(err / bound))


# row lengths across the 3, 6, 10 and 16 float4-per-thread variants
@pytest.mark.parametrize("B,L,D", [(1, 7, 1536), (2, 33, 5120), (1, 5, 8),
                                   (3, 4, 8192), (1, 5, 3072), (2, 3, 6144),
                                   (1, 3, 1540), (1, 2, 5124)])
def test_adaln_modulate(B, L, D):
    x = inputs.randn_f32((B, L, D), 11, 3.0) + 0.5
    shift = inputs.randn_f32((B, D), 12, 0.2)
    scale = inputs.randn_f32((B, D), 13, 0.2)
    out = torch.empty((B, L, D), dtype=torch.bfloat16, device="cuda")
    wan.adaln_modulate(cuda(x), cuda(shift), cuda(scale), out)
    torch.cuda.synchronize()
    want = oblock.adaln_modulate(x.numpy(), shift.numpy(), scale.numpy())
    _bf16_bound(out.double().cpu().numpy(), want, 1e-5 * (1 + np.abs(want)))


# heads <= 40 take the register-resident kernel (4, 8, 12 or 20 rows per
# lane by head count), more heads the two-pass one
@pytest.mark.parametrize("grid,B,H", [((2, 4, 4), 1, 2), ((3, 7, 13), 2, 12),
                                      ((5, 30, 52), 1, 40), ((2, 3, 5), 1, 1),
                                      ((2, 3, 5), 2, 3), ((2, 5, 7), 1, 39),
                                      ((2, 5, 7), 1, 41), ((2, 3, 5), 1, 48),
                                      ((2, 3, 5), 1, 8), ((2, 3, 5), 1, 9),
                                      ((2, 3, 5), 1, 16), ((2, 3, 5), 2, 24),
                                      ((2, 3, 5), 1, 25)])
def test_qk_norm_rope(grid, B, H):
    L = grid[0] * grid[1] * grid[2]
    q = inputs.randn_bf16((B, L, H, 128), 21, 2.0)
    k = inputs.randn_bf16((B, L, H, 128), 22, 0.5)
    wq = inputs.randn_f32((H * 128,), 23)
    wk = inputs.randn_f32((H * 128,), 24)
    g = wan.grid(*grid)
    table = wan.rope3d_table(g)
    qg, kg = cuda(q), cuda(k)
    wan.qk_norm_rope(qg, kg, cuda(wq), cuda(wk), g, table)
    torch.cuda.synchronize()
    for got, x, w in ((qg, q, wq), (kg, k, wk)):
        want = oblock.qk_norm_rope(x.double().numpy(), w.numpy(), grid)
        # |w| up to ~4: scale the fp32 slack with the pair's weighted norm
        _bf16_bound(got.double().cpu().numpy(), want,
                    1e-5 * (1 + np.abs(want)).max(axis=-1, keepdims=True))


@pytest.mark.parametrize("H", [4, 44])
@pytest.mark.parametrize("which", ["q", "k"])
def test_qk_norm_rope_one_tensor(H, which):
    grid, B = (2, 3, 5), 1
    L = 30
    q = inputs.randn_bf16((B, L, H, 128), 31)
    k = inputs.randn_bf16((B, L, H, 128), 32)
    w = inputs.randn_f32((H * 128,), 33)
    g = wan.grid(*grid)
    qg, kg = cuda(q), cuda(k)
    if which == "q":
        wan.qk_norm_rope(qg, None, cuda(w), None, g, wan.rope3d_table(g))
        done, untouched, x, x_other = qg, kg, q, k
    else:
        wan.qk_norm_rope(None, kg, None, cuda(w), g, wan.rope3d_table(g))
        done, untouched, x, x_other = kg, qg, k, q
    torch.cuda.synchronize()
    assert torch.equal(untouched.cpu(), x_other)
    want = oblock.qk_norm_rope(x.double().numpy(), w.numpy(), grid)
    _bf16_bound(done.double().cpu().numpy(), want,
                1e-5 * (1 + np.abs(want)).max(axis=-1, keepdims=True))


@pytest.mark.parametrize("B,L,D", [(1, 9, 1536), (2, 65, 5120)])
def test_gated_residual(B, L, D):
    x = inputs.randn_f32((B, L, D), 41)
    y = inputs.randn_bf16((B, L, D), 42)
    gate = inputs.randn_f32((B, D), 43)
    xg = cuda(x.clone())
    wan.gated_residual(xg, cuda(y), cuda(gate))
    torch.cuda.synchronize()
    want = oblock.gated_residual(x.numpy(), y.double().numpy(), gate.numpy())
    got = xg.double().cpu().numpy()
    # one fp32 fma: |err| <= 2^-24 (|x| + |y g|) (plus the product rounding)
    bound = 1.2e-7 * (np.abs(x.numpy()) + np.abs(want)) + 1e-30
    assert np.all(np.abs(got - want) <= 2 * bound)
