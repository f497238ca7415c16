"""The ctypes binding rejects tensors of the wrong device, dtype, layout or
size before calling into the library (no GPU needed: every case below is
refused in Python)."""

import pytest
import torch

from video_diffusion_transformer_self_b200 import build, wan


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    wan.lib()


def _bf16(*shape):
    return torch.zeros(shape, dtype=torch.bfloat16)


def test_attention_rejects_cpu_and_layout():
    g = wan.grid(2, 4, 4)
    q = _bf16(1, 32, 2, 128)
    with pytest.raises(ValueError):
        wan.self_attn(q, q, q, q, g)                    # CPU tensors
    with pytest.raises(ValueError):
        wan.self_attn(q.float(), q, q, q, g)            # wrong dtype
    with pytest.raises(ValueError):
        wan.cross_attn(q[0], q, q, q, [3])              # 3-D tensor
    with pytest.raises(ValueError):
        wan.block_causal_attn(q.transpose(1, 2), q, q, q, 8)  # not contiguous


def test_step_kernels_reject_cpu_and_dtype():
    x = torch.zeros(16)
    with pytest.raises(ValueError):
        wan.fm_step(x, x, None, 1.0, 1.0, 0.9)
    with pytest.raises(ValueError):
        wan.unipc_step(x, x, None, None, x, x, None, 1.0, [1.0, 0.0], 0)
    with pytest.raises(ValueError):
        wan.gated_residual(torch.zeros(1, 2, 8), _bf16(1, 2, 8),
                           torch.zeros(1, 8))
    with pytest.raises(ValueError):
        wan.adaln_modulate(torch.zeros(1, 2, 8, dtype=torch.float64),
                           torch.zeros(1, 8), torch.zeros(1, 8),
                           _bf16(1, 2, 8))
    with pytest.raises(ValueError):
        wan.transpose_blocks(torch.zeros(64, dtype=torch.uint8),
                             torch.zeros(64, dtype=torch.uint8), 2, 2, 16)


def test_host_calls_validate():
    with pytest.raises(wan.WanError):
        wan.fm_sigmas(0, 12.0)
    with pytest.raises(wan.WanError):
        wan.unipc_coeffs([1.0, 0.5, 0.5, 0.0], 1)       # not decreasing
    with pytest.raises(wan.WanError):
        wan.token_grid(80, 720, 1280)                   # frames not 4n + 1
