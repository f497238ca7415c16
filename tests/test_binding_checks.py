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


# ---- shapes and sizes: checked before the device, so CPU tensors with a
# mismatched shape are refused for the shape (the kernels build their tensor
# maps and strides from q's heads, the grid's F*H*W and k's length, so any
# mismatch would read or write past an allocation).

def test_self_attn_rejects_shape_mismatch():
    g = wan.grid(2, 4, 4)
    q = _bf16(1, 32, 2, 128)
    with pytest.raises(ValueError, match="shape"):
        wan.self_attn(q, _bf16(1, 32, 3, 128), q, q, g)     # k heads
    with pytest.raises(ValueError, match="shape"):
        wan.self_attn(q, q, _bf16(1, 31, 2, 128), q, g)     # v length
    with pytest.raises(ValueError, match="shape"):
        wan.self_attn(q, q, q, _bf16(2, 32, 2, 128), g)     # o batch
    with pytest.raises(ValueError, match="tokens"):
        wan.self_attn(q, q, q, q, wan.grid(2, 4, 5))        # L != F*H*W
    with pytest.raises(ValueError, match="bytes"):
        wan.self_attn(q, q, q, q, g, table=torch.zeros(16, dtype=torch.uint8))


def test_cross_and_causal_reject_shape_mismatch():
    q = _bf16(2, 40, 2, 128)
    kc = _bf16(2, 16, 2, 128)
    with pytest.raises(ValueError, match="shape"):
        wan.cross_attn(q, kc, _bf16(2, 15, 2, 128), q.clone(), [3, 4])
    with pytest.raises(ValueError, match="shape"):
        wan.cross_attn(q, _bf16(1, 16, 2, 128), _bf16(1, 16, 2, 128),
                       q.clone(), [3, 4])                      # k batch
    with pytest.raises(ValueError, match="shape"):
        wan.cross_attn(q, _bf16(2, 16, 4, 128), _bf16(2, 16, 4, 128),
                       q.clone(), [3, 4])                      # k heads
    with pytest.raises(ValueError, match="shape"):
        wan.cross_attn(q, kc, kc.clone(), _bf16(2, 41, 2, 128), [3, 4])
    with pytest.raises(ValueError, match="lengths"):
        wan.cross_attn(q, kc, kc.clone(), q.clone(), [3])
    k = _bf16(2, 80, 2, 128)
    with pytest.raises(ValueError, match="shape"):
        wan.block_causal_attn(q, k, _bf16(2, 79, 2, 128), q.clone(), 8)
    with pytest.raises(ValueError, match="shape"):
        wan.block_causal_attn(q, k, k.clone(), _bf16(2, 40, 1, 128), 8)


def test_rope_and_block_kernels_reject_sizes():
    g = wan.grid(2, 4, 4)
    q = _bf16(1, 32, 2, 128)
    with pytest.raises(ValueError, match="shape"):
        wan.rope3d_qk(q, _bf16(1, 32, 1, 128), g, torch.zeros(4096,
                                                             dtype=torch.uint8))
    with pytest.raises(ValueError, match="tokens"):
        wan.rope3d_qk(q, q.clone(), wan.grid(1, 4, 4),
                      torch.zeros(4096, dtype=torch.uint8))
    with pytest.raises(ValueError, match="bytes"):
        wan.rope3d_qk(q, q.clone(), g, torch.zeros(8, dtype=torch.uint8))
    with pytest.raises(ValueError, match="elements"):
        wan.qk_norm_rope(q, q.clone(), torch.zeros(255), torch.zeros(256), g,
                         torch.zeros(4096, dtype=torch.uint8))
    x = torch.zeros(1, 2, 8)
    with pytest.raises(ValueError, match="size"):
        wan.gated_residual(x, _bf16(1, 2, 7), torch.zeros(1, 8))
    with pytest.raises(ValueError, match="elements"):
        wan.gated_residual(x, _bf16(1, 2, 8), torch.zeros(1, 7))
    with pytest.raises(ValueError, match="elements"):
        wan.adaln_modulate(x, torch.zeros(1, 8), torch.zeros(1, 8),
                           _bf16(1, 2, 7))
    with pytest.raises(ValueError, match="elements"):
        wan.adaln_modulate(x, torch.zeros(1, 9), torch.zeros(1, 8),
                           _bf16(1, 2, 8))
    with pytest.raises(ValueError, match="elements"):
        wan.fm_step(torch.zeros(16), torch.zeros(15), None, 1.0, 1.0, 0.9)
    with pytest.raises(ValueError, match="elements"):
        wan.fm_step(torch.zeros(16), torch.zeros(16), torch.zeros(17), 1.0,
                    1.0, 0.9)


def test_right_shapes_on_cpu_fail_only_for_the_device():
    g = wan.grid(2, 4, 4)
    q = _bf16(1, 32, 2, 128)
    with pytest.raises(ValueError, match="CUDA"):
        wan.self_attn(q, q.clone(), q.clone(), q.clone(), g)
    with pytest.raises(ValueError, match="CUDA"):
        wan.fm_step(torch.zeros(16), torch.zeros(16), None, 1.0, 1.0, 0.9)
