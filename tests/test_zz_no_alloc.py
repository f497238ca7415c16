"""The block-causal split call that allocates nothing
(wan_block_causal_attn_split_noalloc), called through the C ABI: its output
must match the workspace form's (wan_block_causal_attn_split, whose
workspace the caller allocates) within the attention tolerance, on two calls
in a row -- the second reuses the library's scratch array as the first left
it.  It is meant for callers that must not allocate device memory while
they run, so the test also checks that a problem too large for the fixed
array is refused before any device work.  This file is collected last."""

import ctypes
import math

import numpy as np
import pytest
import torch

from gpu_common import assert_attn_close, cuda, f64
from video_diffusion_transformer_self_b200 import build, inputs, wan

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    build.build()
    return wan.lib()


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def test_noalloc_matches_workspace_form_twice(lib):
    # a KV-cache step: the last 1,560-token chunk (one 480p latent frame)
    # against 4 chunks of cache, 12 heads, 3 key ranges
    B, H, chunk, n_chunks, n_split = 1, 12, 1560, 4, 3
    Lk = chunk * n_chunks
    off = Lk - chunk
    need = lib.wan_block_causal_attn_workspace_bytes(B, chunk, H, n_split)
    assert 0 < need <= lib.wan_block_causal_attn_noalloc_max_bytes()
    scale = 1.0 / math.sqrt(128)
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        seed = 7100 + 10 * call
        q = cuda(inputs.randn_bf16((B, chunk, H, 128), seed))
        k = cuda(inputs.randn_bf16((B, Lk, H, 128), seed + 1))
        v = cuda(inputs.randn_bf16((B, Lk, H, 128), seed + 2))
        ws = torch.empty(need, dtype=torch.uint8, device="cuda")
        want = torch.empty_like(q)
        got = torch.full_like(q, float("nan"))
        st = lib.wan_block_causal_attn_split(
            _p(q), _p(k), _p(v), _p(want), B, chunk, Lk, H, 128, chunk, off,
            scale, n_split, _p(ws), need, s)
        assert st == wan.WAN_OK, wan.status_string(st)
        st = lib.wan_block_causal_attn_split_noalloc(
            _p(q), _p(k), _p(v), _p(got), B, chunk, Lk, H, 128, chunk, off,
            scale, n_split, s)
        assert st == wan.WAN_OK, wan.status_string(st)
        torch.cuda.synchronize()
        assert wan.device_status() == 0
        assert_attn_close(f64(got), f64(want), "no-alloc call %d" % call)


def test_noalloc_refuses_what_does_not_fit(lib):
    # 4,680 queries x 40 heads x 3 ranges needs 292 MB of scratch
    p = ctypes.c_void_p(4096)
    o = ctypes.c_void_p(8192)
    assert lib.wan_block_causal_attn_workspace_bytes(1, 4680, 40, 3) > \
        lib.wan_block_causal_attn_noalloc_max_bytes()
    st = lib.wan_block_causal_attn_split_noalloc(
        p, p, p, o, 1, 4680, 65520, 40, 128, 4680, 60840, 0.088, 3, None)
    assert st == wan.WAN_ENOSPACE
    assert "scratch" in wan.status_string(st)
