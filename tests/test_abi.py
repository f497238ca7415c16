"""C-ABI checks that need no GPU: the library loads, exports every symbol
include/wan.h declares, its host-only calls agree with the oracle, and its
argument checks reject bad calls before touching a device."""

import ctypes
import math
import os
import re

import numpy as np
import pytest

from oracle import grid as ogrid
from oracle import schedule as osched
from video_diffusion_transformer_self_b200 import build, wan

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return wan.lib()


def declared_functions():
    src = open(os.path.join(ROOT, "include", "wan.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(wan_[a-z0-9_]+)\s*\(", src)))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(wan._SIGNATURES)


def test_status_strings(lib):
    for st in (0, -1, -2, -3, -4, -5):
        assert wan.status_string(st)
    assert wan.status_string(-99) == "unknown status"
    assert lib.wan_version() >= 100


@pytest.mark.parametrize("frames,h,w", [(81, 720, 1280), (81, 480, 832),
                                        (165, 480, 832), (17, 480, 832),
                                        (5, 64, 64), (1, 16, 16)])
def test_token_grid_matches_oracle(lib, frames, h, w):
    lat, g = wan.token_grid(frames, h, w)
    assert lat == ogrid.latent_shape(frames, h, w)
    assert tuple(g) == ogrid.token_grid(frames, h, w)


@pytest.mark.parametrize("frames,h,w", [(80, 720, 1280), (82, 720, 1280),
                                        (0, 64, 64), (81, 100, 64),
                                        (81, 64, 8)])
def test_token_grid_rejects(lib, frames, h, w):
    with pytest.raises(wan.WanError) as e:
        wan.token_grid(frames, h, w)
    assert e.value.status == wan.WAN_EINVAL


@pytest.mark.parametrize("n,shift,smax", [(40, 12.0, 1.0), (40, 5.0, 1.0),
                                          (40, 12.0, 0.999), (1, 3.0, 1.0),
                                          (7, 1.0, 1.0)])
def test_sigmas_match_oracle(lib, n, shift, smax):
    got = np.array(wan.fm_sigmas(n, shift, smax))
    want = osched.sigmas(n, shift, smax)
    assert got.shape == want.shape
    assert np.max(np.abs(got - want)) <= 1e-15


def test_sigmas_reject(lib):
    out = (ctypes.c_double * 4)()
    assert lib.wan_fm_sigmas(0, 12.0, 1.0, out) == wan.WAN_EINVAL
    assert lib.wan_fm_sigmas(3, -1.0, 1.0, out) == wan.WAN_EINVAL
    assert lib.wan_fm_sigmas(3, 2.0, 1.5, out) == wan.WAN_EINVAL
    assert lib.wan_fm_sigmas(3, 2.0, 1.0, None) == wan.WAN_EINVAL


def test_rope_table_bytes(lib):
    assert wan.rope3d_table_bytes(wan.grid(21, 45, 80)) == \
        (21 + 45 + 80) * 22 * 8
    assert wan.rope3d_table_bytes(wan.grid(1025, 1, 1)) == 0
    assert wan.rope3d_table_bytes(wan.grid(2, 4, 4), 64) == 0


def _g(F, H, W):
    return wan.grid(F, H, W)


def test_argument_checks_without_device(lib):
    # All of these fail validation before any device call.
    p = ctypes.c_void_p(4096)
    odd = ctypes.c_void_p(4098)
    g = _g(2, 4, 4)
    L = lib
    assert L.wan_self_attn(None, p, p, p, 1, g, 2, 128, None, 0.1, None) \
        == wan.WAN_EINVAL
    assert L.wan_self_attn(p, p, p, ctypes.c_void_p(8192), 1, g, 2, 64, None,
                           0.1, None) == wan.WAN_EINVAL
    assert L.wan_self_attn(p, p, p, ctypes.c_void_p(8192), 1, g, 2, 128, None,
                           -1.0, None) == wan.WAN_EINVAL
    assert L.wan_self_attn(p, p, p, ctypes.c_void_p(8192), 1, _g(0, 4, 4), 2,
                           128, None, 0.1, None) == wan.WAN_EINVAL
    assert L.wan_self_attn(odd, p, p, ctypes.c_void_p(8192), 1, g, 2, 128,
                           None, 0.1, None) == wan.WAN_EALIGN
    assert L.wan_self_attn(p, p, p, p, 1, g, 2, 128, None, 0.1, None) \
        == wan.WAN_EINVAL  # o aliases q
    assert L.wan_self_attn(p, p, p, ctypes.c_void_p(8192), 1, _g(1025, 1, 1),
                           2, 128, p, 0.1, None) == wan.WAN_EINVAL
    lens = (ctypes.c_int32 * 2)(5, 0)
    assert L.wan_cross_attn(p, p, p, ctypes.c_void_p(8192), lens, 2, 32, 16,
                            2, 128, 0.1, None) == wan.WAN_EINVAL  # len 0
    lens = (ctypes.c_int32 * 2)(5, 17)
    assert L.wan_cross_attn(p, p, p, ctypes.c_void_p(8192), lens, 2, 32, 16,
                            2, 128, 0.1, None) == wan.WAN_EINVAL  # len > Lk
    assert L.wan_cross_attn(p, p, p, ctypes.c_void_p(8192), None, 2, 32, 16,
                            2, 128, 0.1, None) == wan.WAN_EINVAL
    big = (ctypes.c_int32 * 513)(*([1] * 513))
    assert L.wan_cross_attn(p, p, p, ctypes.c_void_p(8192), big, 513, 32, 16,
                            2, 128, 0.1, None) == wan.WAN_EINVAL
    assert L.wan_fm_step(None, p, None, 1.0, 10, 1.0, 0.9, None) \
        == wan.WAN_EINVAL
    assert L.wan_fm_step(odd, p, None, 1.0, 10, 1.0, 0.9, None) \
        == wan.WAN_EALIGN
    assert L.wan_fm_step(p, p, None, 1.0, 10, 1.0, 0.9, None) \
        == wan.WAN_EINVAL  # x aliases v
    assert L.wan_fm_step(p, ctypes.c_void_p(8192), None, 1.0, 10,
                         math.nan, 0.9, None) == wan.WAN_EINVAL
    assert L.wan_fm_step(None, None, None, 1.0, 0, 1.0, 0.9, None) \
        == wan.WAN_OK  # empty input: nothing to do
    assert L.wan_rope3d_qk(p, p, 1, g, 2, 128, None, None) == wan.WAN_EINVAL
    assert L.wan_rope3d_qk(None, None, 1, g, 2, 128, p, None) \
        == wan.WAN_EINVAL
    assert L.wan_rope3d_qk(odd, None, 1, g, 2, 128, p, None) \
        == wan.WAN_EALIGN
    o = ctypes.c_void_p(8192)
    assert L.wan_block_causal_attn(p, p, p, o, 1, 10, 20, 2, 128, 0, 0, 0.1,
                                   None) == wan.WAN_EINVAL  # chunk 0
    assert L.wan_block_causal_attn(p, p, p, o, 1, 10, 20, 2, 128, 5, 11, 0.1,
                                   None) == wan.WAN_EINVAL  # past the keys
    assert L.wan_block_causal_attn(p, p, p, o, 1, 10, 20, 2, 128, 5, -1, 0.1,
                                   None) == wan.WAN_EINVAL
    assert L.wan_block_causal_attn(odd, p, p, o, 1, 10, 20, 2, 128, 5, 0, 0.1,
                                   None) == wan.WAN_EALIGN
    assert L.wan_adaln_modulate(p, p, p, o, 1, 4, 6, 1e-6, None) \
        == wan.WAN_EINVAL  # D % 4
    assert L.wan_adaln_modulate(p, p, p, o, 1, 4, 8196 + 4, 1e-6, None) \
        == wan.WAN_EINVAL  # D too large
    assert L.wan_adaln_modulate(p, p, p, o, 1, 4, 8, 0.0, None) \
        == wan.WAN_EINVAL  # eps
    assert L.wan_adaln_modulate(odd, p, p, o, 1, 4, 8, 1e-6, None) \
        == wan.WAN_EALIGN
    assert L.wan_qk_norm_rope(p, None, None, None, 1, g, 2, 128, p, 1e-6,
                              None) == wan.WAN_EINVAL  # q without weight
    assert L.wan_qk_norm_rope(None, None, p, p, 1, g, 2, 128, p, 1e-6,
                              None) == wan.WAN_EINVAL
    assert L.wan_qk_norm_rope(p, p, p, p, 1, g, 2, 128, p, 1e-6, None) \
        == wan.WAN_EINVAL  # q aliases k
    assert L.wan_gated_residual(p, p, p, 1, 4, 6, None) == wan.WAN_EINVAL
    assert L.wan_gated_residual(odd, p, p, 1, 4, 8, None) == wan.WAN_EALIGN
    big_o = ctypes.c_void_p(1 << 20)
    assert L.wan_transpose_blocks(p, big_o, 2, 3, 24, None) == wan.WAN_EINVAL
    assert L.wan_transpose_blocks(p, ctypes.c_void_p(4096 + 64), 2, 3, 16,
                                  None) == wan.WAN_EINVAL  # overlap
    assert L.wan_transpose_blocks(odd, big_o, 2, 3, 16, None) \
        == wan.WAN_EALIGN
    assert L.wan_transpose_blocks(None, None, 0, 3, 16, None) == wan.WAN_OK
    assert L.wan_transpose_blocks(None, big_o, 2, 3, 16, None) \
        == wan.WAN_EINVAL


def test_split_block_causal_host_checks(lib):
    # workspace size: n_split * rows * (512 + 8) bytes, 0 without a split
    assert lib.wan_block_causal_attn_workspace_bytes(1, 4680, 40, 1) == 0
    assert lib.wan_block_causal_attn_workspace_bytes(1, 4680, 40, 3) == \
        3 * 4680 * 40 * 520
    assert lib.wan_block_causal_attn_workspace_bytes(2, 10, 3, 2) == \
        2 * 2 * 10 * 3 * 520
    assert lib.wan_block_causal_attn_workspace_bytes(1, 10, 2, 9) == 0
    assert lib.wan_block_causal_attn_workspace_bytes(0, 10, 2, 2) == 0
    p = ctypes.c_void_p(4096)
    o = ctypes.c_void_p(8192)
    ws = ctypes.c_void_p(1 << 24)
    need = lib.wan_block_causal_attn_workspace_bytes(1, 600, 2, 2)
    L = lib
    for fn in (L.wan_block_causal_attn_split,
               L.wan_block_causal_attn_pair_split):
        # n_split out of range
        assert fn(p, p, p, o, 1, 600, 600, 2, 128, 120, 0, 0.1, 0, ws, need,
                  None) == wan.WAN_EINVAL
        assert fn(p, p, p, o, 1, 600, 600, 2, 128, 120, 0, 0.1, 9, ws, need,
                  None) == wan.WAN_EINVAL
        # the lightest item (the first 256 queries, keys < 256) has 2 key
        # blocks: 3 ranges would leave one empty
        assert fn(p, p, p, o, 1, 600, 600, 2, 128, 128, 0, 0.1, 3, ws,
                  1 << 20, None) == wan.WAN_EINVAL
        # workspace missing, too small, misaligned
        assert fn(p, p, p, o, 1, 600, 600, 2, 128, 120, 0, 0.1, 2, None,
                  need, None) == wan.WAN_EINVAL
        assert fn(p, p, p, o, 1, 600, 600, 2, 128, 120, 0, 0.1, 2, ws,
                  need - 1, None) == wan.WAN_EINVAL
        assert fn(p, p, p, o, 1, 600, 600, 2, 128, 120, 0, 0.1, 2,
                  ctypes.c_void_p((1 << 24) + 8), need, None) \
            == wan.WAN_EALIGN
    assert L.wan_block_causal_attn_splits(1, 10, 5, 2, 4, 0) == wan.WAN_EINVAL
    assert L.wan_block_causal_attn_pair_splits(1, 10, 5, 2, 4, 0) \
        == wan.WAN_EINVAL
