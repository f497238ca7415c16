"""Pins of the oracle's block prologue / epilogue: definition invariants and
agreement with torch's fp64 layer_norm / rms_norm."""

import numpy as np
import torch

from oracle import block, rope


def _rng(s):
    return np.random.default_rng(s)


def test_layer_norm_moments_and_torch():
    x = _rng(1).standard_normal((2, 7, 96)) * 3 + 1.5
    y = block.layer_norm(x)
    assert np.max(np.abs(y.mean(-1))) < 1e-12
    assert np.max(np.abs(y.var(-1) - 1)) < 1e-5  # eps = 1e-6 shrinks it
    ref = torch.nn.functional.layer_norm(torch.from_numpy(x), (96,),
                                         eps=1e-6).numpy()
    assert np.max(np.abs(y - ref)) < 1e-12


def test_modulate_special_cases():
    r = _rng(2)
    x = r.standard_normal((2, 5, 32))
    z = np.zeros((2, 32))
    assert np.max(np.abs(block.adaln_modulate(x, z, z) -
                         block.layer_norm(x))) < 1e-15
    shift = r.standard_normal((2, 32))
    scale = r.standard_normal((2, 32))
    got = block.adaln_modulate(x, shift, scale)
    want = block.layer_norm(x) * (1 + scale[:, None]) + shift[:, None]
    assert np.max(np.abs(got - want)) < 1e-14
    # scale = -1 removes the normalised input entirely
    only_shift = block.adaln_modulate(x, shift, -np.ones((2, 32)))
    assert np.max(np.abs(only_shift - shift[:, None])) < 1e-15


def test_rms_norm_unit_rms_scale_invariant_and_torch():
    r = _rng(3)
    x = r.standard_normal((3, 4, 64)) * 5
    w = r.standard_normal(64)
    y = block.rms_norm(x, np.ones(64))
    assert np.max(np.abs(np.sqrt((y * y).mean(-1)) - 1)) < 1e-6
    assert np.max(np.abs(block.rms_norm(7 * x, w) - block.rms_norm(x, w))) \
        < 1e-6
    ref = torch.nn.functional.rms_norm(torch.from_numpy(x), (64,),
                                       torch.from_numpy(w), eps=1e-6).numpy()
    assert np.max(np.abs(block.rms_norm(x, w) - ref)) < 1e-12


def test_qk_norm_rope_composition():
    r = _rng(4)
    g = (2, 3, 4)
    x = r.standard_normal((1, 24, 3, 128))
    w = r.standard_normal(3 * 128)
    got = block.qk_norm_rope(x, w, g)
    normed = block.rms_norm(x.reshape(1, 24, 384), w).reshape(x.shape)
    assert np.max(np.abs(got - rope.rope3d(normed, g))) < 1e-13
    # the norm spans all heads: scaling one head changes every head's output
    x2 = x.copy()
    x2[..., 0, :] *= 3
    assert np.max(np.abs(block.qk_norm_rope(x2, w, g)[..., 1, :] -
                         got[..., 1, :])) > 1e-3


def test_gated_residual():
    r = _rng(5)
    x, y = r.standard_normal((2, 3, 8)), r.standard_normal((2, 3, 8))
    assert np.array_equal(block.gated_residual(x, y, np.zeros((2, 8))), x)
    got = block.gated_residual(x, y, np.full((2, 8), 0.5))
    assert np.max(np.abs(got - (x + 0.5 * y))) < 1e-15
