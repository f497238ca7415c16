"""Pins of the oracle's 3D RoPE to the properties the page states."""

import numpy as np
import pytest

from oracle import rope


def _rng(seed):
    return np.random.default_rng(seed)


def test_band_widths(gold):
    assert list(rope.band_widths(128)) == gold("rope_band_widths_d128")
    assert sum(rope.band_widths(128)) == 128


def test_origin_is_identity():
    x = _rng(1).standard_normal((1, 1, 3, 128))
    assert np.array_equal(rope.rope3d(x, (1, 1, 1)), x)


def test_pair_norm_preserved():
    g = (3, 4, 5)
    x = _rng(2).standard_normal((2, 60, 2, 128))
    y = rope.rope3d(x, g)
    nx = x[..., 0::2] ** 2 + x[..., 1::2] ** 2
    ny = y[..., 0::2] ** 2 + y[..., 1::2] ** 2
    assert np.max(np.abs(nx - ny)) < 1e-12


def _rot_at(x, coord, theta=10000.0):
    """Rotate one vector x[128] as if it sat at grid coordinate ``coord``."""
    f, h, w = coord
    g = (f + 1, h + 1, w + 1)
    n = (f * g[1] + h) * g[2] + w
    xx = np.zeros((1, g[0] * g[1] * g[2], 1, 128))
    xx[0, n, 0] = x
    return rope.rope3d(xx, g, theta)[0, n, 0]


def test_translation_invariance():
    # q.k after rotation depends only on the coordinate difference.
    r = _rng(3)
    q, k = r.standard_normal(128), r.standard_normal(128)
    a, b = (2, 5, 1), (0, 3, 7)
    base = _rot_at(q, a) @ _rot_at(k, b)
    for c in [(1, 0, 0), (0, 4, 0), (0, 0, 9), (3, 2, 6)]:
        a2 = tuple(x + y for x, y in zip(a, c))
        b2 = tuple(x + y for x, y in zip(b, c))
        assert abs(_rot_at(q, a2) @ _rot_at(k, b2) - base) < 1e-11
    # and it does change with the difference itself
    assert abs(_rot_at(q, (3, 5, 1)) @ _rot_at(k, b) - base) > 1e-3


@pytest.mark.parametrize("axis,lo,hi", [(0, 0, 44), (1, 44, 86), (2, 86, 128)])
def test_band_placement(axis, lo, hi):
    # Moving a token along one axis changes only that axis's band
    # (bands concatenated in the order time, height, width).
    x = _rng(4).standard_normal(128)
    c0 = [1, 1, 1]
    c1 = list(c0)
    c1[axis] += 2
    d = _rot_at(x, tuple(c1)) - _rot_at(x, tuple(c0))
    mask = np.zeros(128, bool)
    mask[lo:hi] = True
    assert np.max(np.abs(d[~mask])) == 0.0
    assert np.max(np.abs(d[mask])) > 1e-3


def test_first_pair_of_each_band_turns_by_position():
    # j = 0 has frequency theta^0 = 1: the angle equals the coordinate.
    x = np.zeros(128)
    for off in (0, 44, 86):
        x[off] = 1.0
    coord = (2, 3, 4)
    y = _rot_at(x, coord)
    for off, p in zip((0, 44, 86), coord):
        assert abs(y[off] - np.cos(p)) < 1e-15
        assert abs(y[off + 1] - np.sin(p)) < 1e-15


def test_inverse_rotation():
    g = (2, 3, 4)
    x = _rng(5).standard_normal((1, 24, 2, 128))
    ang = rope.token_angles(g)
    y = rope.apply_angles(rope.apply_angles(x, ang), -ang)
    assert np.max(np.abs(y - x)) < 1e-12


def test_grid_bounds():
    with pytest.raises(ValueError):
        rope.token_angles((1025, 1, 1))
    with pytest.raises(ValueError):
        rope.token_angles((0, 1, 1))
