"""3D rotary position embedding in fp64 (oracle; test infrastructure only).

Wan2.2 source reading, ch. 4, section "3D RoPE: letting a token know where it
is": each head's ``d = dim // num_heads = 128`` channels are split into three
bands built by ``rope_params(1024, d - 4*(d//6))`` (time, 44 channels) and
twice ``rope_params(1024, 2*(d//6))`` (height and width, 42 channels each),
concatenated in the order time, height, width.  At application every token
takes the rotation of its own (f, h, w) coordinate in each band, and the
rotation is applied to q and k as a complex multiplication, in float64 with
autocast disabled.  The section states that after rotation q.k depends only
on the coordinate difference of the two tokens (translation invariance).

Readings where the page is silent:

* base theta = 10000 (the workloads state it; the page does not print the
  body of ``rope_params``);
* within a band of width D the j-th complex pair (j = 0 .. D/2 - 1) turns by
  ``pos * theta ** (-2 j / D)``, each band with its own D, because
  ``rope_params`` is called once per band with that band's width;
* "complex multiplication" pairs adjacent channels (2j, 2j+1) as
  (real, imaginary) of one complex number;
* the tables cover positions 0 .. 1023 (the ``1024`` argument), so a grid
  side above 1024 is out of range.

The RoPE values themselves are parity unpinned: the pages print no rotated
number.  The pins are the invariants the page states or implies (identity at
position 0, per-pair norm preservation, translation invariance of q.k,
inverse rotation).
"""

import numpy as np

MAX_POS = 1024


def band_widths(head_dim):
    """Channel widths (time, height, width) of the three RoPE bands."""
    d6 = head_dim // 6
    return (head_dim - 4 * d6, 2 * d6, 2 * d6)


def band_angles(positions, width, theta=10000.0):
    """Angle table of one band: rows = positions, columns = complex pairs.

    ``angle[p, j] = p * theta ** (-2 j / width)`` for j < width / 2.
    """
    pos = np.asarray(positions, dtype=np.float64)
    j = np.arange(width // 2, dtype=np.float64)
    inv_freq = theta ** (-2.0 * j / width)
    return np.outer(pos, inv_freq)


def token_angles(grid, head_dim=128, theta=10000.0):
    """Per-token angles, shape [L, head_dim/2], bands in order t, h, w."""
    f_, h_, w_ = grid
    if max(grid) > MAX_POS or min(grid) < 1:
        raise ValueError("grid side outside the 1..1024 position table")
    wt, wh, ww = band_widths(head_dim)
    n = np.arange(f_ * h_ * w_)
    f = n // (h_ * w_)
    h = (n // w_) % h_
    w = n % w_
    return np.concatenate([band_angles(f, wt, theta),
                           band_angles(h, wh, theta),
                           band_angles(w, ww, theta)], axis=1)


def apply_angles(x, angles):
    """Rotate adjacent channel pairs of x by the given angles.

    x: [..., L, heads, head_dim] (any float); angles: [L, head_dim/2].
    Returns float64.  Pair (x[2j], x[2j+1]) viewed as x[2j] + i x[2j+1] is
    multiplied by exp(i * angle[j]).
    """
    x = np.asarray(x, dtype=np.float64)
    re = x[..., 0::2]
    im = x[..., 1::2]
    c = np.cos(angles)[:, None, :]
    s = np.sin(angles)[:, None, :]
    out = np.empty_like(x)
    out[..., 0::2] = re * c - im * s
    out[..., 1::2] = re * s + im * c
    return out


def rope3d(x, grid, theta=10000.0):
    """3D RoPE of q or k laid out [B, L, heads, head_dim], in float64."""
    x = np.asarray(x, dtype=np.float64)
    return apply_angles(x, token_angles(grid, x.shape[-1], theta))
