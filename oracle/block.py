"""Block prologue / epilogue around attention in fp64 (oracle; test
infrastructure only).

Wan2.2 source reading, ch. 4, section "Full forward of one block": the
self-attention input is ``norm1(x) * (1 + e[1]) + e[0]`` and the block output
``x + y * e[2]``, all under fp32 autocast, with e the six modulation chunks
(shift, scale, gate for self-attention; the same three for the FFN).  Section
"3D RoPE", last paragraph: in the self-attention, q and k each go through an
RMSNorm (QK-Norm) after their linear layers, before the rotation.

Readings taken where the page is silent:

* norm1 is a LayerNorm over the model dim without its own affine weights
  (the modulation supplies scale and shift), eps = 1e-6;
* QK-Norm is an RMSNorm over the whole projection output (all heads, dim =
  heads * head_dim) with a learned per-channel weight, eps = 1e-6, applied
  before the 3D RoPE;
* shift / scale / gate are per batch row and channel ([B, dim]), broadcast
  over tokens.

Parity unpinned beyond what the pins fix: the pages print no values for
these steps, so the pins are the definitions' invariants (zero mean and unit
variance after LayerNorm, unit rms after RMSNorm, scale invariance) and
agreement with torch's fp64 layer_norm / rms_norm.
"""

import numpy as np

from . import rope as _rope

EPS = 1e-6


def layer_norm(x, eps=EPS):
    """(x - mean) / sqrt(var + eps) over the last axis, fp64."""
    x = np.asarray(x, dtype=np.float64)
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    return (x - mu) / np.sqrt(var + eps)


def adaln_modulate(x, shift, scale, eps=EPS):
    """norm1(x) * (1 + scale) + shift; x [B, L, D], shift/scale [B, D]."""
    y = layer_norm(x, eps)
    return y * (1.0 + np.asarray(scale, np.float64)[:, None, :]) + \
        np.asarray(shift, np.float64)[:, None, :]


def rms_norm(x, weight, eps=EPS):
    """x / sqrt(mean(x^2) + eps) * weight over the last axis, fp64."""
    x = np.asarray(x, dtype=np.float64)
    ms = (x * x).mean(axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * np.asarray(weight, np.float64)


def qk_norm_rope(x, weight, grid, theta=10000.0, eps=EPS):
    """QK-Norm over all heads of a token, then 3D RoPE.

    x: [B, L, heads, head_dim]; weight: [heads * head_dim].
    """
    x = np.asarray(x, dtype=np.float64)
    b_, l_, h_, d_ = x.shape
    y = rms_norm(x.reshape(b_, l_, h_ * d_), weight, eps)
    return _rope.rope3d(y.reshape(b_, l_, h_, d_), grid, theta)


def gated_residual(x, y, gate):
    """x + y * gate; x, y [B, L, D], gate [B, D], fp64."""
    return np.asarray(x, np.float64) + np.asarray(y, np.float64) * \
        np.asarray(gate, np.float64)[:, None, :]
