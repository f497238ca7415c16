"""ctypes binding of libwan.so (declared in include/wan.h).

Argument marshalling only: torch tensors are turned into raw device
pointers, sizes and the current CUDA stream, and every status code other
than WAN_OK raises ``WanError``.  All arithmetic of the hot path runs in the
library's CUDA kernels (or, for the grid / schedule / RoPE-table set-up
calls, in the library's host code).  There is no fallback: if libwan.so is
missing or fails to load, importing the functions raises.
"""

import ctypes
import math
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libwan.so")

WAN_OK = 0
WAN_EINVAL = -1
WAN_EALIGN = -2
WAN_EUNSUPPORTED = -3
WAN_ECUDA = -4
WAN_ETIMEOUT = -5
WAN_ENOSPACE = -6


class WanError(RuntimeError):
    def __init__(self, status, what):
        self.status = status
        super().__init__("%s: %s (%d)" % (what, status_string(status), status))


class Grid(ctypes.Structure):
    _fields_ = [("F", ctypes.c_int32), ("H", ctypes.c_int32),
                ("W", ctypes.c_int32)]

    def __iter__(self):
        return iter((self.F, self.H, self.W))

    def __repr__(self):
        return "Grid(%d, %d, %d)" % (self.F, self.H, self.W)


class UniPCCoef(ctypes.Structure):
    """wan_unipc_coef_t: folded coefficients of one UniPC stop."""
    _fields_ = [("sigma", ctypes.c_double), ("cx", ctypes.c_double),
                ("cm1", ctypes.c_double), ("cm2", ctypes.c_double),
                ("cm", ctypes.c_double), ("px", ctypes.c_double),
                ("pm", ctypes.c_double), ("pm1", ctypes.c_double),
                ("pred_order", ctypes.c_int32),
                ("corr_order", ctypes.c_int32)]

    def as_dict(self):
        return {name: getattr(self, name) for name, _ in self._fields_}


_P = ctypes.c_void_p
_I = ctypes.c_int
_D = ctypes.POINTER(ctypes.c_double)
_SIGNATURES = {
    "wan_status_string": (ctypes.c_char_p, [_I]),
    "wan_version": (_I, []),
    "wan_token_grid": (_I, [_I, _I, _I, ctypes.POINTER(ctypes.c_int32),
                            ctypes.POINTER(Grid)]),
    "wan_rope3d_table_bytes": (ctypes.c_size_t, [Grid, _I]),
    "wan_rope3d_table": (_I, [Grid, _I, ctypes.c_double, _P,
                              ctypes.c_size_t, _P]),
    "wan_rope3d_qk": (_I, [_P, _P, _I, Grid, _I, _I, _P, _P]),
    "wan_self_attn": (_I, [_P, _P, _P, _P, _I, Grid, _I, _I, _P,
                           ctypes.c_float, _P]),
    "wan_self_attn_rope_q": (_I, [_P, _P, _P, _P, _I, Grid, _I, _I, _P,
                                  ctypes.c_float, _P]),
    "wan_self_attn_pair": (_I, [_P, _P, _P, _P, _I, Grid, _I, _I, _P,
                                ctypes.c_float, _P]),
    "wan_cross_attn": (_I, [_P, _P, _P, _P, ctypes.POINTER(ctypes.c_int32),
                            _I, _I, _I, _I, _I, ctypes.c_float, _P]),
    "wan_block_causal_attn": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _I,
                                   _I, ctypes.c_float, _P]),
    "wan_block_causal_attn_pair": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I,
                                        _I, _I, ctypes.c_float, _P]),
    "wan_block_causal_attn_split": (_I, [_P, _P, _P, _P, _I, _I, _I, _I,
                                         _I, _I, _I, ctypes.c_float, _I, _P,
                                         ctypes.c_size_t, _P]),
    "wan_block_causal_attn_workspace_bytes": (ctypes.c_size_t,
                                              [_I, _I, _I, _I]),
    "wan_block_causal_attn_splits": (_I, [_I, _I, _I, _I, _I, _I]),
    "wan_block_causal_attn_pair_split": (_I, [_P, _P, _P, _P, _I, _I, _I,
                                              _I, _I, _I, _I, ctypes.c_float,
                                              _I, _P, ctypes.c_size_t, _P]),
    "wan_block_causal_attn_pair_splits": (_I, [_I, _I, _I, _I, _I, _I]),
    "wan_block_causal_attn_split_noalloc": (_I, [_P, _P, _P, _P, _I, _I, _I,
                                                 _I, _I, _I, _I,
                                                 ctypes.c_float, _I, _P]),
    "wan_block_causal_attn_noalloc_max_bytes": (ctypes.c_size_t, []),
    "wan_adaln_modulate": (_I, [_P, _P, _P, _P, _I, _I, _I, ctypes.c_float,
                                _P]),
    "wan_qk_norm_rope": (_I, [_P, _P, _P, _P, _I, Grid, _I, _I, _P,
                              ctypes.c_float, _P]),
    "wan_gated_residual": (_I, [_P, _P, _P, _I, _I, _I, _P]),
    "wan_fm_sigmas": (_I, [_I, ctypes.c_double, ctypes.c_double,
                           ctypes.POINTER(ctypes.c_double)]),
    "wan_fm_step": (_I, [_P, _P, _P, ctypes.c_float, ctypes.c_int64,
                         ctypes.c_double, ctypes.c_double, _P]),
    "wan_unipc_coeffs": (_I, [_D, _I, _I, ctypes.POINTER(UniPCCoef)]),
    "wan_unipc_step": (_I, [_P, _P, _P, _P, _P, _P, _P, ctypes.c_float,
                            ctypes.c_int64, _D, _I, _I, _P]),
    "wan_transpose_blocks": (_I, [_P, _P, ctypes.c_int64, ctypes.c_int64,
                                  ctypes.c_int64, _P]),
    "wan_attn_pair_resident_clusters": (_I, []),
    "wan_wait_selftest": (_I, [_I, _P]),
    "wan_device_status": (_I, [_I]),
}

_lib = None


def lib():
    """The loaded library (ctypes.CDLL); raises if it cannot be loaded."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                "libwan.so not built: run `python -m "
                "video_diffusion_transformer_self_b200.build`")
        l = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(l, name)
            fn.restype = res
            fn.argtypes = args
        _lib = l
    return _lib


def status_string(status):
    return lib().wan_status_string(int(status)).decode()


def _check(status, what):
    if status != WAN_OK:
        raise WanError(status, what)


def _stream(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


# Argument checks run in this order: dtype / rank / layout, then shapes and
# sizes against each other, then the device (every tensor on one CUDA
# device), all before the library is called.


def _bf16_bl(t, name):
    import torch
    if t.dtype != torch.bfloat16 or t.dim() != 4 or not t.is_contiguous():
        raise ValueError("%s must be a contiguous bf16 [B, L, heads, d] "
                         "tensor" % name)


def _on_cuda(*named):
    """Every given (name, tensor) pair (None skipped) is a CUDA tensor, all
    on the same device."""
    for name, t in named:
        if t is not None and not t.is_cuda:
            raise ValueError("%s must be a CUDA tensor" % name)
    devs = {t.device for _, t in named if t is not None}
    if len(devs) > 1:
        raise ValueError("tensors on different devices: %s" % ", ".join(
            "%s on %s" % (name, t.device) for name, t in named
            if t is not None))


def _shape_is(t, shape, name):
    if tuple(t.shape) != tuple(shape):
        raise ValueError("%s has shape %s, expected %s"
                         % (name, tuple(t.shape), tuple(shape)))


def _grid_tokens(g):
    return int(g.F) * int(g.H) * int(g.W)


def _check_table(table, g, head_dim, name="table"):
    """A RoPE table must be a contiguous CUDA tensor of at least
    rope3d_table_bytes(g) bytes (the kernels read that many)."""
    if table is None:
        return
    if not table.is_contiguous():
        raise ValueError("%s must be a contiguous tensor" % name)
    need = rope3d_table_bytes(g, head_dim)
    if need == 0:
        raise ValueError("grid %r has no RoPE table" % (g,))
    if table.numel() * table.element_size() < need:
        raise ValueError("%s holds %d bytes, grid %r needs %d"
                         % (name, table.numel() * table.element_size(), g,
                            need))


def _f32_n(t, n, name):
    """Contiguous fp32 tensor of exactly n elements."""
    _f32(t, name)
    if t.numel() != n:
        raise ValueError("%s has %d elements, expected %d"
                         % (name, t.numel(), n))


# ---------------------------------------------------------------- host ---

def token_grid(frames, height, width):
    """(latent shape (16, F, h, w), token Grid) for a pixel video."""
    lat = (ctypes.c_int32 * 4)()
    g = Grid()
    _check(lib().wan_token_grid(frames, height, width, lat, ctypes.byref(g)),
           "wan_token_grid")
    return tuple(lat), g


def grid(F, H, W):
    return Grid(F, H, W)


def fm_sigmas(n_steps, shift, s_max=1.0):
    """sigma_0 .. sigma_N (list of N + 1 floats)."""
    out = (ctypes.c_double * (n_steps + 1))()
    _check(lib().wan_fm_sigmas(n_steps, shift, s_max, out), "wan_fm_sigmas")
    return list(out)


def rope3d_table_bytes(g, head_dim=128):
    return lib().wan_rope3d_table_bytes(g, head_dim)


# -------------------------------------------------------------- device ---

def rope3d_table(g, theta=10000.0, head_dim=128, out=None, stream=None):
    """Device RoPE table for grid g (a uint8 CUDA tensor)."""
    import torch
    n = rope3d_table_bytes(g, head_dim)
    if n == 0:
        raise WanError(WAN_EINVAL, "wan_rope3d_table_bytes")
    if out is None:
        out = torch.empty(n, dtype=torch.uint8, device="cuda")
    elif not out.is_contiguous() or out.numel() * out.element_size() < n:
        raise ValueError("out must be a contiguous tensor of at least %d "
                         "bytes" % n)
    _on_cuda(("out", out))
    _check(lib().wan_rope3d_table(g, head_dim, theta, _ptr(out), out.numel(),
                                  _stream(stream)), "wan_rope3d_table")
    return out


def rope3d_qk(q, k, g, table, stream=None):
    """In-place 3D RoPE of q and k ([B, L, heads, 128] bf16)."""
    t = q if q is not None else k
    if t is None:
        raise ValueError("q and k are both None")
    for name, x in (("q", q), ("k", k)):
        if x is not None:
            _bf16_bl(x, name)
            _shape_is(x, t.shape, name)
    if t.shape[1] != _grid_tokens(g):
        raise ValueError("q/k hold %d tokens, grid %r has %d"
                         % (t.shape[1], g, _grid_tokens(g)))
    _check_table(table, g, t.shape[3])
    if table is None:
        raise ValueError("rope3d_qk needs a table")
    _on_cuda(("q", q), ("k", k), ("table", table))
    _check(lib().wan_rope3d_qk(_ptr(q), _ptr(k), t.shape[0], g, t.shape[2],
                               t.shape[3], _ptr(table), _stream(stream)),
           "wan_rope3d_qk")


def self_attn(q, k, v, o, g, table=None, softmax_scale=None, stream=None):
    """o = softmax(rope(q) rope(k)^T * scale) v; RoPE fused if table given."""
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o)):
        _bf16_bl(t, name)
        _shape_is(t, q.shape, name)
    B, L, H, D = q.shape
    if L != _grid_tokens(g):
        raise ValueError("q holds %d tokens, grid %r has %d"
                         % (L, g, _grid_tokens(g)))
    _check_table(table, g, D)
    _on_cuda(("q", q), ("k", k), ("v", v), ("o", o), ("table", table))
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(D)
    _check(lib().wan_self_attn(_ptr(q), _ptr(k), _ptr(v), _ptr(o), B, g, H, D,
                               _ptr(table), softmax_scale, _stream(stream)),
           "wan_self_attn")


def self_attn_rope_q(q, k, v, o, g, table, softmax_scale=None,
                     stream=None):
    """o = softmax(rope(q) k^T * scale) v: q rotated in the attention
    kernel's tile stage, k already rotated (e.g. rope3d_qk(None, k, ...))."""
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o)):
        _bf16_bl(t, name)
        _shape_is(t, q.shape, name)
    B, L, H, D = q.shape
    if L != _grid_tokens(g):
        raise ValueError("q holds %d tokens, grid %r has %d"
                         % (L, g, _grid_tokens(g)))
    if table is None:
        raise ValueError("self_attn_rope_q needs a table")
    _check_table(table, g, D)
    _on_cuda(("q", q), ("k", k), ("v", v), ("o", o), ("table", table))
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(D)
    _check(lib().wan_self_attn_rope_q(_ptr(q), _ptr(k), _ptr(v), _ptr(o), B,
                                      g, H, D, _ptr(table), softmax_scale,
                                      _stream(stream)),
           "wan_self_attn_rope_q")


def self_attn_pair(q, k, v, o, g, table_q=None, softmax_scale=None,
                   stream=None):
    """o = softmax(rope(q) k^T * scale) v over the grid's tokens, computed by
    the CTA-pair kernel (one MMA over two SMs).  k already rotated; q rotated
    in the kernel if table_q is given, else used as given."""
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o)):
        _bf16_bl(t, name)
        _shape_is(t, q.shape, name)
    B, L, H, D = q.shape
    if L != _grid_tokens(g):
        raise ValueError("q holds %d tokens, grid %r has %d"
                         % (L, g, _grid_tokens(g)))
    _check_table(table_q, g, D, "table_q")
    _on_cuda(("q", q), ("k", k), ("v", v), ("o", o), ("table_q", table_q))
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(D)
    _check(lib().wan_self_attn_pair(_ptr(q), _ptr(k), _ptr(v), _ptr(o), B, g,
                                    H, D, _ptr(table_q), softmax_scale,
                                    _stream(stream)), "wan_self_attn_pair")


def cross_attn(q, k_ctx, v_ctx, o, ctx_lens, softmax_scale=None,
               stream=None):
    """o[b] = softmax(q[b] k_ctx[b,:len_b]^T * scale) v_ctx[b,:len_b]."""
    for name, t in (("q", q), ("k_ctx", k_ctx), ("v_ctx", v_ctx), ("o", o)):
        _bf16_bl(t, name)
    B, Lq, H, D = q.shape
    Lk = k_ctx.shape[1]
    _shape_is(o, q.shape, "o")
    _shape_is(k_ctx, (B, Lk, H, D), "k_ctx")
    _shape_is(v_ctx, k_ctx.shape, "v_ctx")
    ctx_lens = [int(x) for x in ctx_lens]
    if len(ctx_lens) != B:
        raise ValueError("%d text lengths for batch %d" % (len(ctx_lens), B))
    _on_cuda(("q", q), ("k_ctx", k_ctx), ("v_ctx", v_ctx), ("o", o))
    lens = (ctypes.c_int32 * B)(*ctx_lens)
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(D)
    _check(lib().wan_cross_attn(_ptr(q), _ptr(k_ctx), _ptr(v_ctx), _ptr(o),
                                lens, B, Lq, Lk, H, D, softmax_scale,
                                _stream(stream)), "wan_cross_attn")


def block_causal_attn(q, k, v, o, chunk_tokens, q_offset=0,
                      softmax_scale=None, stream=None, pair=None,
                      split=None, workspace=None):
    """Chunk-wise causal attention: query a = q_offset + i sees keys
    j < (a // chunk_tokens + 1) * chunk_tokens (and j < Lk).

    pair: True runs the CTA-pair kernel (wan_block_causal_attn_pair), False
    the two-tile kernel (wan_block_causal_attn), None (the default) the
    kernel block_causal_default_pair picks.
    split: None (one key range per item), "auto" (block_causal_splits for
    the kernel chosen) or a count; with more than one range the call
    (wan_block_causal_attn_split or _pair_split) needs a workspace (a CUDA
    tensor of at least block_causal_workspace_bytes(...) bytes), allocated
    here with torch if not given."""
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o)):
        _bf16_bl(t, name)
    B, Lq, H, D = q.shape
    Lk = k.shape[1]
    _shape_is(o, q.shape, "o")
    _shape_is(k, (B, Lk, H, D), "k")
    _shape_is(v, k.shape, "v")
    _on_cuda(("q", q), ("k", k), ("v", v), ("o", o))
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(D)
    if pair is None:
        pair = block_causal_default_pair(B, Lq, Lk, H, chunk_tokens,
                                         q_offset)
    n_split = 1
    if split == "auto":
        n_split = block_causal_splits(B, Lq, Lk, H, chunk_tokens, q_offset,
                                      pair=pair)
    elif split is not None:
        n_split = int(split)
    if n_split > 1:
        need = block_causal_workspace_bytes(B, Lq, H, n_split)
        if workspace is None:
            import torch
            workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
        if not workspace.is_contiguous() or \
                workspace.numel() * workspace.element_size() < need:
            raise ValueError("workspace must be a contiguous tensor of at "
                             "least %d bytes" % need)
        _on_cuda(("q", q), ("workspace", workspace))
        name = "wan_block_causal_attn_pair_split" if pair else \
            "wan_block_causal_attn_split"
        _check(getattr(lib(), name)(
            _ptr(q), _ptr(k), _ptr(v), _ptr(o), B, Lq, Lk, H, D,
            int(chunk_tokens), int(q_offset), softmax_scale, n_split,
            _ptr(workspace), workspace.numel() * workspace.element_size(),
            _stream(stream)), name)
        return
    fn = lib().wan_block_causal_attn_pair if pair else \
        lib().wan_block_causal_attn
    _check(fn(_ptr(q), _ptr(k), _ptr(v), _ptr(o), B, Lq, Lk, H, D,
              int(chunk_tokens), int(q_offset), softmax_scale,
              _stream(stream)), "wan_block_causal_attn")


def block_causal_default_pair(B, Lq, Lk, heads, chunk_tokens, q_offset=0):
    """The kernel block_causal_attn runs by default: the CTA-pair kernel
    where the two-tile kernel would cut its equal work items into key
    ranges (wan_block_causal_attn_splits > 1, e.g. a KV-cache step), the
    two-tile kernel otherwise.  Measured at 480p-165f (65,520 tokens, 40
    heads, 4,680-token chunks), interleaved timings on four boxes: the
    KV-cache step of the last chunk ran -2 to +8 % (mean +4 %) on the pair
    kernel against the two-tile kernel with its key ranges; the full
    sequence -5 to +5 % (mean -1 %)."""
    return block_causal_splits(B, Lq, Lk, heads, chunk_tokens, q_offset) > 1


def block_causal_workspace_bytes(B, Lq, heads, n_split):
    """Workspace bytes of the split block-causal call."""
    return lib().wan_block_causal_attn_workspace_bytes(B, Lq, heads, n_split)


def block_causal_splits(B, Lq, Lk, heads, chunk_tokens, q_offset=0,
                        pair=False):
    """Key-range count for the split block-causal call on the two-tile
    kernel (wan_block_causal_attn_splits) or, with pair=True, on the
    CTA-pair kernel (wan_block_causal_attn_pair_splits)."""
    name = "wan_block_causal_attn_pair_splits" if pair else \
        "wan_block_causal_attn_splits"
    n = getattr(lib(), name)(B, Lq, Lk, heads, int(chunk_tokens),
                             int(q_offset))
    if n < 1:
        _check(n, name)
    return n


def _f32(t, name):
    import torch
    if t.dtype != torch.float32 or not t.is_contiguous():
        raise ValueError("%s must be a contiguous fp32 tensor" % name)


def adaln_modulate(x, shift, scale, out, eps=1e-6, stream=None):
    """out = LayerNorm(x) * (1 + scale[b]) + shift[b]; x fp32 [B, L, D]."""
    import torch
    _f32(x, "x")
    if x.dim() != 3:
        raise ValueError("x must be [B, L, D]")
    B, L, D = x.shape
    _f32_n(shift, B * D, "shift")
    _f32_n(scale, B * D, "scale")
    if out.dtype != torch.bfloat16 or not out.is_contiguous() \
            or out.numel() != B * L * D:
        raise ValueError("out must be a contiguous bf16 tensor of "
                         "B * L * D elements")
    _on_cuda(("x", x), ("shift", shift), ("scale", scale), ("out", out))
    _check(lib().wan_adaln_modulate(_ptr(x), _ptr(shift), _ptr(scale),
                                    _ptr(out), B, L, D, eps,
                                    _stream(stream)), "wan_adaln_modulate")


def qk_norm_rope(q, k, wq, wk, g, table, eps=1e-6, stream=None):
    """In place: t = rope3d(RMSNorm_{heads*128}(t) * w) for t in (q, k)."""
    t = q if q is not None else k
    if t is None:
        raise ValueError("q and k are both None")
    for name, x in (("q", q), ("k", k)):
        if x is not None:
            _bf16_bl(x, name)
            _shape_is(x, t.shape, name)
    if t.shape[1] != _grid_tokens(g):
        raise ValueError("q/k hold %d tokens, grid %r has %d"
                         % (t.shape[1], g, _grid_tokens(g)))
    if table is None:
        raise ValueError("qk_norm_rope needs a table")
    _check_table(table, g, t.shape[3])
    nw = t.shape[2] * t.shape[3]
    for name, x, w in (("wq", q, wq), ("wk", k, wk)):
        if x is not None:
            if w is None:
                raise ValueError("%s is needed with its tensor" % name)
            _f32_n(w, nw, name)
    _on_cuda(("q", q), ("k", k), ("wq", wq), ("wk", wk),
                 ("table", table))
    _check(lib().wan_qk_norm_rope(_ptr(q), _ptr(k), _ptr(wq), _ptr(wk),
                                  t.shape[0], g, t.shape[2], t.shape[3],
                                  _ptr(table), eps, _stream(stream)),
           "wan_qk_norm_rope")


def gated_residual(x, y, gate, stream=None):
    """x += y * gate[b]; x fp32 [B, L, D], y bf16 [B, L, D], gate [B, D]."""
    import torch
    _f32(x, "x")
    if x.dim() != 3:
        raise ValueError("x must be [B, L, D]")
    B, L, D = x.shape
    _f32_n(gate, B * D, "gate")
    if y.dtype != torch.bfloat16 or not y.is_contiguous() \
            or y.numel() != x.numel():
        raise ValueError("y must be a contiguous bf16 tensor of x's size")
    _on_cuda(("x", x), ("y", y), ("gate", gate))
    _check(lib().wan_gated_residual(_ptr(x), _ptr(y), _ptr(gate), B, L, D,
                                    _stream(stream)), "wan_gated_residual")


def fm_step(x, v_cond, v_uncond, guide, sigma, sigma_next, stream=None):
    """x += (sigma_next - sigma) * (v_uncond + guide (v_cond - v_uncond))."""
    _f32(x, "x")
    _f32_n(v_cond, x.numel(), "v_cond")
    if v_uncond is not None:
        _f32_n(v_uncond, x.numel(), "v_uncond")
    _on_cuda(("x", x), ("v_cond", v_cond), ("v_uncond", v_uncond))
    _check(lib().wan_fm_step(_ptr(x), _ptr(v_cond), _ptr(v_uncond), guide,
                             x.numel(), sigma, sigma_next, _stream(stream)),
           "wan_fm_step")


def _sigma_array(sigmas):
    arr = (ctypes.c_double * len(sigmas))(*[float(x) for x in sigmas])
    return arr, len(sigmas) - 1


def unipc_coeffs(sigmas, i):
    """Folded UniPC coefficients of stop i (dict of wan_unipc_coef_t)."""
    arr, n = _sigma_array(sigmas)
    out = UniPCCoef()
    _check(lib().wan_unipc_coeffs(arr, n, int(i), ctypes.byref(out)),
           "wan_unipc_coeffs")
    return out.as_dict()


def unipc_step(x, x_corr, m_prev1, m_prev2, m_out, v_cond, v_uncond, guide,
               sigmas, i, stream=None):
    """One fused UniPC stop (see include/wan.h): x and x_corr in place,
    m_i into m_out (which may be the m_prev2 buffer)."""
    import torch
    for name, t in (("x", x), ("x_corr", x_corr), ("m_out", m_out),
                    ("v_cond", v_cond), ("v_uncond", v_uncond),
                    ("m_prev1", m_prev1), ("m_prev2", m_prev2)):
        if t is not None and (t.dtype != torch.float32
                              or not t.is_contiguous()
                              or t.numel() != x.numel()):
            raise ValueError("%s must be a contiguous fp32 tensor of x's "
                             "size" % name)
    _on_cuda(("x", x), ("x_corr", x_corr), ("m_out", m_out),
                 ("v_cond", v_cond), ("v_uncond", v_uncond),
                 ("m_prev1", m_prev1), ("m_prev2", m_prev2))
    arr, n = _sigma_array(sigmas)
    _check(lib().wan_unipc_step(_ptr(x), _ptr(x_corr), _ptr(m_prev1),
                                _ptr(m_prev2), _ptr(m_out), _ptr(v_cond),
                                _ptr(v_uncond), guide, x.numel(), arr, n,
                                int(i), _stream(stream)), "wan_unipc_step")


def transpose_blocks(inp, out, a, b, row_bytes, stream=None):
    """out[j][i][:] = inp[i][j][:] (i < a, j < b, rows of row_bytes)."""
    for name, t in (("inp", inp), ("out", out)):
        if not t.is_contiguous():
            raise ValueError("%s must be a contiguous tensor" % name)
        if t.numel() * t.element_size() < a * b * row_bytes:
            raise ValueError("%s is smaller than a * b * row_bytes" % name)
    _on_cuda(("inp", inp), ("out", out))
    _check(lib().wan_transpose_blocks(_ptr(inp), _ptr(out), int(a), int(b),
                                      int(row_bytes), _stream(stream)),
           "wan_transpose_blocks")


def attn_pair_resident_clusters():
    """CTA pairs of the pair kernels resident at once on this device."""
    n = lib().wan_attn_pair_resident_clusters()
    if n < 0:
        _check(n, "wan_attn_pair_resident_clusters")
    return n


def wait_selftest(arrive, stream=None):
    """Launch the bounded-wait self-test kernel (see include/wan.h)."""
    _check(lib().wan_wait_selftest(int(arrive), _stream(stream)),
           "wan_wait_selftest")


def device_status(clear=True):
    """0, or WAN_ETIMEOUT if a bounded in-kernel wait ran out."""
    st = lib().wan_device_status(1 if clear else 0)
    if st not in (0, WAN_ETIMEOUT):
        _check(st, "wan_device_status")
    return st
