"""Latent shape and token-grid arithmetic (oracle; test infrastructure only).

Wan2.2 source reading, ch. 2 "VAE: the video is first made 46x smaller":
the configuration gives ``vae_stride = (4, 8, 8)`` (time x4, height x8,
width x8) and ``patch_size = (1, 2, 2)``; the latent shape is
``(z_dim, (F - 1) // 4 + 1, height // 8, width // 8)`` with ``z_dim = 16``,
and the frame count must be of the form 4n+1 (section "The origin of 4n+1").

Wan2.2 source reading, ch. 4 "DiT: attention over 75600 tokens", section
"From latent to token": the patch embedding is a Conv3d with kernel = stride
= (1, 2, 2), so each 2x2 block of latent positions becomes one token and
the token count is ``latent_frames * (lat_h / 2) * (lat_w / 2)``.

Token order (a reading: the pages only say the tokens are laid out as a 1-D
sequence, ch. 4 section "3D RoPE"): frame-major, then height, then width,
``n = (f * H + h) * W + w``, positions starting at 0.
"""

Z_DIM = 16
VAE_STRIDE = (4, 8, 8)
PATCH = (1, 2, 2)


def latent_shape(frames, height, width):
    """Latent tensor shape (z_dim, F_lat, h_lat, w_lat) for a pixel video.

    Follows the ``target_shape`` expression of ch. 2 (section "VAE"): the
    first frame is encoded alone and every further 4 frames become one
    latent frame.  Raises ValueError for a frame count that is not 4n+1 or
    a pixel size that is not a multiple of the spatial stride, the cases the
    page says make the tensor shapes not fit.
    """
    if frames < 1 or (frames - 1) % VAE_STRIDE[0] != 0:
        raise ValueError("frame count must be 4n+1")
    if height % VAE_STRIDE[1] or width % VAE_STRIDE[2]:
        raise ValueError("pixel size must be a multiple of 8")
    return (Z_DIM, (frames - 1) // VAE_STRIDE[0] + 1,
            height // VAE_STRIDE[1], width // VAE_STRIDE[2])


def token_grid(frames, height, width):
    """Token grid (F, H, W) after the (1, 2, 2) patchify of ch. 4."""
    _, f, h, w = latent_shape(frames, height, width)
    if f % PATCH[0] or h % PATCH[1] or w % PATCH[2]:
        raise ValueError("latent size must be a multiple of the patch size")
    return (f // PATCH[0], h // PATCH[1], w // PATCH[2])


def token_count(grid):
    """Sequence length L = F * H * W of a token grid."""
    f, h, w = grid
    return f * h * w


def token_coords(n, grid):
    """(f, h, w) coordinates of flat token index n (frame-major order)."""
    _, h_, w_ = grid
    return (n // (h_ * w_), (n // w_) % h_, n % w_)


def attention_flops(batch, heads, lq, lk, head_dim):
    """Attention FLOPs per call as the pages count them.

    Wan2.2 source reading, ch. 8 "What is 75600^2": two matrix products
    (QK^T and AV), each multiply and add counted as one FLOP, giving
    ``2 * 2 * L^2 * dim`` per layer with ``dim = heads * head_dim``.
    """
    return 4 * batch * heads * lq * lk * head_dim
