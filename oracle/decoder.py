"""fp64 CPU oracle of the lightweight video decoder's forward pass (test
infrastructure only; see the package docstring).

Sources:

* [tokendh] section "解码器瓶颈：被忽视的那一半时间": once few-step
  distillation has shrunk the denoiser, the decoder that turns latents back
  into frames becomes the slow part; a student decoder distilled from a
  36-layer teacher has 26 layers, keeps hidden width 2048 and a four-fold
  feed-forward expansion, and cut decoding of a 22-frame 540p clip on one
  H100 from 469 to 340 ms.
* [ananclaw explainer] section 3.4 "推理加速": the Flash model runs with a
  lightweight VAE decoder.

Readings where the pages leave a step open:

* Architecture.  The pages give depth, width and FFN ratio only; "hidden
  width" and "feed-forward expansion" are transformer terms, so the decoder
  is a transformer over the latent tokens: one token per latent cell, a
  linear latent projection (c_lat -> hidden, with bias), blocks of the same
  pre-norm form as the backbone's (RMSNorm, QKV with 3D RoPE at the cell's
  (t, h, w), full bidirectional attention over the clip with heads of 128
  channels, GELU-tanh FFN), a final RMSNorm and a linear pixel head per
  token.  No noise time and no modality embedding enter: a VAE decoder sees
  clean latents only.
* Pixel patch.  Each latent cell covers ps x ps pixels (16: the 34 x 60 grid
  of the 540p workload is 544 x 960 pixels) and pt frames (4), causal in
  time: latent frame 0 yields one frame (its last temporal slice) and
  latent frame t >= 1 yields frames pt*t - pt + 1 .. pt*t, so T latent
  frames decode to 1 + pt*(T - 1) frames (6 -> 21; the pages' 22 frames fit
  no integer stride).  The head's output columns are ordered
  (channel, dt, dy, dx) with dx fastest.
* Output layout: pixels [F, c_pix, H*ps, W*ps] (frames of channel planes).
* Colour conversion ([PaperDaily] section 二: the fully accelerated
  configuration converts colours on the GPU): the decoder's values are read
  as lying in [-1, 1] and mapped linearly onto 8-bit codes, 127.5 * (v + 1)
  taken in fp32 as a product and then a sum (each rounded), clamped to
  [0, 255] and rounded to the nearest integer, ties to even.
"""

import numpy as np

from .dit import dit_block, linear, rms_norm

F64 = np.float64


def grid_positions(T, H, W):
    """(t, h, w) of every cell of a T x H x W latent grid, row-major."""
    t, h, w = np.meshgrid(np.arange(T), np.arange(H), np.arange(W), indexing="ij")
    return np.stack([t.ravel(), h.ravel(), w.ravel()], axis=1).astype(np.int64)


def decoder_frames(T, pt):
    """Frames decoded from T latent frames, causal temporal patch pt."""
    return 1 + pt * (T - 1) if T > 0 else 0


def head_column(c, dt, dy, dx, pt, ps):
    """Column of the pixel head that holds channel c, temporal slice dt and
    pixel (dy, dx) of a cell's patch."""
    return ((c * pt + dt) * ps + dy) * ps + dx


def unpatchify(y, T, H, W, c_pix, pt, ps):
    """Place the pixel head's rows y [T*H*W, c_pix*pt*ps*ps] into frames
    [1 + pt*(T-1), c_pix, H*ps, W*ps]: cell (t, h, w), column (c, dt, dy, dx)
    lands in frame pt*t + dt - (pt - 1) (dropped when negative), channel c,
    pixel (ps*h + dy, ps*w + dx)."""
    y = np.asarray(y, dtype=F64).reshape(T, H, W, c_pix, pt, ps, ps)
    # axes: t, h, w, c, dt, dy, dx  ->  t, dt, c, h, dy, w, dx
    frames = y.transpose(0, 4, 3, 1, 5, 2, 6).reshape(T * pt, c_pix, H * ps, W * ps)
    return frames[pt - 1:]


def decoder_tokens(latents, layers, io, T, H, W, heads, head_dim, rope_split=(32, 48, 48), eps=1e-6,
                   theta=10000.0, block_fn=dit_block):
    """Hidden states after the blocks: x [T*H*W, hidden]."""
    x = linear(np.asarray(latents, dtype=F64).reshape(T * H * W, -1), io["w_in"], io["b_in"])
    pos = grid_positions(T, H, W)
    for w in layers:
        x = block_fn(x, w, pos, heads, head_dim, rope_split, eps, theta)
    return x


def pixel_head(x, io, eps=1e-6):
    """Final RMSNorm and the per-token pixel head: [rows, c_pix*pt*ps*ps]."""
    return linear(rms_norm(x, io["g_out"], eps), io["w_out"], io["b_out"])


def decoder_forward(latents, layers, io, T, H, W, heads, head_dim, c_pix, pt, ps, rope_split=(32, 48, 48),
                    eps=1e-6, theta=10000.0, block_fn=dit_block):
    """Decode latents [T*H*W, c_lat] (cells in (t, h, w) row-major order) to
    pixels [1 + pt*(T-1), c_pix, H*ps, W*ps]."""
    x = decoder_tokens(latents, layers, io, T, H, W, heads, head_dim, rope_split, eps, theta, block_fn)
    return unpatchify(pixel_head(x, io, eps), T, H, W, c_pix, pt, ps)


def to_rgb8(pixels):
    """8-bit codes of decoder values (fp32 arithmetic, see the module
    docstring): uint8 array of the same shape."""
    v = np.asarray(pixels, dtype=np.float32)
    t = (v * np.float32(127.5)).astype(np.float32)
    t = (t + np.float32(127.5)).astype(np.float32)
    t = np.clip(t, np.float32(0.0), np.float32(255.0))
    return np.rint(t).astype(np.uint8)
