"""fp64 CPU oracle of the Flash DiT block with spatial token compression, the
backbone stack, and the few-step flow-matching Euler loop.

Test infrastructure only (see the package docstring).  Everything here is
written from the pages' prose; no listing exists on them.

Conventions shared by every function:

* Activations are token-major ``[rows, hidden]``.  The row order of a packed
  sequence is ``[target video (t, h, w) row-major | control video | text |
  audio]``; joint attention has no mask, so the order is a layout choice.
* Linear weights use the ``[out_features, in_features]`` layout: ``y = x @ W.T + b``.
* Modality codes: 0 text, 1 video (target), 2 audio, 3 video control.
"""

from __future__ import annotations

import math

import numpy as np

F64 = np.float64

MOD_TEXT, MOD_VIDEO, MOD_AUDIO, MOD_CONTROL = 0, 1, 2, 3

# [tokendh, training section, dual-clock paragraph]: for four evaluations the
# clean times are about 0, 0.027, 0.0769, 0.2 (video) and 0, 0.1, 0.25, 0.5
# (audio).  The Flash model runs three evaluations that start from the largest
# listed time and land on 0.
FLASH_VIDEO_CLOCK = (0.2, 0.0769, 0.027, 0.0)
FLASH_AUDIO_CLOCK = (0.5, 0.25, 0.1, 0.0)
# Reading (4-eval standard model): prepend t=1 (pure noise) so that the four
# evaluations land on the four listed times.
STANDARD_VIDEO_CLOCK = (1.0, 0.2, 0.0769, 0.027, 0.0)
STANDARD_AUDIO_CLOCK = (1.0, 0.5, 0.25, 0.1, 0.0)

# Flash layer schedule [tokendh, training section, Flash paragraph; PaperDaily
# section 二]: the first 2 layers see the full sequence, the middle 26 layers
# run on compressed video tokens, the last 14 layers are full again.
FLASH_SCHEDULE = (2, 26, 14)


def flash_layer_compress(n_full_head=2, n_comp=26, n_full_tail=14):
    """Per-layer compression flags of the Flash 42-layer schedule."""
    return [0] * n_full_head + [1] * n_comp + [0] * n_full_tail


# ---------------------------------------------------------------------------
# Keep-index map  [tokendh, training section, Flash paragraph: 2x spatial
# down-sampling that keeps the border rows/columns; PaperDaily section 二:
# every other video token along each spatial axis of every frame, edge rows
# and columns kept, no temporal drop].
# ---------------------------------------------------------------------------

def axis_keep(n: int) -> list[int]:
    """Kept indices along one spatial axis of length n: 0, 2, 4, ... and n-1."""
    if n <= 0:
        return []
    kept = list(range(0, n, 2))
    if kept[-1] != n - 1:
        kept.append(n - 1)
    return kept


def axis_nearest(n: int) -> list[int]:
    """For each index of an axis, the nearest kept index on that axis.

    Reading: a dropped index i is odd and both i-1 and i+1 are kept, so the
    pages' "nearest" is a tie; the lower index wins.
    """
    kept = axis_keep(n)
    out = []
    for i in range(n):
        best_d, best_k = None, None
        for k in kept:
            d = abs(i - k)
            if best_d is None or d < best_d or (d == best_d and k < best_k):
                best_d, best_k = d, k
        out.append(best_k)
    return out


def keep_map(T: int, H: int, W: int):
    """Keep-index map of a T x H x W video grid (row id = t*H*W + h*W + w).

    Returns ``(keep_idx, near_idx)``:
    * ``keep_idx[c]`` -- full-grid row id of the c-th kept token, in
      (t, kept h, kept w) row-major order;
    * ``near_idx[p]`` -- compact id c of the kept token nearest to row p in
      the same frame ([tokendh] "同一帧里最近的那个被保留token").  The kept set
      of a frame is a product of per-axis sets, so the per-axis nearest pair
      is also the Euclidean nearest; ties go to the lower h, then lower w.
    """
    rows, cols = axis_keep(H), axis_keep(W)
    keep_idx = [t * H * W + h * W + w for t in range(T) for h in rows for w in cols]
    compact = {p: c for c, p in enumerate(keep_idx)}
    nh, nw = axis_nearest(H), axis_nearest(W)
    near_idx = [compact[t * H * W + nh[h] * W + nw[w]]
                for t in range(T) for h in range(H) for w in range(W)]
    return np.asarray(keep_idx, dtype=np.int32), np.asarray(near_idx, dtype=np.int32)


# ---------------------------------------------------------------------------
# Elementwise pieces of the block.
# ---------------------------------------------------------------------------

def rms_norm(x, g, eps=1e-6):
    """RMSNorm over the last axis: x / sqrt(mean(x^2) + eps) * g."""
    x = np.asarray(x, dtype=F64)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * np.asarray(g, dtype=F64)


def gelu_tanh(x):
    """GELU, tanh form: 0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3)))."""
    x = np.asarray(x, dtype=F64)
    return 0.5 * x * (1.0 + np.tanh(math.sqrt(2.0 / math.pi) * (x + 0.044715 * x ** 3)))


def silu(x):
    """SiLU, x * sigmoid(x) (the timestep MLP's activation, reading R7)."""
    x = np.asarray(x, dtype=F64)
    return x / (1.0 + np.exp(-x))


def rope_angles(pos, split=(32, 48, 48), theta=10000.0):
    """Rotation angle of every (2j, 2j+1) pair of a head for each token.

    [tokendh, backbone section]: every row carries a 3D rotary position.
    Reading: the head dimension is cut into consecutive chunks of 32 (t),
    48 (h) and 48 (w) channels; inside the chunk of axis a (width d_a) pair j
    turns by pos_a * theta^(-2j/d_a), theta = 10000.
    Returns float64 ``[n, sum(split)//2]``.
    """
    pos = np.asarray(pos, dtype=F64)
    parts = []
    for a, da in enumerate(split):
        j = np.arange(da // 2, dtype=F64)
        inv_freq = theta ** (-2.0 * j / da)
        parts.append(pos[:, a:a + 1] * inv_freq[None, :])
    return np.concatenate(parts, axis=1)


def apply_rope(x, pos, split=(32, 48, 48), theta=10000.0):
    """Rotate interleaved pairs (x_2j, x_2j+1) of x ``[n, heads, d]``."""
    x = np.asarray(x, dtype=F64)
    ang = rope_angles(pos, split, theta)[:, None, :]
    c, s = np.cos(ang), np.sin(ang)
    xe, xo = x[..., 0::2], x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = xe * c - xo * s
    out[..., 1::2] = xe * s + xo * c
    return out


def attention(q, k, v):
    """Joint full attention, per head: softmax(q k^T / sqrt(d)) v.

    [tokendh, backbone section; PaperDaily section 一]: text, video and audio
    tokens go through one denoiser as one sequence.  Reading: no mask, plain
    scaled softmax, no QK norm.  q, k, v are ``[n, heads, d]``; returns
    ``[n, heads * d]``.
    """
    q, k, v = (np.asarray(a, dtype=F64) for a in (q, k, v))
    n, nh, d = q.shape
    out = np.empty((n, nh, d), dtype=F64)
    scale = 1.0 / math.sqrt(d)
    for h in range(nh):
        s = (q[:, h, :] @ k[:, h, :].T) * scale
        s = s - s.max(axis=1, keepdims=True)
        p = np.exp(s)
        p /= p.sum(axis=1, keepdims=True)
        out[:, h, :] = p @ v[:, h, :]
    return out.reshape(n, nh * d)


def linear(x, w, b=None):
    """x W^T (+ b) in float64; W in Linear layout [out, in]."""
    y = np.asarray(x, dtype=F64) @ np.asarray(w, dtype=F64).T
    if b is not None:
        y = y + np.asarray(b, dtype=F64)
    return y


# ---------------------------------------------------------------------------
# One DiT block (uncompressed).
# ---------------------------------------------------------------------------

def dit_block(x, w, pos, heads, head_dim, rope_split=(32, 48, 48), eps=1e-6,
              theta=10000.0):
    """One pre-norm DiT block over all rows of x ``[n, H]``.

    h = x + Wo . attn(rope(q), rope(k), v) + bo, with [q k v] = Wqkv . rmsnorm(x) + b;
    y = h + W2 . gelu_tanh(W1 . rmsnorm(h) + b1) + b2.
    [tokendh, backbone section] gives hidden 5376 and 56 heads of 128: the
    heads span 56 x 128 = 7168 channels, so q, k, v are each heads*head_dim
    wide (Wqkv is [3*heads*head_dim, H]) and Wo maps them back to H.
    Reading: pre-RMSNorm with a learned gain, biases on every projection,
    RoPE on q and k at each token's own (t, h, w) position.
    """
    x = np.asarray(x, dtype=F64)
    n = x.shape[0]
    A = heads * head_dim          # attention width; 56 x 128 = 7168 next to hidden 5376
    xn = rms_norm(x, w["g_attn"], eps)
    qkv = linear(xn, w["w_qkv"], w["b_qkv"])
    q = qkv[:, 0 * A:1 * A].reshape(n, heads, head_dim)
    k = qkv[:, 1 * A:2 * A].reshape(n, heads, head_dim)
    v = qkv[:, 2 * A:3 * A].reshape(n, heads, head_dim)
    q = apply_rope(q, pos, rope_split, theta)
    k = apply_rope(k, pos, rope_split, theta)
    a = attention(q, k, v)
    h = x + linear(a, w["w_o"], w["b_o"])
    hn = rms_norm(h, w["g_ffn"], eps)
    u = gelu_tanh(linear(hn, w["w_1"], w["b_1"]))
    return h + linear(u, w["w_2"], w["b_2"])


def dit_block_rows(x, w, pos, heads, head_dim, rows, rope_split=(32, 48, 48), eps=1e-6,
                   theta=10000.0):
    """``dit_block(x, ...)[rows]`` computed for the requested rows only.

    Keys and values are formed for every row (each output row attends to all
    of them); queries, the output projection and the FFN only for ``rows``.
    Same definition as ``dit_block``, restricted -- used to check outputs of
    full-size blocks one row at a time."""
    x = np.asarray(x, dtype=F64)
    n = x.shape[0]
    rows = np.asarray(rows, dtype=np.int64)
    A = heads * head_dim
    xn = rms_norm(x, w["g_attn"], eps)
    w_qkv = np.asarray(w["w_qkv"], dtype=F64)
    b_qkv = np.asarray(w["b_qkv"], dtype=F64)
    q = linear(xn[rows], w_qkv[:A], b_qkv[:A]).reshape(len(rows), heads, head_dim)
    k = linear(xn, w_qkv[A:2 * A], b_qkv[A:2 * A]).reshape(n, heads, head_dim)
    v = linear(xn, w_qkv[2 * A:], b_qkv[2 * A:]).reshape(n, heads, head_dim)
    q = apply_rope(q, np.asarray(pos)[rows], rope_split, theta)
    k = apply_rope(k, pos, rope_split, theta)
    scale = 1.0 / math.sqrt(head_dim)
    a = np.empty((len(rows), heads, head_dim), dtype=F64)
    for h in range(heads):
        s = (q[:, h, :] @ k[:, h, :].T) * scale
        s = s - s.max(axis=1, keepdims=True)
        p = np.exp(s)
        p /= p.sum(axis=1, keepdims=True)
        a[:, h, :] = p @ v[:, h, :]
    hrow = x[rows] + linear(a.reshape(len(rows), A), w["w_o"], w["b_o"])
    u = gelu_tanh(linear(rms_norm(hrow, w["g_ffn"], eps), w["w_1"], w["b_1"]))
    return hrow + linear(u, w["w_2"], w["b_2"])


# ---------------------------------------------------------------------------
# Compressed block: gather kept rows, run the block, broadcast back.
# ---------------------------------------------------------------------------

def gather_rows(x, keep_idx, n_video):
    """Compressed sequence: kept video rows (keep_idx order), then every
    non-grid row (control, text, audio) unchanged [PaperDaily section 二:
    text and audio tokens are never compressed]."""
    x = np.asarray(x)
    sel = np.concatenate([np.asarray(keep_idx, dtype=np.int64),
                          np.arange(n_video, x.shape[0], dtype=np.int64)])
    return x[sel]


def broadcast_residual(x, y_c, keep_idx, near_idx, n_video):
    """Scatter the compressed block's result back to full resolution.

    [PaperDaily section 二]: compressed layers compute the feature update only
    at kept positions; a missing position takes the update of the nearest kept
    position of its frame, and the update is added back to the full-resolution
    features.  [tokendh, training section]: a residual connection carries it.

    Reading: the update of kept token c is d_c = y_c[c] - x[keep_idx[c]].
    A kept row p takes y_c directly (so a keep-all map reproduces the plain
    block exactly); a dropped row p takes x[p] + d_{near_idx[p]}.  Non-grid
    rows take their y_c rows.
    """
    x = np.asarray(x, dtype=F64)
    y_c = np.asarray(y_c, dtype=F64)
    keep_idx = np.asarray(keep_idx, dtype=np.int64)
    near_idx = np.asarray(near_idx, dtype=np.int64)
    n_keep = keep_idx.shape[0]
    out = np.empty_like(x)
    src = keep_idx[near_idx]                       # full-grid row of the nearest kept token
    is_kept = src == np.arange(n_video)
    delta = y_c[near_idx] - x[src]
    out[:n_video] = np.where(is_kept[:, None], y_c[near_idx], x[:n_video] + delta)
    out[n_video:] = y_c[n_keep:]
    return out


def dit_block_compressed(x, w, pos, heads, head_dim, keep_idx, near_idx, n_video,
                         rope_split=(32, 48, 48), eps=1e-6, theta=10000.0, block_fn=None):
    """The Flash compressed block, per-block form: gather, block, broadcast.

    RoPE positions of kept tokens are their original (t, h, w) coordinates
    (Reading: the pages do not renumber them).  ``block_fn`` replaces
    ``dit_block`` (e.g. the low-bit block of ``oracle.fp8``)."""
    block_fn = block_fn or dit_block
    x_c = gather_rows(x, keep_idx, n_video)
    pos_c = gather_rows(pos, keep_idx, n_video)
    y_c = block_fn(x_c, w, pos_c, heads, head_dim, rope_split, eps, theta)
    return broadcast_residual(x, y_c, keep_idx, near_idx, n_video)


def dit_block_compressed_rows(x, w, pos, heads, head_dim, keep_idx, near_idx, n_video, rows,
                              rope_split=(32, 48, 48), eps=1e-6, theta=10000.0, rows_fn=None):
    """``dit_block_compressed(...)[rows]`` for the requested rows only: the
    compressed block is evaluated (via ``dit_block_rows``, or ``rows_fn`` with
    the same signature, e.g. the low-bit block's row restriction) just for the
    compressed rows those outputs read, then the same broadcast rule applies."""
    rows_fn = rows_fn or dit_block_rows
    x = np.asarray(x, dtype=F64)
    rows = np.asarray(rows, dtype=np.int64)
    keep_idx = np.asarray(keep_idx, dtype=np.int64)
    near_idx = np.asarray(near_idx, dtype=np.int64)
    n_keep = keep_idx.shape[0]
    need = np.unique(np.where(rows < n_video, near_idx[np.minimum(rows, n_video - 1)],
                              n_keep + rows - n_video))
    x_c = gather_rows(x, keep_idx, n_video)
    pos_c = gather_rows(pos, keep_idx, n_video)
    y_c = np.zeros_like(x_c)
    y_c[need] = rows_fn(x_c, w, pos_c, heads, head_dim, need, rope_split, eps, theta)
    return broadcast_residual(x, y_c, keep_idx, near_idx, n_video)[rows]


# ---------------------------------------------------------------------------
# Embedding and output heads.
# ---------------------------------------------------------------------------

def timestep_features(t, dim=256, max_period=10000.0):
    """Sinusoidal features of 1000*t: [cos(args), sin(args)],
    args_j = 1000 t * max_period^(-j/(dim/2)).

    Reading: the pages say each row carries a noise time ([tokendh, backbone
    section]); how it enters the network is not stated.  A standard DiT
    timestep embedding is used."""
    half = dim // 2
    freqs = np.exp(-math.log(max_period) * np.arange(half, dtype=F64) / half)
    args = 1000.0 * float(t) * freqs
    return np.concatenate([np.cos(args), np.sin(args)])


def time_embedding(t, io):
    """Linear(256, H) -> SiLU -> Linear(H, H) of the sinusoidal features."""
    f = timestep_features(t, np.asarray(io["w_t1"]).shape[1])
    h = silu(linear(f[None, :], io["w_t1"], io["b_t1"]))
    return linear(h, io["w_t2"], io["b_t2"])[0]


def embed(io, modality, time_id, time_table, video_lat, text_emb, audio_lat):
    """Input embedding of a packed sequence.

    Rows with modality video or control read ``video_lat`` in order, text rows
    read ``text_emb``, audio rows read ``audio_lat``.  Each row gets its
    modality's input projection, a learned modality embedding and the time
    embedding of its own noise time ``time_table[time_id[row]]``
    (Reading: additive conditioning, no adaptive norm)."""
    modality = np.asarray(modality)
    time_id = np.asarray(time_id)
    n = modality.shape[0]
    H = np.asarray(io["mod_emb"]).shape[1]
    x = np.zeros((n, H), dtype=F64)
    vid = np.nonzero((modality == MOD_VIDEO) | (modality == MOD_CONTROL))[0]
    txt = np.nonzero(modality == MOD_TEXT)[0]
    aud = np.nonzero(modality == MOD_AUDIO)[0]
    if vid.size:
        x[vid] = linear(video_lat, io["w_vin"], io["b_vin"])
    if txt.size:
        x[txt] = linear(text_emb, io["w_tin"], io["b_tin"])
    if aud.size:
        x[aud] = linear(audio_lat, io["w_ain"], io["b_ain"])
    x += np.asarray(io["mod_emb"], dtype=F64)[modality]
    temb = np.stack([time_embedding(t, io) for t in time_table])
    x += temb[time_id]
    return x


def output_heads(x, io, modality, eps=1e-6):
    """Final RMSNorm, then video rows -> video velocity, audio rows -> audio
    velocity [tokendh, backbone section: one forward predicts both]."""
    modality = np.asarray(modality)
    xf = rms_norm(x, io["g_out"], eps)
    vid = np.nonzero((modality == MOD_VIDEO) | (modality == MOD_CONTROL))[0]
    aud = np.nonzero(modality == MOD_AUDIO)[0]
    v_video = linear(xf[vid], io["w_vout"], io["b_vout"])
    v_audio = linear(xf[aud], io["w_aout"], io["b_aout"])
    return v_video, v_audio


# ---------------------------------------------------------------------------
# Backbone stack.
# ---------------------------------------------------------------------------

def dit_stack(layers, layer_compress, io, tok, time_table, video_lat, text_emb,
              audio_lat, heads, head_dim, rope_split=(32, 48, 48), eps=1e-6,
              theta=10000.0, segment=False, block_fn=None):
    """One backbone evaluation: embed, layers, heads -> (v_video, v_audio).

    ``tok`` holds the packed tags: ``modality``, ``time_id``, ``pos`` [n,3],
    ``n_video`` (rows of the target grid) and, when any layer compresses,
    ``keep_idx`` / ``near_idx`` of that grid.

    ``segment=False`` applies the compressed block layer by layer (gather and
    broadcast around every compressed layer).  ``segment=True`` gathers once
    before a run of compressed layers and broadcasts once after it; in exact
    arithmetic the two agree because kept rows only ever read kept rows and
    the dropped-row updates telescope.

    ``block_fn`` replaces ``dit_block`` for every layer (e.g. the low-bit block
    ``oracle.fp8.dit_block_fp8``); the default is the full-precision block.
    """
    block_fn = block_fn or dit_block
    x = embed(io, tok["modality"], tok["time_id"], time_table, video_lat,
              text_emb, audio_lat)
    pos = tok["pos"]
    L = len(layers)
    l = 0
    while l < L:
        if not layer_compress[l]:
            x = block_fn(x, layers[l], pos, heads, head_dim, rope_split, eps, theta)
            l += 1
        elif not segment:
            x = dit_block_compressed(x, layers[l], pos, heads, head_dim,
                                     tok["keep_idx"], tok["near_idx"], tok["n_video"],
                                     rope_split, eps, theta, block_fn)
            l += 1
        else:
            x_c = gather_rows(x, tok["keep_idx"], tok["n_video"])
            pos_c = gather_rows(pos, tok["keep_idx"], tok["n_video"])
            while l < L and layer_compress[l]:
                x_c = block_fn(x_c, layers[l], pos_c, heads, head_dim, rope_split,
                                eps, theta)
                l += 1
            x = broadcast_residual(x, x_c, tok["keep_idx"], tok["near_idx"],
                                   tok["n_video"])
    return output_heads(x, io, tok["modality"], eps)


# ---------------------------------------------------------------------------
# Flow matching and the Euler loop.
# ---------------------------------------------------------------------------

def flow_interpolate(x0, eps_noise, t):
    """[tokendh, training section]: mix clean data and noise by time:
    x_t = (1 - t) x0 + t eps."""
    return (1.0 - t) * np.asarray(x0, dtype=F64) + t * np.asarray(eps_noise, dtype=F64)


def flow_velocity(x0, eps_noise):
    """Velocity the network learns: v = eps - x0 (= d x_t / d t)."""
    return np.asarray(eps_noise, dtype=F64) - np.asarray(x0, dtype=F64)


def euler_step(x, v, row_modality, out_mask, t_cur, t_next):
    """One Euler step on each row with its own modality's clock:
    x <- x + (t_next[m] - t_cur[m]) v for rows with out_mask set; other rows
    (clean conditions) are left as they are [PaperDaily section 一: video and
    audio share the forward but keep separate noise clocks]."""
    x = np.array(x, dtype=F64, copy=True)
    v = np.asarray(v, dtype=F64)
    row_modality = np.asarray(row_modality)
    out_mask = np.asarray(out_mask).astype(bool)
    dt = np.asarray(t_next, dtype=F64) - np.asarray(t_cur, dtype=F64)
    step = dt[row_modality][:, None]
    x[out_mask] = x[out_mask] + step[out_mask] * v[out_mask]
    return x


def flow_sample(layers, layer_compress, io, tok, video_clock, audio_clock,
                video_lat, text_emb, audio_lat, heads, head_dim,
                rope_split=(32, 48, 48), eps=1e-6, theta=10000.0, segment=False, block_fn=None):
    """The few-step sampler: len(clock)-1 evaluations; evaluation e runs the
    stack with time table [0, t_v[e], t_a[e]] and moves target video rows from
    t_v[e] to t_v[e+1] and audio rows from t_a[e] to t_a[e+1].

    ``tok`` must carry ``video_modality``/``video_out`` (per video-latent row:
    modality code and whether it is updated) and ``audio_out``.
    Returns the final (video_lat, audio_lat)."""
    vl = np.asarray(video_lat, dtype=F64)
    al = np.asarray(audio_lat, dtype=F64)
    E = len(video_clock) - 1
    for e in range(E):
        table = [0.0, video_clock[e], audio_clock[e]]
        v_vid, v_aud = dit_stack(layers, layer_compress, io, tok, table, vl, text_emb,
                                 al, heads, head_dim, rope_split, eps, theta, segment, block_fn)
        t_cur = [0.0, video_clock[e], audio_clock[e], 0.0]
        t_nxt = [0.0, video_clock[e + 1], audio_clock[e + 1], 0.0]
        vl = euler_step(vl, v_vid, tok["video_modality"], tok["video_out"], t_cur, t_nxt)
        al = euler_step(al, v_aud, np.full(al.shape[0], MOD_AUDIO), tok["audio_out"],
                        t_cur, t_nxt)
    return vl, al


def rel_l2(a, b):
    """Relative L2 error ||a - b|| / ||b|| in float64."""
    a = np.asarray(a, dtype=F64)
    b = np.asarray(b, dtype=F64)
    den = np.linalg.norm(b.ravel())
    return float(np.linalg.norm((a - b).ravel()) / (den if den > 0 else 1.0))


__all__ = [name for name in dir() if not name.startswith("_") and name not in
           ("annotations", "math", "np")]
