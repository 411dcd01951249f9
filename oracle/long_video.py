"""fp64 CPU oracle of long-video generation by chunks with a bounded,
multi-stride history (test infrastructure only; see the package docstring).

Sources:

* [tokendh] section "长视频生成：怎么记住十分钟前发生的事": video is generated
  in fixed-length chunks; the last frame of the previous chunk is shared as a
  fixed boundary frame from which the model predicts the next latents; the
  history keeps the earliest latent frame at full spatial resolution, the two
  most recent at spatial stride 2 and at most eight earlier ones at stride 4,
  so the history never holds more tokens than about two full-resolution
  frames, however long the video gets.
* [PaperDaily] section 三 "长视频不是无限塞历史，而是保留“够用的记忆”": each
  round delivers 17 new frames; the boundary frame sits at the first latent
  position of the next chunk's target and is followed by five future latents;
  storage is bounded too: once full, the initial frame and the most recent
  frames are kept and the middle entries dropped.

Readings where the pages leave a step open:

* Stride-s sampling of a latent frame keeps the positions whose row and
  column are both multiples of s (no extra edge row/column: the pages state
  edge retention only for the Flash token compression).  With a 34 x 60 frame
  this gives 2,040 + 2 x 510 + 8 x 135 = 4,140 history tokens, 2.03 frames:
  "about two full frames".
* The history of a chunk is made of the latent frames before its boundary
  frame (the boundary is the chunk's first target latent and is not repeated
  in the history).
* No VAE is available (it needs trained weights), so the boundary latent of a
  chunk is the last generated latent frame of the chunk before: the
  decode-then-encode round trip is taken as the identity.
* History rows are clean conditions: video modality, noise time 0, not
  updated, RoPE at their original (t, h, w); the token compression acts on
  the chunk's target grid only and history rows pass through it unchanged,
  as control frames do.
* The first chunk has no boundary and no history: it generates all its
  latent frames.  Each later chunk appends its future latents to the stored
  video.
"""

from __future__ import annotations

import numpy as np

from .dit import MOD_AUDIO, MOD_TEXT, MOD_VIDEO, flow_sample

F64 = np.float64

# [tokendh, long-video section; PaperDaily section 三]
HISTORY_FULL = 1       # earliest latent frame, full resolution
HISTORY_RECENT = 2     # most recent frames, spatial stride 2
HISTORY_OLDER = 8      # at most this many frames before them, spatial stride 4
STRIDE_RECENT = 2
STRIDE_OLDER = 4
FUTURE_LATENTS = 5     # future latents after the boundary latent in each chunk
NEW_FRAMES_PER_CHUNK = 17


def stride_positions(H: int, W: int, s: int):
    """(h, w) positions kept by stride-s sampling of an H x W frame, row-major.
    Reading: rows and columns that are multiples of s."""
    return [(h, w) for h in range(0, H, s) for w in range(0, W, s)]


def history_select(n_frames: int):
    """Which stored latent frames form the history, and at what stride.

    ``n_frames`` latent frames exist before the boundary (indices 0 ..
    n_frames-1, oldest first).  Returns [(frame_index, stride)] in time order:
    frame 0 at stride 1; the two newest at stride 2; up to eight before those
    at stride 4; every frame between frame 0 and those ten is dropped."""
    if n_frames <= 0:
        return []
    sel = [(0, 1)]
    rest = list(range(1, n_frames))
    recent = rest[-HISTORY_RECENT:]
    older = rest[:len(rest) - len(recent)][-HISTORY_OLDER:]
    sel += [(i, STRIDE_OLDER) for i in older]
    sel += [(i, STRIDE_RECENT) for i in recent]
    return sel


def history_token_count(n_frames: int, H: int, W: int) -> int:
    """Rows of the history of a chunk preceded by ``n_frames`` latent frames:
    the stride-sampled positions of every frame ``history_select`` keeps."""
    return sum(len(stride_positions(H, W, s)) for _, s in history_select(n_frames))


def history_tokens(frames, selection, t_of_frame=None):
    """Gather the history rows from the stored latent frames.

    ``frames`` is [n, H, W, C]; returns (latents [n_hist, C], pos [n_hist, 3])
    with pos = (t, h, w) at the frame's original coordinates (t = frame index,
    or ``t_of_frame[i]``)."""
    frames = np.asarray(frames, dtype=F64)
    _, H, W, C = frames.shape
    lat, pos = [], []
    for i, s in selection:
        t = i if t_of_frame is None else t_of_frame[i]
        for h, w in stride_positions(H, W, s):
            lat.append(frames[i, h, w])
            pos.append((t, h, w))
    if not lat:
        return np.zeros((0, C), F64), np.zeros((0, 3), np.int32)
    return np.stack(lat), np.asarray(pos, np.int32)


def chunk_tags(grid, base, hist_pos, n_text, n_audio, has_boundary):
    """Per-row tags of one chunk's packed sequence:
    [target grid (T, H, W) at t = base + 0 .. T-1 | history | text | audio].

    Grid frame 0 is the fixed boundary latent when ``has_boundary``: clean
    (time 0) and not updated.  History rows are clean conditions.  Time ids
    index the table [0, t_video, t_audio]."""
    T, H, W = grid
    n_grid = T * H * W
    n_hist = len(hist_pos)
    n = n_grid + n_hist + n_text + n_audio
    modality = np.empty(n, np.uint8)
    time_id = np.zeros(n, np.uint8)
    out_mask = np.zeros(n, np.uint8)
    pos = np.zeros((n, 3), np.int32)
    tt, hh, ww = np.meshgrid(np.arange(T), np.arange(H), np.arange(W), indexing="ij")
    pos[:n_grid] = np.stack([tt.ravel() + base, hh.ravel(), ww.ravel()], axis=1)
    modality[:n_grid] = MOD_VIDEO
    time_id[:n_grid] = 1
    out_mask[:n_grid] = 1
    if has_boundary:
        time_id[:H * W] = 0
        out_mask[:H * W] = 0
    r = n_grid
    modality[r:r + n_hist] = MOD_VIDEO
    if n_hist:
        pos[r:r + n_hist] = hist_pos
    r += n_hist
    modality[r:r + n_text] = MOD_TEXT
    r += n_text
    modality[r:r + n_audio] = MOD_AUDIO
    time_id[r:r + n_audio] = 2
    out_mask[r:r + n_audio] = 1
    if n_audio:
        j = np.arange(n_audio)
        pos[r:r + n_audio, 0] = (j * T) // n_audio + base
    n_vrows = n_grid + n_hist
    return dict(modality=modality, time_id=time_id, out_mask=out_mask, pos=pos,
                n_video=n_grid, video_modality=modality[:n_vrows].copy(),
                video_out=out_mask[:n_vrows].copy(), audio_out=np.ones(n_audio, np.uint8))


def generate_chunks(layers, layer_compress, io, keep_map_fn, grid, n_chunks, noise_video,
                    noise_audio, text_emb, video_clock, audio_clock, heads, head_dim,
                    rope_split=(32, 48, 48), eps=1e-6, theta=10000.0):
    """Generate ``n_chunks`` chunks.  ``noise_video[k]`` is chunk k's initial
    target latents [T*H*W, C] (the boundary slot of chunks k >= 1 is
    overwritten by the boundary latent), ``noise_audio[k]`` its audio latents.

    Returns (frames [n, H, W, C] of the whole video in latent space, the
    per-chunk audio latents, the per-chunk history selections)."""
    T, H, W = grid
    C = np.asarray(noise_video[0]).shape[1]
    frames = np.zeros((0, H, W, C), F64)
    audios, selections = [], []
    keep_idx, near_idx = keep_map_fn(T, H, W)
    for k in range(n_chunks):
        has_b = k > 0
        base = frames.shape[0] - 1 if has_b else 0
        n_before = base if has_b else 0
        sel = history_select(n_before)
        h_lat, h_pos = history_tokens(frames, sel)
        tags = chunk_tags(grid, base, h_pos, np.asarray(text_emb).shape[0],
                          np.asarray(noise_audio[k]).shape[0], has_b)
        tags["keep_idx"], tags["near_idx"] = keep_idx, near_idx
        vl = np.array(noise_video[k], dtype=F64, copy=True)
        if has_b:
            vl[:H * W] = frames[-1].reshape(H * W, C)
        vl = np.concatenate([vl, h_lat], axis=0)
        vl, al = flow_sample(layers, layer_compress, io, tags, video_clock, audio_clock, vl,
                             text_emb, noise_audio[k], heads, head_dim, rope_split, eps, theta)
        new = vl[:T * H * W].reshape(T, H, W, C)
        frames = np.concatenate([frames, new[1:] if has_b else new], axis=0)
        audios.append(al)
        selections.append(sel)
    return frames, audios, selections
