"""Seeded synthetic workloads: shapes, token packing and random tensors.

This module holds no arithmetic of the method: it only draws seeded random
tensors of the right shapes and writes the per-row tags a caller packs
(modality, noise-time slot, 3D position, output mark).  Both the CUDA path's
tests/bench and the oracle's tests take their inputs from here.

Input recipe (the pages' 540p / 22-frame workload is real video; none is
available, so i.i.d. Gaussians of the same shapes stand in for it):
* latents, text features, noise: N(0, 1) from a torch Generator seeded 1234;
* linear weights and biases, modality embeddings: N(0, 0.02), seed 4321;
* RMSNorm gains: 1 + N(0, 0.02);
* bf16 workloads round every drawn value to bf16 once; both sides see the
  same rounded values.

Packing (a caller-side convention, not method arithmetic): rows are
[target video (t, h, w) row-major | control video | text | audio];
positions are (t, h, w) for video, (t - offset, h, w) for control frames so
that target minus control is the constant offset, (0, 0, 0) for text and
(floor(j * T / A), 0, 0) for audio token j.  Time slots: 0 = clean (t = 0),
1 = video clock, 2 = audio clock.
"""

from __future__ import annotations

from dataclasses import dataclass, field, replace

import numpy as np
import torch

MOD_TEXT, MOD_VIDEO, MOD_AUDIO, MOD_CONTROL = 0, 1, 2, 3
SEED_INPUTS = 1234
SEED_WEIGHTS = 4321


@dataclass(frozen=True)
class Workload:
    name: str
    hidden: int = 5376
    heads: int = 56
    head_dim: int = 128
    ffn: int = 14336
    grid: tuple = (6, 34, 60)          # target video grid T, H, W
    control_frames: int = 0            # clean control frames (same H, W)
    control_offset: int = 16           # target t - control t
    n_text: int = 256
    text_dim: int = 5120
    n_audio: int = 64
    audio_dim: int = 64
    video_ch: int = 24
    n_layers: int = 1
    compress: tuple = ()               # per-layer compression flag
    video_clock: tuple = (0.2, 0.0769, 0.027, 0.0)
    audio_clock: tuple = (0.5, 0.25, 0.1, 0.0)
    dtype: str = "bf16"                # "f32" or "bf16"
    rope_split: tuple = (32, 48, 48)
    t_freq: int = 256
    rms_eps: float = 1e-6
    rope_theta: float = 10000.0

    @property
    def attn_dim(self):
        return self.heads * self.head_dim

    @property
    def n_video(self):
        T, H, W = self.grid
        return T * H * W

    @property
    def n_control(self):
        return self.control_frames * self.grid[1] * self.grid[2]

    @property
    def n_tokens(self):
        return self.n_video + self.n_control + self.n_text + self.n_audio

    @property
    def n_evals(self):
        return len(self.video_clock) - 1

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16


def _flash_schedule():
    return tuple([0] * 2 + [1] * 26 + [0] * 14)


WORKLOADS = {
    # tiny fp32 block, checkable on the CPU in seconds
    "tiny_block_f32": Workload("tiny_block_f32", hidden=256, heads=2, head_dim=128,
                               ffn=512, grid=(2, 9, 10), n_text=16, n_audio=8,
                               n_layers=1, compress=(1,), dtype="f32",
                               video_clock=(0.2, 0.0769), audio_clock=(0.5, 0.25)),
    # one full-width Flash block, 6x34x60 video grid
    "flash_block_6x34x60": Workload("flash_block_6x34x60", grid=(6, 34, 60), n_layers=1,
                                    compress=(1,)),
    "flash_block_6x17x30": Workload("flash_block_6x17x30", grid=(6, 17, 30), n_layers=1,
                                    compress=(1,)),
    "flash_block_12x34x60": Workload("flash_block_12x34x60", grid=(12, 34, 60), n_layers=1,
                                     compress=(1,)),
    # the 42-layer Flash backbone, 3 evaluations
    "flash_backbone_6x34x60": Workload("flash_backbone_6x34x60", grid=(6, 34, 60),
                                       n_layers=42, compress=_flash_schedule()),
    "flash_backbone_6x17x30": Workload("flash_backbone_6x17x30", grid=(6, 17, 30),
                                       n_layers=42, compress=_flash_schedule()),
    # the 50-layer standard backbone, 4 evaluations, 4 control frames
    "standard_backbone_12x34x60": Workload(
        "standard_backbone_12x34x60", grid=(12, 34, 60), control_frames=4, n_text=512,
        n_audio=128, n_layers=50, compress=tuple([0] * 50),
        video_clock=(1.0, 0.2, 0.0769, 0.027, 0.0),
        audio_clock=(1.0, 0.5, 0.25, 0.1, 0.0)),
}


@dataclass(frozen=True)
class DecoderWorkload:
    """Shapes of the lightweight video decoder: a transformer over the latent
    cells of a T x H x W grid (hidden 2048, 26 layers, FFN 4 x hidden), each
    cell decoded to a c_pix x patch_t x patch_s x patch_s pixel patch."""
    name: str
    hidden: int = 2048
    heads: int = 16
    head_dim: int = 128
    ffn: int = 8192
    n_layers: int = 26
    grid: tuple = (6, 34, 60)
    c_lat: int = 24
    c_pix: int = 3
    patch_t: int = 4
    patch_s: int = 16
    dtype: str = "bf16"
    rope_split: tuple = (32, 48, 48)
    rms_eps: float = 1e-6
    rope_theta: float = 10000.0

    @property
    def attn_dim(self):
        return self.heads * self.head_dim

    @property
    def n_cells(self):
        T, H, W = self.grid
        return T * H * W

    @property
    def n_frames(self):
        return 1 + self.patch_t * (self.grid[0] - 1)

    @property
    def pixel_cols(self):
        return self.c_pix * self.patch_t * self.patch_s * self.patch_s

    @property
    def pixel_shape(self):
        T, H, W = self.grid
        return (self.n_frames, self.c_pix, H * self.patch_s, W * self.patch_s)

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16


DECODER_WORKLOADS = {
    # tiny fp32 decoder, checkable on the CPU in seconds
    "tiny_decoder_f32": DecoderWorkload("tiny_decoder_f32", hidden=256, heads=2, ffn=1024, n_layers=2,
                                        grid=(3, 4, 5), patch_s=4, dtype="f32"),
    # the 26-layer decoder on the 540p clip's 6 x 34 x 60 latents -> 21 x 3 x 544 x 960
    "decoder_6x34x60": DecoderWorkload("decoder_6x34x60"),
}


def scaled(w: Workload, **kw) -> Workload:
    """A copy of a workload with some fields replaced (smaller test cases)."""
    return replace(w, **kw)


# ---------------------------------------------------------------------------
# Token packing (per-row tags).
# ---------------------------------------------------------------------------

def pack_tokens(w: Workload) -> dict:
    """Per-row tags of the packed sequence as numpy arrays."""
    T, H, W = w.grid
    n = w.n_tokens
    modality = np.empty(n, np.uint8)
    time_id = np.empty(n, np.uint8)
    out_mask = np.zeros(n, np.uint8)
    pos = np.zeros((n, 3), np.int32)
    r = 0
    off = w.control_offset if w.control_frames else 0
    tt, hh, ww = np.meshgrid(np.arange(T), np.arange(H), np.arange(W), indexing="ij")
    vp = np.stack([tt.ravel() + off, hh.ravel(), ww.ravel()], axis=1)
    modality[r:r + w.n_video] = MOD_VIDEO
    time_id[r:r + w.n_video] = 1
    out_mask[r:r + w.n_video] = 1
    pos[r:r + w.n_video] = vp
    r += w.n_video
    if w.control_frames:
        tc, hc, wc = np.meshgrid(np.arange(w.control_frames), np.arange(H), np.arange(W),
                                 indexing="ij")
        modality[r:r + w.n_control] = MOD_CONTROL
        time_id[r:r + w.n_control] = 0
        pos[r:r + w.n_control] = np.stack([tc.ravel(), hc.ravel(), wc.ravel()], axis=1)
        r += w.n_control
    modality[r:r + w.n_text] = MOD_TEXT
    time_id[r:r + w.n_text] = 0
    r += w.n_text
    modality[r:r + w.n_audio] = MOD_AUDIO
    time_id[r:r + w.n_audio] = 2
    out_mask[r:r + w.n_audio] = 1
    if w.n_audio:
        j = np.arange(w.n_audio)
        pos[r:r + w.n_audio, 0] = (j * T) // w.n_audio + off
    r += w.n_audio
    assert r == n
    n_vrows = w.n_video + w.n_control
    return dict(modality=modality, time_id=time_id, out_mask=out_mask, pos=pos,
                n_video=w.n_video,
                video_modality=modality[:n_vrows].copy(),
                video_out=out_mask[:n_vrows].copy(),
                audio_out=np.ones(w.n_audio, np.uint8))


# ---------------------------------------------------------------------------
# Random tensors.
# ---------------------------------------------------------------------------

def _gen(seed, device="cpu"):
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _randn(shape, g, std, dtype, device):
    t = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(dtype)


def make_block_weights(w: Workload, g: torch.Generator, device="cpu", dtype=None):
    """Raw block weights (Linear layout [out, in]) and RMSNorm gains."""
    dt = dtype or w.torch_dtype
    H, F, A = w.hidden, w.ffn, w.attn_dim
    s = 0.02
    out = {
        "w_qkv": _randn((3 * A, H), g, s, dt, device),
        "b_qkv": _randn((3 * A,), g, s, dt, device),
        "w_o": _randn((H, A), g, s, dt, device),
        "b_o": _randn((H,), g, s, dt, device),
        "w_1": _randn((F, H), g, s, dt, device),
        "b_1": _randn((F,), g, s, dt, device),
        "w_2": _randn((H, F), g, s, dt, device),
        "b_2": _randn((H,), g, s, dt, device),
    }
    out["g_attn"] = (1.0 + _randn((H,), g, s, torch.float32, device)).to(dt)
    out["g_ffn"] = (1.0 + _randn((H,), g, s, torch.float32, device)).to(dt)
    return out


def make_io_weights(w: Workload, g: torch.Generator, device="cpu", dtype=None):
    """Embedding, time-MLP and output-head weights."""
    dt = dtype or w.torch_dtype
    H, s = w.hidden, 0.02
    out = {
        "w_vin": _randn((H, w.video_ch), g, s, dt, device),
        "b_vin": _randn((H,), g, s, dt, device),
        "w_tin": _randn((H, w.text_dim), g, s, dt, device),
        "b_tin": _randn((H,), g, s, dt, device),
        "w_ain": _randn((H, w.audio_dim), g, s, dt, device),
        "b_ain": _randn((H,), g, s, dt, device),
        "mod_emb": _randn((4, H), g, s, dt, device),
        "w_t1": _randn((H, w.t_freq), g, s, dt, device),
        "b_t1": _randn((H,), g, s, dt, device),
        "w_t2": _randn((H, H), g, s, dt, device),
        "b_t2": _randn((H,), g, s, dt, device),
        "w_vout": _randn((w.video_ch, H), g, s, dt, device),
        "b_vout": _randn((w.video_ch,), g, s, dt, device),
        "w_aout": _randn((w.audio_dim, H), g, s, dt, device),
        "b_aout": _randn((w.audio_dim,), g, s, dt, device),
    }
    out["g_out"] = (1.0 + _randn((H,), g, s, torch.float32, device)).to(dt)
    return out


def make_inputs(w: Workload, device="cpu", seed=SEED_INPUTS):
    """Noise latents (fp32 state), text features (compute dtype) and the block
    input activations x for single-block workloads."""
    g = _gen(seed, device)
    n_vrows = w.n_video + w.n_control
    return {
        "video_lat": _randn((n_vrows, w.video_ch), g, 1.0, torch.float32, device),
        "audio_lat": _randn((w.n_audio, w.audio_dim), g, 1.0, torch.float32, device),
        "text_emb": _randn((w.n_text, w.text_dim), g, 1.0, w.torch_dtype, device),
        "x": _randn((w.n_tokens, w.hidden), g, 1.0, w.torch_dtype, device),
    }


def make_weights(w: Workload, device="cpu", seed=SEED_WEIGHTS, n_layers=None):
    """All weights of a workload: (list of block weights, io weights)."""
    g = _gen(seed, device)
    L = w.n_layers if n_layers is None else n_layers
    layers = [make_block_weights(w, g, device) for _ in range(L)]
    io = make_io_weights(w, g, device)
    return layers, io


def to_numpy64(d):
    """Dict of tensors -> dict of float64 numpy arrays (for the oracle)."""
    out = {}
    for k, v in d.items():
        if isinstance(v, torch.Tensor):
            out[k] = v.detach().to("cpu", torch.float64).numpy()
        else:
            out[k] = v
    return out


def make_decoder_weights(w: DecoderWorkload, device="cpu", seed=SEED_WEIGHTS, n_layers=None):
    """Decoder weights: (list of block weights, io dict with w_in [hidden,
    c_lat], b_in, g_out, w_out [pixel_cols, hidden], b_out); same init recipe
    as the backbone's."""
    g = _gen(seed, device)
    L = w.n_layers if n_layers is None else n_layers
    layers = [make_block_weights(w, g, device) for _ in range(L)]
    dt, H, s = w.torch_dtype, w.hidden, 0.02
    io = {
        "w_in": _randn((H, w.c_lat), g, s, dt, device),
        "b_in": _randn((H,), g, s, dt, device),
        "w_out": _randn((w.pixel_cols, H), g, s, dt, device),
        "b_out": _randn((w.pixel_cols,), g, s, dt, device),
    }
    io["g_out"] = (1.0 + _randn((H,), g, s, torch.float32, device)).to(dt)
    return layers, io


def make_decoder_latents(w: DecoderWorkload, device="cpu", seed=SEED_INPUTS):
    """Latents [T*H*W, c_lat] fp32, N(0, 1), cells (t, h, w) row-major."""
    return _randn((w.n_cells, w.c_lat), _gen(seed, device), 1.0, torch.float32, device)
