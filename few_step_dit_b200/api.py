"""Python API over the C ABI: torch tensors in, torch tensors out.

PyTorch supplies device memory and streams only; every step runs in
libfsdit.so.  Buffers (outputs, workspaces) are allocated here with torch, so
the library itself allocates nothing.
"""

from __future__ import annotations

import ctypes as C

import numpy as np
import torch

from . import lib as L

TORCH_OF = {L.F32: torch.float32, L.BF16: torch.bfloat16}


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return C.c_void_p(s.cuda_stream)


def dtype_code(t_dtype):
    return L.BF16 if t_dtype == torch.bfloat16 else L.F32


def make_dims(hidden, heads, ffn, dtype, head_dim=128, rope_split=(32, 48, 48), rms_eps=1e-6,
              rope_theta=10000.0, proj_fp8=False):
    d = L.Dims()
    d.hidden, d.heads, d.head_dim, d.ffn = hidden, heads, head_dim, ffn
    d.rope_split[:] = list(rope_split)
    d.rms_eps, d.rope_theta = rms_eps, rope_theta
    d.dtype = dtype if isinstance(dtype, int) else dtype_code(dtype)
    d.proj_fp8 = int(bool(proj_fp8))
    return d


def dims_of(w, proj_fp8=False):
    """Dims of a synthetic Workload."""
    return make_dims(w.hidden, w.heads, w.ffn, L.F32 if w.dtype == "f32" else L.BF16,
                     w.head_dim, w.rope_split, w.rms_eps, w.rope_theta, proj_fp8)


class BlockWeights:
    """Device weights of one block (dict of tensors) and their C struct.  For
    E4M3 projections the four projection weights are uint8 code tensors and
    s_qkv, s_o, s_1, s_2 their scales (see quantize_block_weights)."""

    def __init__(self, tensors: dict):
        self.tensors = {k: v.contiguous() for k, v in tensors.items()}
        ptrs = [self.tensors[k].data_ptr() for k in L.BLOCK_FIELDS]
        ptrs += [self.tensors[k].data_ptr() if k in self.tensors else None for k in L.BLOCK_SCALE_FIELDS]
        self.struct = L.BlockWeights(*ptrs)


_PROJ = (("w_qkv", "s_qkv"), ("w_o", "s_o"), ("w_1", "s_1"), ("w_2", "s_2"))


def quantize_rows(a, stream=None):
    """Per-row E4M3 codes (uint8) and fp32 scales of a [rows, cols] fp32 or bf16 matrix."""
    rows, cols = a.shape
    q = torch.empty(rows, cols, dtype=torch.uint8, device=a.device)
    s = torch.empty(max(rows, 1), dtype=torch.float32, device=a.device)
    L.call("fsdit_quantize_rows", L.ptr(a), dtype_code(a.dtype), rows, cols, L.ptr(q), L.ptr(s), _stream(stream))
    return q, s[:rows]


def quantize_block_weights(tensors: dict, stream=None):
    """The same block with its four projection weights quantized per output
    channel (E4M3 codes + scales), ready for dims with proj_fp8."""
    out = dict(tensors)
    for w, s in _PROJ:
        out[w], out[s] = quantize_rows(tensors[w].contiguous(), stream)
    return out


def rmsnorm_quant(x, g, eps=1e-6, stream=None):
    rows, hidden = x.shape
    q = torch.empty(rows, hidden, dtype=torch.uint8, device=x.device)
    s = torch.empty(max(rows, 1), dtype=torch.float32, device=x.device)
    L.call("fsdit_rmsnorm_quant", L.ptr(x), L.ptr(g), rows, hidden, float(eps), L.ptr(q), L.ptr(s),
           _stream(stream))
    return q, s[:rows]


def linear_fp8(dims, qa, sa, qw, sw, b, epilogue=L.EPI_BIAS, resid=None, pos=None, out=None, scratch=None,
               stream=None):
    """E4M3 projection: epilogue((qa qw^T) * sa[row] * sw[col] + b)."""
    M, K = qa.shape
    N = qw.shape[0]
    if out is None:
        od = torch.float32 if epilogue in (L.EPI_RESIDUAL, L.EPI_BIAS_F32) else torch.bfloat16
        out = torch.empty(M, N, dtype=od, device=qa.device)
    L.call("fsdit_linear_fp8_ws", C.byref(dims), L.ptr(qa), L.ptr(sa), L.ptr(qw), L.ptr(sw), L.ptr(b), L.ptr(out),
           L.ptr(resid), L.ptr(pos), M, N, K, epilogue, L.ptr(scratch),
           scratch.numel() if scratch is not None else 0, _stream(stream))
    return out


class IOWeights:
    def __init__(self, tensors: dict):
        self.tensors = {k: v.contiguous() for k, v in tensors.items()}
        t = self.tensors
        self.struct = L.IOWeights(*[t[k].data_ptr() for k in L.IO_FIELDS],
                                  t["w_vin"].shape[1], t["w_tin"].shape[1], t["w_ain"].shape[1],
                                  t["w_t1"].shape[1])


def keep_map(T, H, W, device="cuda", stream=None):
    """Device keep-index map of a T x H x W grid: (keep_idx, near_idx) int32."""
    lib = L.load()
    n_keep = lib.fsdit_keep_count(T, H, W)
    keep_idx = torch.empty(max(n_keep, 1), dtype=torch.int32, device=device)
    near_idx = torch.empty(max(T * H * W, 1), dtype=torch.int32, device=device)
    L.call("fsdit_build_keep_map", T, H, W, L.ptr(keep_idx), L.ptr(near_idx), _stream(stream))
    return keep_idx[:n_keep], near_idx[:T * H * W]


class Sequence:
    """Per-row tags of a packed sequence on the device, plus the keep map of
    its target grid when `compress` is set."""

    def __init__(self, tags: dict, grid, n_vrows, n_text, n_audio, device="cuda", compress=True,
                 stream=None):
        self.grid = tuple(grid)
        self.n_vrows, self.n_text, self.n_audio = n_vrows, n_text, n_audio
        self.n_tokens = n_vrows + n_text + n_audio
        dev = torch.device(device)
        self.pos = torch.as_tensor(np.ascontiguousarray(tags["pos"], np.int32)).to(dev)
        self.modality = torch.as_tensor(np.ascontiguousarray(tags["modality"], np.uint8)).to(dev)
        self.time_id = torch.as_tensor(np.ascontiguousarray(tags["time_id"], np.uint8)).to(dev)
        self.out_mask = torch.as_tensor(np.ascontiguousarray(tags["out_mask"], np.uint8)).to(dev)
        T, H, W = self.grid
        self.n_grid = T * H * W
        self.keep_idx = self.near_idx = None
        self.n_keep = 0
        if compress and self.n_grid > 0:
            self.keep_idx, self.near_idx = keep_map(T, H, W, dev, stream)
            self.n_keep = int(self.keep_idx.numel())
        self.struct = self._make_struct(compress)
        self.struct_full = self._make_struct(False)

    @property
    def n_compressed(self):
        return self.n_keep + self.n_tokens - self.n_grid

    def _make_struct(self, compress):
        T, H, W = self.grid
        s = L.Tokens()
        s.n_tokens, s.n_vrows, s.n_text, s.n_audio = self.n_tokens, self.n_vrows, self.n_text, self.n_audio
        s.grid_t, s.grid_h, s.grid_w = T, H, W
        s.pos_thw = self.pos.data_ptr()
        s.modality = self.modality.data_ptr()
        s.time_id = self.time_id.data_ptr()
        s.out_mask = self.out_mask.data_ptr()
        if compress and self.keep_idx is not None:
            s.keep_idx, s.n_keep, s.near_idx = self.keep_idx.data_ptr(), self.n_keep, self.near_idx.data_ptr()
        else:
            s.keep_idx, s.n_keep, s.near_idx = None, 0, None
        return s

    @classmethod
    def from_workload(cls, w, tags, device="cuda", compress=None):
        comp = any(w.compress) if compress is None else compress
        return cls(tags, w.grid, w.n_video + w.n_control, w.n_text, w.n_audio, device, comp)


# ---------------------------------------------------------------- single steps

def gather_rows(x, pos, keep_idx, n_grid, stream=None):
    n_rows, hidden = x.shape
    n_keep = keep_idx.numel()
    n_out = n_keep + n_rows - n_grid
    xc = torch.empty(n_out, hidden, dtype=torch.float32, device=x.device)
    posc = torch.empty(n_out, 3, dtype=torch.int32, device=x.device) if pos is not None else None
    L.call("fsdit_gather_rows", L.ptr(x), L.ptr(pos), L.ptr(xc), L.ptr(posc), L.ptr(keep_idx),
           n_keep, n_grid, n_rows, hidden, _stream(stream))
    return xc, posc


def broadcast_residual(x, yc, keep_idx, near_idx, grid, out=None, stream=None):
    n_rows, hidden = x.shape
    T, H, W = grid
    if out is None:
        out = torch.empty_like(x)
    L.call("fsdit_broadcast_residual", L.ptr(x), L.ptr(yc), L.ptr(out), L.ptr(keep_idx),
           L.ptr(near_idx), keep_idx.numel(), T, H, W, n_rows, hidden, _stream(stream))
    return out


def rmsnorm_cast(x, g, eps=1e-6, stream=None):
    rows, hidden = x.shape
    xn = torch.empty(rows, hidden, dtype=g.dtype, device=x.device)
    L.call("fsdit_rmsnorm_cast", L.ptr(x), L.ptr(g), L.ptr(xn), rows, hidden, eps,
           dtype_code(g.dtype), _stream(stream))
    return xn


def gemm_scratch(device):
    """Caller scratch for the projections' tail cut (fsdit_gemm_scratch_size bytes)."""
    return torch.empty(L.load().fsdit_gemm_scratch_size(), dtype=torch.uint8, device=device)


def linear(dims, a, w, b, epilogue=L.EPI_BIAS, resid=None, pos=None, out=None, scratch=None, stream=None):
    """out = epilogue(a w^T + b); with `scratch` (gemm_scratch) the last wave's
    tiles may be cut along K (fsdit_linear_ws)."""
    M, K = a.shape
    N = w.shape[0]
    if out is None:
        od = torch.float32 if epilogue in (L.EPI_BIAS_F32, L.EPI_RESIDUAL) else a.dtype
        out = torch.empty(M, N, dtype=od, device=a.device)
    L.call("fsdit_linear_ws", C.byref(dims), L.ptr(a), L.ptr(w), L.ptr(b), L.ptr(out), L.ptr(resid),
           L.ptr(pos), M, N, K, epilogue, L.ptr(scratch), scratch.numel() if scratch is not None else 0,
           _stream(stream))
    return out


def attention(dims, qkv, out=None, stream=None):
    n = qkv.shape[0]
    if out is None:
        out = torch.empty(n, dims.heads * dims.head_dim, dtype=qkv.dtype, device=qkv.device)
    L.call("fsdit_attention", C.byref(dims), L.ptr(qkv), L.ptr(out), n, _stream(stream))
    return out


def euler_step(x, v, row_modality, out_mask, t_cur, t_next, stream=None):
    n_rows, width = x.shape
    tc = (C.c_float * 4)(*[float(t) for t in t_cur])
    tn = (C.c_float * 4)(*[float(t) for t in t_next])
    L.call("flow_euler_step", L.ptr(x), L.ptr(v), L.ptr(row_modality), L.ptr(out_mask), n_rows, width,
           tc, tn, _stream(stream))
    return x


def device_error(stream=None):
    L.call("fsdit_device_error", _stream(stream))


# ---------------------------------------------------------------- block / stack / sampler

_ws_cache: dict = {}


def workspace(nbytes, device):
    """A cached uint8 device buffer of at least nbytes (caller-side allocation).

    One buffer per device serves every call of this module, so calls on one
    device must not overlap in time (issue them on one stream, or synchronize
    between streams); concurrent work needs the C ABI with a workspace per
    stream."""
    key = str(device)
    buf = _ws_cache.get(key)
    if buf is None or buf.numel() < nbytes:
        _ws_cache.pop(key, None)
        buf = torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)
        _ws_cache[key] = buf
    return buf


def block_forward(dims, weights: BlockWeights, seq: Sequence, x_in, x_out=None, compress=True,
                  stream=None):
    lib = L.load()
    tok = seq.struct if compress else seq.struct_full
    nbytes = lib.fsdit_block_workspace_size(C.byref(dims), seq.n_tokens, tok.n_keep)
    ws = workspace(nbytes, x_in.device)
    if x_out is None:
        x_out = torch.empty_like(x_in)
    L.call("dit_block_forward", C.byref(dims), C.byref(weights.struct), C.byref(tok), L.ptr(x_in),
           L.ptr(x_out), L.ptr(ws), ws.numel(), _stream(stream))
    return x_out


class Backbone:
    """Stack of blocks + io weights, ready for dit_stack_forward / dit_flow_sample."""

    def __init__(self, dims, layers, io: IOWeights, layer_compress):
        self.dims = dims
        self.layers = layers
        self.io = io
        n = len(layers)
        self.n_layers = n
        self.layer_structs = (L.BlockWeights * max(n, 1))(*[lw.struct for lw in layers])
        self.compress = (C.c_uint8 * max(n, 1))(*[int(c) for c in layer_compress])

    def workspace_bytes(self, seq: Sequence, compress=True, n_times=3):
        tok = seq.struct if compress else seq.struct_full
        return L.load().fsdit_stack_workspace_size(C.byref(self.dims), C.byref(self.io.struct),
                                                   C.byref(tok), n_times)

    def forward(self, seq: Sequence, time_table, video_lat, text_emb, audio_lat, compress=True,
                v_video=None, v_audio=None, stream=None):
        tok = seq.struct if compress else seq.struct_full
        dev = video_lat.device
        ws = workspace(self.workspace_bytes(seq, compress, len(time_table)), dev)
        if v_video is None:
            v_video = torch.empty(seq.n_vrows, self.io.struct.c_video, dtype=torch.float32, device=dev)
        if v_audio is None:
            v_audio = torch.empty(seq.n_audio, self.io.struct.c_audio, dtype=torch.float32, device=dev)
        tt = (C.c_float * len(time_table))(*[float(t) for t in time_table])
        L.call("dit_stack_forward", C.byref(self.dims), self.n_layers, self.layer_structs, self.compress,
               C.byref(self.io.struct), C.byref(tok), tt, len(time_table), L.ptr(video_lat),
               L.ptr(text_emb), L.ptr(audio_lat), L.ptr(v_video), L.ptr(v_audio), L.ptr(ws), ws.numel(),
               _stream(stream))
        return v_video, v_audio

    def sample(self, seq: Sequence, video_clock, audio_clock, video_lat, text_emb, audio_lat,
               compress=True, stream=None):
        """Few-step sampler; updates video_lat / audio_lat in place and returns them."""
        tok = seq.struct if compress else seq.struct_full
        ws = workspace(self.workspace_bytes(seq, compress, 3), video_lat.device)
        E = len(video_clock) - 1
        tv = (C.c_float * (E + 1))(*[float(t) for t in video_clock])
        ta = (C.c_float * (E + 1))(*[float(t) for t in audio_clock])
        L.call("dit_flow_sample", C.byref(self.dims), self.n_layers, self.layer_structs, self.compress,
               C.byref(self.io.struct), C.byref(tok), E, tv, ta, L.ptr(video_lat), L.ptr(text_emb),
               L.ptr(audio_lat), L.ptr(ws), ws.numel(), _stream(stream))
        return video_lat, audio_lat


# ---------------------------------------------------------------- long video

class HistoryStore:
    """Device store of a video's latent frames for the bounded multi-stride
    history (fsdit_history_*): frame 0 plus the newest capacity-1 frames."""

    def __init__(self, H, W, C_ch, capacity=L.HISTORY_MIN_SLOTS, device="cuda"):
        lib = L.load()
        nbytes = lib.fsdit_history_bytes(capacity, H, W, C_ch)
        self.frames = torch.empty(max(nbytes // 4, 1), dtype=torch.float32, device=device)
        self.s = L.HistoryStore()
        self.H, self.W, self.C = H, W, C_ch
        L.call("fsdit_history_init", C.byref(self.s), L.ptr(self.frames), capacity, H, W, C_ch)

    @property
    def n_frames(self):
        return self.s.n_frames

    def push(self, frames, stream=None):
        """Append latent frames (contiguous fp32, H*W*C values per frame)."""
        fe = self.H * self.W * self.C
        assert frames.dtype == torch.float32 and frames.is_contiguous() and frames.numel() % fe == 0
        L.call("fsdit_history_push", C.byref(self.s), L.ptr(frames), frames.numel() // fe, _stream(stream))

    def plan(self, n_before):
        """History plan of a chunk whose boundary is frame n_before."""
        out = (L.HistoryEntry * L.HISTORY_MAX_ENTRIES)()
        n = L.load().fsdit_history_plan(int(n_before), out, L.HISTORY_MAX_ENTRIES)
        if n < 0:
            raise L.FsditError("fsdit_history_plan", n, "bad n_before")
        return out, n

    def rows(self, plan, n):
        return L.load().fsdit_history_rows(plan, n, self.H, self.W)

    def gather(self, plan, n, lat, pos, stream=None):
        """Write the plan's rows into lat [rows, >= C] fp32 and pos [rows, 3] int32."""
        L.call("fsdit_history_gather", C.byref(self.s), plan, n, L.ptr(lat), lat.stride(0), L.ptr(pos),
               _stream(stream))

    def copy_frame(self, frame, dst, stream=None):
        L.call("fsdit_history_copy_frame", C.byref(self.s), int(frame), L.ptr(dst), _stream(stream))


def chunk_tags(grid, base, has_boundary, n_hist, n_text, n_audio):
    """Host row tags of one chunk (fsdit_chunk_tags); history pos rows are left
    zero for the gather to fill."""
    T, H, W = grid
    n = T * H * W + n_hist + n_text + n_audio
    mod = np.zeros(n, np.uint8)
    tid = np.zeros(n, np.uint8)
    out = np.zeros(n, np.uint8)
    pos = np.zeros((n, 3), np.int32)
    L.call("fsdit_chunk_tags", T, H, W, int(base), int(bool(has_boundary)), n_hist, n_text, n_audio,
           mod.ctypes.data, tid.ctypes.data, out.ctypes.data, pos.ctypes.data)
    return dict(modality=mod, time_id=tid, out_mask=out, pos=pos)


class LongVideo:
    """Chunked long-video generation: each chunk samples [boundary + future
    latents | history | text | audio] with the few-step sampler and appends its
    new latent frames to the history store."""

    def __init__(self, backbone: Backbone, grid, n_text, n_audio, video_ch, capacity=L.HISTORY_MIN_SLOTS,
                 device="cuda"):
        self.bb = backbone
        self.grid = tuple(grid)
        self.n_text, self.n_audio = n_text, n_audio
        T, H, W = self.grid
        self.store = HistoryStore(H, W, video_ch, capacity, device)
        self.device = torch.device(device)
        self.compress = any(int(c) for c in backbone.compress)

    def prepare(self, stream=None):
        """Sequence and latent buffer of the next chunk, history gathered, the
        boundary latent in place.  Returns (seq, video_lat, has_boundary)."""
        T, H, W = self.grid
        hw, n_grid = H * W, T * H * W
        has_b = self.store.n_frames > 0
        base = self.store.n_frames - 1 if has_b else 0
        plan, n_plan = self.store.plan(base if has_b else 0)
        n_hist = self.store.rows(plan, n_plan)
        tags = chunk_tags(self.grid, base, has_b, n_hist, self.n_text, self.n_audio)
        seq = Sequence(tags, self.grid, n_grid + n_hist, self.n_text, self.n_audio, self.device,
                       self.compress, stream)
        vl = torch.empty(n_grid + n_hist, self.store.C, dtype=torch.float32, device=self.device)
        if n_hist:
            self.store.gather(plan, n_plan, vl[n_grid:], seq.pos[n_grid:n_grid + n_hist], stream)
        return seq, vl, has_b, base

    def chunk(self, noise_video, text_emb, noise_audio, video_clock, audio_clock, stream=None):
        """Generate one chunk from its initial target latents [T*H*W, C] and
        audio latents; returns (target latents [T*H*W, C], audio latents)."""
        T, H, W = self.grid
        hw, n_grid = H * W, T * H * W
        seq, vl, has_b, base = self.prepare(stream)
        vl[:n_grid].copy_(noise_video)
        if has_b:
            self.store.copy_frame(base, vl[:hw], stream)
        al = noise_audio.clone()
        self.bb.sample(seq, video_clock, audio_clock, vl, text_emb, al, stream=stream)
        self.store.push(vl[hw:n_grid] if has_b else vl[:n_grid], stream)
        return vl[:n_grid], al


# ---------------------------------------------------------------- decoder

class DecoderIO:
    """Latent projection, final RMSNorm gain and pixel head of the decoder
    (w_in [hidden, c_lat], b_in, g_out, w_out [c_pix*patch_t*patch_s^2, hidden], b_out)."""

    def __init__(self, tensors: dict, c_pix=3, patch_t=4, patch_s=16):
        self.tensors = {k: v.contiguous() for k, v in tensors.items()}
        t = self.tensors
        if t["w_out"].shape[0] != c_pix * patch_t * patch_s * patch_s:
            raise ValueError("w_out must have c_pix * patch_t * patch_s^2 rows")
        self.struct = L.DecoderIO(*[t[k].data_ptr() for k in L.DECODER_IO_FIELDS], t["w_in"].shape[1],
                                  c_pix, patch_t, patch_s)


class Decoder:
    """The lightweight video decoder: latents [T*H*W, c_lat] (cells (t, h, w)
    row-major) -> pixels [1 + patch_t*(T-1), c_pix, H*patch_s, W*patch_s]."""

    def __init__(self, dims, layers, io: DecoderIO):
        self.dims = dims
        self.layers = layers
        self.io = io
        self.n_layers = len(layers)
        self.layer_structs = (L.BlockWeights * max(self.n_layers, 1))(*[lw.struct for lw in layers])

    def frames(self, T):
        return L.load().fsdit_decoder_frames(T, self.io.struct.patch_t)

    def workspace_bytes(self, grid):
        T, H, W = grid
        return L.load().fsdit_decoder_workspace_size(C.byref(self.dims), C.byref(self.io.struct), T, H, W)

    def forward(self, latents, grid, pixels=None, rgb8=False, stream=None):
        """Pixels as fp32 values, or (rgb8) as the uint8 codes of the fused
        colour conversion."""
        T, H, W = grid
        s = self.io.struct
        if pixels is None:
            pixels = torch.empty(self.frames(T), s.c_pix, H * s.patch_s, W * s.patch_s,
                                 dtype=torch.uint8 if rgb8 else torch.float32, device=latents.device)
        ws = workspace(self.workspace_bytes(grid), latents.device)
        L.call("fsdit_decoder_forward", C.byref(self.dims), self.n_layers, self.layer_structs, C.byref(s), T, H, W,
               L.ptr(latents), L.ptr(pixels), L.PIXELS_RGB8 if rgb8 else L.PIXELS_F32, L.ptr(ws), ws.numel(),
               _stream(stream))
        return pixels
