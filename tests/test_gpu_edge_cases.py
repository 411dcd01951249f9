"""Degenerate inputs through the CUDA path against the oracle (fp32, rel-L2 <=
1e-5): sequences without text or audio rows, a one-token grid (compression
keeps everything), frames two wide (the stride-2 set and the edge set
coincide), the sampler with empty modalities, and the smallest long-video
chunk (boundary + one future frame)."""

import numpy as np
import pytest
import torch

import oracle as O
from oracle import long_video as LV
from few_step_dit_b200 import api, build, lib as L
from few_step_dit_b200 import synthetic as S

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    L.load()
    yield
    torch.cuda.synchronize()
    api.device_error()


def _tiny(**kw):
    return S.scaled(S.WORKLOADS["tiny_block_f32"], **kw)


@pytest.mark.parametrize("grid,n_text,n_audio", [((2, 9, 10), 0, 0), ((2, 9, 10), 16, 0), ((2, 9, 10), 0, 8),
                                                 ((1, 1, 1), 16, 8), ((3, 2, 2), 5, 3), ((1, 2, 7), 0, 1)])
@pytest.mark.parametrize("compress", [True, False])
def test_block_degenerate_sequences(grid, n_text, n_audio, compress):
    w = _tiny(grid=grid, n_text=n_text, n_audio=n_audio)
    layers, _ = S.make_weights(w, n_layers=1)
    inp = S.make_inputs(w)
    tags = S.pack_tokens(w)
    seq = api.Sequence.from_workload(w, tags, DEV, compress=True)
    bw = api.BlockWeights({k: v.to(DEV) for k, v in layers[0].items()})
    x = inp["x"].float()
    out = api.block_forward(api.dims_of(w), bw, seq, x.to(DEV), compress=compress)
    torch.cuda.synchronize()
    xn = x.double().numpy()
    wn = S.to_numpy64(layers[0])
    if compress:
        k, n = O.keep_map(*w.grid)
        ref = O.dit_block_compressed(xn, wn, tags["pos"], w.heads, w.head_dim, k, n, w.n_video)
    else:
        ref = O.dit_block(xn, wn, tags["pos"], w.heads, w.head_dim)
    assert O.rel_l2(out.double().cpu().numpy(), ref) < 1e-5
    assert O.rel_l2(out.double().cpu().numpy() - xn, ref - xn) < 1e-5


@pytest.mark.parametrize("dtype,bound", [("f32", 1e-5), ("bf16", 1e-2)])
@pytest.mark.parametrize("split", [(34, 46, 48), (30, 50, 48)])
def test_block_rope_split_with_odd_pair_counts(split, dtype, bound):
    # chunk widths of 17 / 23 and 15 / 25 pairs: the RoPE table, the QKV
    # epilogue and the oracle all take the axis of each pair from the split
    w = _tiny(rope_split=split, dtype=dtype)
    layers, _ = S.make_weights(w, n_layers=1)
    inp = S.make_inputs(w)
    tags = S.pack_tokens(w)
    seq = api.Sequence.from_workload(w, tags, DEV, compress=True)
    bw = api.BlockWeights({k: v.to(DEV) for k, v in layers[0].items()})
    x = inp["x"].float()
    out = api.block_forward(api.dims_of(w), bw, seq, x.to(DEV), compress=True)
    torch.cuda.synchronize()
    xn = x.double().numpy()
    k, n = O.keep_map(*w.grid)
    ref = O.dit_block_compressed(xn, S.to_numpy64(layers[0]), tags["pos"], w.heads, w.head_dim, k, n, w.n_video,
                                 rope_split=split)
    got = out.double().cpu().numpy()
    assert O.rel_l2(got, ref) < bound
    assert O.rel_l2(got - xn, ref - xn) < bound


def test_one_token_grid_compression_keeps_everything():
    # a 1 x 1 x 1 grid keeps its only token: compressed block == plain block bit for bit
    w = _tiny(grid=(1, 1, 1))
    layers, _ = S.make_weights(w, n_layers=1)
    inp = S.make_inputs(w)
    seq = api.Sequence.from_workload(w, S.pack_tokens(w), DEV, compress=True)
    assert seq.n_keep == 1
    bw = api.BlockWeights({k: v.to(DEV) for k, v in layers[0].items()})
    x = inp["x"].float().to(DEV)
    a = api.block_forward(api.dims_of(w), bw, seq, x, compress=True)
    b = api.block_forward(api.dims_of(w), bw, seq, x, compress=False)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


@pytest.mark.parametrize("n_text,n_audio", [(0, 0), (0, 8), (16, 0)])
def test_sampler_with_empty_modalities(n_text, n_audio):
    w = _tiny(grid=(2, 5, 6), n_text=n_text, n_audio=n_audio, n_layers=3, compress=(0, 1, 0),
              video_clock=S.WORKLOADS["flash_backbone_6x34x60"].video_clock,
              audio_clock=S.WORKLOADS["flash_backbone_6x34x60"].audio_clock)
    layers, io = S.make_weights(w)
    inp = S.make_inputs(w)
    tags = S.pack_tokens(w)
    seq = api.Sequence.from_workload(w, tags, DEV)
    bb = api.Backbone(api.dims_of(w), [api.BlockWeights({k: v.to(DEV) for k, v in l.items()}) for l in layers],
                      api.IOWeights({k: v.to(DEV) for k, v in io.items()}), w.compress)
    vl, al = inp["video_lat"].to(DEV).clone(), inp["audio_lat"].to(DEV).clone()
    bb.sample(seq, w.video_clock, w.audio_clock, vl, inp["text_emb"].to(DEV), al)
    torch.cuda.synchronize()
    tok = dict(tags)
    tok["keep_idx"], tok["near_idx"] = O.keep_map(*w.grid)
    rv, ra = O.flow_sample([S.to_numpy64(l) for l in layers], w.compress, S.to_numpy64(io), tok, w.video_clock,
                           w.audio_clock, inp["video_lat"].double().numpy(), inp["text_emb"].double().numpy(),
                           inp["audio_lat"].double().numpy(), w.heads, w.head_dim)
    assert O.rel_l2(vl.double().cpu().numpy(), rv) < 1e-5
    if n_audio:
        assert O.rel_l2(al.double().cpu().numpy(), ra) < 1e-5


@pytest.mark.parametrize("grid,n_text,n_audio", [((1, 1, 1), 16, 8), ((3, 2, 2), 5, 3), ((1, 2, 7), 0, 1),
                                                 ((2, 9, 10), 0, 0)])
def test_bf16_sampler_on_tiny_sequences(grid, n_text, n_audio):
    # bf16 at hidden 256 (the stack applies each norm after its consuming
    # GEMM) on sequences of 13 to 180 rows: the projections run on the
    # single-CTA GEMM (M <= 128) or on partly filled pair tiles
    w = _tiny(grid=grid, n_text=n_text, n_audio=n_audio, n_layers=4, compress=(0, 1, 1, 0), dtype="bf16",
              video_clock=S.WORKLOADS["flash_backbone_6x34x60"].video_clock,
              audio_clock=S.WORKLOADS["flash_backbone_6x34x60"].audio_clock)
    layers, io = S.make_weights(w)
    inp = S.make_inputs(w)
    tags = S.pack_tokens(w)
    seq = api.Sequence.from_workload(w, tags, DEV)
    bb = api.Backbone(api.dims_of(w), [api.BlockWeights({k: v.to(DEV) for k, v in l.items()}) for l in layers],
                      api.IOWeights({k: v.to(DEV) for k, v in io.items()}), w.compress)
    vl, al = inp["video_lat"].to(DEV).clone(), inp["audio_lat"].to(DEV).clone()
    bb.sample(seq, w.video_clock, w.audio_clock, vl, inp["text_emb"].to(DEV), al)
    torch.cuda.synchronize()
    tok = dict(tags)
    tok["keep_idx"], tok["near_idx"] = O.keep_map(*w.grid)
    rv, ra = O.flow_sample([S.to_numpy64(l) for l in layers], w.compress, S.to_numpy64(io), tok, w.video_clock,
                           w.audio_clock, inp["video_lat"].double().numpy(), inp["text_emb"].double().numpy(),
                           inp["audio_lat"].double().numpy(), w.heads, w.head_dim)
    v0 = inp["video_lat"].double().numpy()
    got = vl.double().cpu().numpy()
    assert O.rel_l2(got, rv) < 1e-2
    assert O.rel_l2(got - v0, rv - v0) < 1e-2
    if n_audio:
        assert O.rel_l2(al.double().cpu().numpy(), ra) < 1e-2


def test_smallest_long_video_chunks():
    # T = 2: each later chunk is one boundary latent and one new latent
    w = _tiny(grid=(2, 4, 5), n_layers=2, compress=(1, 0))
    layers, io = S.make_weights(w)
    bb = api.Backbone(api.dims_of(w), [api.BlockWeights({k: v.to(DEV) for k, v in l.items()}) for l in layers],
                      api.IOWeights({k: v.to(DEV) for k, v in io.items()}), w.compress)
    T, H, W = w.grid
    g = np.random.default_rng(12)
    f32 = lambda a: a.astype(np.float32).astype(np.float64)
    n_chunks = 5
    nv = [f32(g.standard_normal((T * H * W, w.video_ch))) for _ in range(n_chunks)]
    na = [f32(g.standard_normal((w.n_audio, w.audio_dim))) for _ in range(n_chunks)]
    te = f32(g.standard_normal((w.n_text, w.text_dim)))
    lv = api.LongVideo(bb, w.grid, w.n_text, w.n_audio, w.video_ch)
    got = []
    for k in range(n_chunks):
        out, _ = lv.chunk(torch.as_tensor(nv[k], dtype=torch.float32).to(DEV),
                          torch.as_tensor(te, dtype=torch.float32).to(DEV),
                          torch.as_tensor(na[k], dtype=torch.float32).to(DEV), w.video_clock, w.audio_clock)
        o = out.double().cpu().numpy().reshape(T, H, W, -1)
        got.append(o if k == 0 else o[1:])
    torch.cuda.synchronize()
    frames, _, _ = LV.generate_chunks([S.to_numpy64(l) for l in layers], w.compress, S.to_numpy64(io), O.keep_map,
                                      w.grid, n_chunks, nv, na, te, w.video_clock, w.audio_clock, w.heads, w.head_dim)
    got = np.concatenate(got)
    assert got.shape == frames.shape == (T + n_chunks - 1, H, W, w.video_ch)
    assert O.rel_l2(got, frames) < 1e-5
