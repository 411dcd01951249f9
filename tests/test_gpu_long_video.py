"""Long-video chunking on the GPU (through the C ABI) against the oracle.

History gather: bit-exact (index work), at the full 34 x 60 x 24 latent frame
size.  Chunked generation: fp32 relative L2 <= 1e-5, bf16 <= 1e-2 on every
generated frame and on the audio latents.  Full width: the properties every
chunk must have (boundary and history rows untouched, futures moved)."""

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


@pytest.mark.parametrize("capacity,batches", [(12, [6, 5, 5, 5, 5, 1, 5]), (13, [1, 1, 1, 9, 5, 5]),
                                              (12, [30])])
def test_history_gather_bit_exact_full_frame(capacity, batches):
    H, W, Cc = 34, 60, 24
    rng = np.random.default_rng(3)
    total = sum(batches)
    frames = rng.standard_normal((total, H, W, Cc)).astype(np.float32)
    store = api.HistoryStore(H, W, Cc, capacity, DEV)
    fd = torch.as_tensor(frames).to(DEV)
    done = 0
    for b in batches:
        store.push(fd[done:done + b].contiguous())
        done += b
        for n_before in (done - 1, done):
            plan, n = store.plan(n_before)
            rows = store.rows(plan, n)
            if rows == 0:
                continue
            lat = torch.full((rows, Cc + 8), float("nan"), device=DEV)  # ld_lat = C + 8
            pos = torch.full((rows, 3), -7, dtype=torch.int32, device=DEV)
            store.gather(plan, n, lat, pos)
            torch.cuda.synchronize()
            ref_lat, ref_pos = LV.history_tokens(frames[:done], LV.history_select(n_before))
            np.testing.assert_array_equal(lat[:, :Cc].cpu().numpy(), ref_lat.astype(np.float32))
            np.testing.assert_array_equal(pos.cpu().numpy(), ref_pos)
            assert torch.isnan(lat[:, Cc:]).all()  # columns past C untouched
    # the boundary copy reads the newest frame back exactly; an evicted frame is refused
    dst = torch.empty(H * W, Cc, device=DEV)
    store.copy_frame(done - 1, dst)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(dst.cpu().numpy(), frames[done - 1].reshape(H * W, Cc))
    if done > capacity:
        with pytest.raises(L.FsditError):
            store.copy_frame(1, dst)


def _model(dtype, hidden=256, heads=2, ffn=512):
    w = S.scaled(S.WORKLOADS["tiny_block_f32"], grid=(3, 4, 6), n_layers=3, compress=(0, 1, 0), dtype=dtype,
                 hidden=hidden, heads=heads, ffn=ffn)
    layers, io = S.make_weights(w)
    bb = api.Backbone(api.dims_of(w), [api.BlockWeights({k: v.to(DEV) for k, v in l.items()}) for l in layers],
                      api.IOWeights({k: v.to(DEV) for k, v in io.items()}), w.compress)
    return w, layers, io, bb


@pytest.mark.parametrize("dtype,bound", [("f32", 1e-5), ("bf16", 1e-2)])
def test_chunked_generation_matches_oracle(dtype, bound):
    n_chunks = 4
    w, layers, io, bb = _model(dtype)
    T, H, W = w.grid
    g = np.random.default_rng(5)
    f32 = lambda a: a.astype(np.float32).astype(np.float64)  # both sides start from the same values
    nv = [f32(g.standard_normal((T * H * W, w.video_ch))) for _ in range(n_chunks)]
    na = [f32(g.standard_normal((w.n_audio, w.audio_dim))) for _ in range(n_chunks)]
    te = g.standard_normal((w.n_text, w.text_dim))
    lv = api.LongVideo(bb, w.grid, w.n_text, w.n_audio, w.video_ch)
    te_d = torch.as_tensor(te).to(DEV, w.torch_dtype)
    got_frames, got_audio = [], []
    for k in range(n_chunks):
        out, al = lv.chunk(torch.as_tensor(nv[k], dtype=torch.float32).to(DEV), te_d,
                           torch.as_tensor(na[k], dtype=torch.float32).to(DEV), w.video_clock, w.audio_clock)
        o = out.double().cpu().numpy().reshape(T, H, W, -1)
        got_frames.append(o if k == 0 else o[1:])
        got_audio.append(al.double().cpu().numpy())
    torch.cuda.synchronize()
    assert lv.store.n_frames == T + (n_chunks - 1) * (T - 1)
    # the oracle sees the same bf16-rounded text the GPU path reads
    te_ref = torch.as_tensor(te).to(w.torch_dtype).double().numpy()
    frames, audios, sels = LV.generate_chunks([S.to_numpy64(l) for l in layers], w.compress, S.to_numpy64(io),
                                              O.keep_map, w.grid, n_chunks, nv, na, te_ref, w.video_clock,
                                              w.audio_clock, w.heads, w.head_dim)
    got = np.concatenate(got_frames)
    assert got.shape == frames.shape
    assert O.rel_l2(got, frames) < bound
    for k in range(n_chunks):
        assert O.rel_l2(got_audio[k], audios[k]) < bound
    # chunk 3 already drops nothing but uses every kind of history entry
    assert {s for _, s in sels[-1]} == {1, 2, 4}


def test_full_width_steady_state_chunk_keeps_boundary_and_history():
    w = S.scaled(S.WORKLOADS["flash_backbone_6x34x60"], n_layers=4, compress=(0, 1, 1, 0))
    T, H, W = w.grid
    layers, io = S.make_weights(w, device=DEV)
    bb = api.Backbone(api.dims_of(w), [api.BlockWeights(l) for l in layers], api.IOWeights(io), w.compress)
    inp = S.make_inputs(w, device=DEV)
    lv = api.LongVideo(bb, w.grid, w.n_text, w.n_audio, w.video_ch)
    g = torch.Generator(device=DEV).manual_seed(8)
    past = torch.randn(21 * H * W, w.video_ch, generator=g, device=DEV)
    lv.store.push(past)                                  # 21 frames: a full 11-entry history
    seq, vl, has_b, base = lv.prepare()
    n_grid, hw = T * H * W, H * W
    assert has_b and base == 20 and vl.shape[0] - n_grid == 4140
    vl[:n_grid].copy_(inp["video_lat"][:n_grid])
    lv.store.copy_frame(base, vl[:hw])
    before = vl.clone()
    al = inp["audio_lat"].clone()
    bb.sample(seq, w.video_clock, w.audio_clock, vl, inp["text_emb"], al)
    torch.cuda.synchronize()
    assert torch.equal(vl[:hw], past[20 * hw:21 * hw])          # boundary = newest stored frame
    assert torch.equal(vl[:hw], before[:hw])                    # and fixed through 3 evaluations
    assert torch.equal(vl[n_grid:], before[n_grid:])            # history rows fixed
    assert torch.isfinite(vl).all() and torch.isfinite(al).all()
    assert not torch.equal(vl[hw:n_grid], before[hw:n_grid])    # futures moved
    assert not torch.equal(al, inp["audio_lat"])
    # the history rows are the oracle's gather of the stored frames
    ref_lat, ref_pos = LV.history_tokens(past.cpu().numpy().reshape(21, H, W, -1), LV.history_select(20))
    np.testing.assert_array_equal(vl[n_grid:].cpu().numpy(), ref_lat.astype(np.float32))
    np.testing.assert_array_equal(seq.pos[n_grid:n_grid + 4140].cpu().numpy(), ref_pos)
