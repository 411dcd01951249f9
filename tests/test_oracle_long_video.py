"""Pins of the long-video oracle (chunked generation with a bounded,
multi-stride history) against what the pages fix, brute force and
invariants.  CPU only."""

import numpy as np
import pytest

import oracle as O
from oracle import long_video as LV
from few_step_dit_b200 import synthetic as S
from tests.conftest import golden_path


def _golden():
    g = {}
    with open(golden_path("history_budget.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                k, *v = line.split()
                g.setdefault(k, []).append([int(x) for x in v])
    return g


def test_stride_token_counts_and_budget_match_fixture():
    g = _golden()
    for s, n in g["stride"]:
        assert len(LV.stride_positions(34, 60, s)) == n
    assert LV.HISTORY_FULL == g["full_frames"][0][0]
    assert LV.HISTORY_RECENT == g["recent_frames"][0][0]
    assert LV.HISTORY_OLDER == g["older_frames"][0][0]
    # a long video's history holds exactly the printed number of tokens ...
    for n_frames in (11, 12, 40, 500):
        assert LV.history_token_count(n_frames, 34, 60) == g["steady_tokens"][0][0]
    # ... which is "about two full frames" and never more, however long the video
    full = g["full_frame_tokens"][0][0]
    assert max(LV.history_token_count(n, 34, 60) for n in range(0, 80)) == g["steady_tokens"][0][0]
    assert g["steady_tokens"][0][0] <= 2.05 * full


def _select_bruteforce(n):
    """The pages' rule restated per frame: keep frame 0 at full resolution;
    rank every other frame by age (0 = newest); rank 0-1 -> stride 2,
    rank 2-9 -> stride 4, older -> dropped."""
    out = []
    for i in range(n):
        if i == 0:
            out.append((0, 1))
            continue
        rank = n - 1 - i
        if rank < 2:
            out.append((i, 2))
        elif rank < 10:
            out.append((i, 4))
    return out


@pytest.mark.parametrize("n", list(range(0, 30)) + [57, 200])
def test_history_selection_equals_per_frame_rule(n):
    assert LV.history_select(n) == _select_bruteforce(n)


def test_history_selection_examples():
    assert LV.history_select(0) == []
    assert LV.history_select(1) == [(0, 1)]
    assert LV.history_select(3) == [(0, 1), (1, 2), (2, 2)]
    # 20 frames: 1..9 evicted, the initial frame and the ten newest kept
    sel = LV.history_select(20)
    assert [i for i, _ in sel] == [0] + list(range(10, 20))
    assert [s for _, s in sel] == [1] + [4] * 8 + [2] * 2


@pytest.mark.parametrize("H,W", [(34, 60), (9, 10), (7, 5), (1, 1), (4, 8)])
def test_stride_sets_are_nested_and_counted(H, W):
    full = set(LV.stride_positions(H, W, 1))
    s2 = set(LV.stride_positions(H, W, 2))
    s4 = set(LV.stride_positions(H, W, 4))
    assert len(full) == H * W
    assert s4 <= s2 <= full   # a stride-2 copy can be thinned to stride 4
    for s, st in ((2, s2), (4, s4)):
        assert len(st) == -(-H // s) * -(-W // s)
        assert all(h % s == 0 and w % s == 0 for h, w in st)


def test_history_tokens_carry_their_frame_and_position():
    H, W, C, n = 6, 9, 3, 14
    t = np.arange(n)[:, None, None]
    h = np.arange(H)[None, :, None]
    w = np.arange(W)[None, None, :]
    code = (t * 10000 + h * 100 + w).astype(float)
    frames = np.stack([code, -code, code + 0.5], axis=-1)  # value encodes (t, h, w)
    sel = LV.history_select(n)
    lat, pos = LV.history_tokens(frames, sel)
    assert lat.shape == (LV.history_token_count(n, H, W), C)
    dec = lat[:, 0].astype(int)
    np.testing.assert_array_equal(dec // 10000, pos[:, 0])
    np.testing.assert_array_equal((dec // 100) % 100, pos[:, 1])
    np.testing.assert_array_equal(dec % 100, pos[:, 2])
    np.testing.assert_array_equal(lat[:, 1], -lat[:, 0])
    # rows come frame by frame in time order, each frame at its own stride
    r = 0
    for i, s in sel:
        k = len(LV.stride_positions(H, W, s))
        assert (pos[r:r + k, 0] == i).all()
        assert (pos[r:r + k, 1] % s == 0).all() and (pos[r:r + k, 2] % s == 0).all()
        r += k


def test_chunk_tags_boundary_and_history_are_clean_conditions():
    grid = (6, 4, 5)
    _, h_pos = LV.history_tokens(np.zeros((3, 4, 5, 2)), LV.history_select(3))
    tags = LV.chunk_tags(grid, base=10, hist_pos=h_pos, n_text=3, n_audio=4, has_boundary=True)
    n_grid, hw, nh = 6 * 4 * 5, 4 * 5, len(h_pos)
    # boundary frame: clean, fixed, at t = base
    assert (tags["out_mask"][:hw] == 0).all() and (tags["time_id"][:hw] == 0).all()
    assert (tags["pos"][:hw, 0] == 10).all()
    # future latents: noisy, updated, at t = base + 1 .. base + 5
    assert (tags["out_mask"][hw:n_grid] == 1).all() and (tags["time_id"][hw:n_grid] == 1).all()
    assert tags["pos"][hw:n_grid, 0].min() == 11 and tags["pos"][hw:n_grid, 0].max() == 15
    # history: clean video conditions at their own coordinates
    hs = slice(n_grid, n_grid + nh)
    assert (tags["modality"][hs] == O.MOD_VIDEO).all()
    assert (tags["out_mask"][hs] == 0).all() and (tags["time_id"][hs] == 0).all()
    np.testing.assert_array_equal(tags["pos"][hs], h_pos)
    # first chunk: no boundary, every grid row generated
    t0 = LV.chunk_tags(grid, 0, np.zeros((0, 3), np.int32), 3, 4, has_boundary=False)
    assert (t0["out_mask"][:n_grid] == 1).all()


def _tiny_model(dtype="f32"):
    w = S.scaled(S.WORKLOADS["tiny_block_f32"], grid=(3, 4, 6), n_layers=3, compress=(0, 1, 0),
                 dtype=dtype)
    layers, io = S.make_weights(w)
    return w, [S.to_numpy64(l) for l in layers], S.to_numpy64(io)


def _chunk_noise(w, n_chunks, seed=5):
    g = np.random.default_rng(seed)
    T, H, W = w.grid
    nv = [g.standard_normal((T * H * W, w.video_ch)) for _ in range(n_chunks)]
    na = [g.standard_normal((w.n_audio, w.audio_dim)) for _ in range(n_chunks)]
    te = g.standard_normal((w.n_text, w.text_dim))
    return nv, na, te


def test_first_chunk_is_the_plain_sampler_and_boundaries_chain():
    w, layers, io = _tiny_model()
    T, H, W = w.grid
    nv, na, te = _chunk_noise(w, 3)
    frames, audios, sels = LV.generate_chunks(layers, w.compress, io, O.keep_map, w.grid, 3, nv, na, te,
                                              w.video_clock, w.audio_clock, w.heads, w.head_dim)
    # T frames from the first chunk, then T-1 new ones per chunk
    assert frames.shape[0] == T + 2 * (T - 1)
    assert [len(s) for s in sels] == [0, len(LV.history_select(T - 1)), len(LV.history_select(2 * T - 2))]
    # chunk 0 alone is exactly the ordinary few-step sampler on the grid
    tags = LV.chunk_tags(w.grid, 0, np.zeros((0, 3), np.int32), w.n_text, w.n_audio, False)
    tags["keep_idx"], tags["near_idx"] = O.keep_map(*w.grid)
    v0, a0 = O.flow_sample(layers, w.compress, io, tags, w.video_clock, w.audio_clock, nv[0], te, na[0],
                           w.heads, w.head_dim)
    np.testing.assert_array_equal(frames[:T].reshape(-1, w.video_ch), v0)
    np.testing.assert_array_equal(audios[0], a0)
    assert np.isfinite(frames).all()


def test_sampler_leaves_boundary_and_history_rows_untouched():
    w, layers, io = _tiny_model()
    T, H, W = w.grid
    rng = np.random.default_rng(9)
    stored = rng.standard_normal((7, H, W, w.video_ch))
    sel = LV.history_select(6)
    h_lat, h_pos = LV.history_tokens(stored, sel)
    tags = LV.chunk_tags(w.grid, 6, h_pos, w.n_text, w.n_audio, True)
    tags["keep_idx"], tags["near_idx"] = O.keep_map(*w.grid)
    vl = rng.standard_normal((T * H * W, w.video_ch))
    vl[:H * W] = stored[6].reshape(H * W, -1)
    vl = np.concatenate([vl, h_lat])
    te = rng.standard_normal((w.n_text, w.text_dim))
    al = rng.standard_normal((w.n_audio, w.audio_dim))
    out, _ = O.flow_sample(layers, w.compress, io, tags, w.video_clock, w.audio_clock, vl, te, al,
                           w.heads, w.head_dim)
    np.testing.assert_array_equal(out[:H * W], vl[:H * W])               # boundary fixed
    np.testing.assert_array_equal(out[T * H * W:], vl[T * H * W:])       # history fixed
    assert not np.allclose(out[H * W:T * H * W], vl[H * W:T * H * W])    # futures move


def test_history_changes_the_generated_chunk():
    # the history rows are attended to: zeroing them changes the futures
    w, layers, io = _tiny_model()
    T, H, W = w.grid
    rng = np.random.default_rng(11)
    stored = rng.standard_normal((7, H, W, w.video_ch)) * 3
    sel = LV.history_select(6)
    h_lat, h_pos = LV.history_tokens(stored, sel)
    tags = LV.chunk_tags(w.grid, 6, h_pos, w.n_text, w.n_audio, True)
    tags["keep_idx"], tags["near_idx"] = O.keep_map(*w.grid)
    vl = rng.standard_normal((T * H * W, w.video_ch))
    te = rng.standard_normal((w.n_text, w.text_dim))
    al = rng.standard_normal((w.n_audio, w.audio_dim))
    a, _ = O.flow_sample(layers, w.compress, io, tags, w.video_clock, w.audio_clock,
                         np.concatenate([vl, h_lat]), te, al, w.heads, w.head_dim)
    b, _ = O.flow_sample(layers, w.compress, io, tags, w.video_clock, w.audio_clock,
                         np.concatenate([vl, 0 * h_lat]), te, al, w.heads, w.head_dim)
    assert O.rel_l2(a[H * W:T * H * W], b[H * W:T * H * W]) > 1e-6
