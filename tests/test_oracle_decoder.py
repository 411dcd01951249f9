"""Pins of the decoder oracle (CPU only): the placement of the pixel head's
columns is checked against an element-by-element restatement of the
unpatchify rule and against closed forms and locality properties of a
decoder without blocks; the blocks are the backbone's pinned DiT block."""

import numpy as np
import pytest

import oracle as O
from oracle import decoder as D


def _io(rng, hidden, c_lat, c_pix, pt, ps):
    n_out = c_pix * pt * ps * ps
    return {
        "w_in": rng.standard_normal((hidden, c_lat)) * 0.2,
        "b_in": rng.standard_normal(hidden) * 0.1,
        "g_out": 1 + 0.1 * rng.standard_normal(hidden),
        "w_out": rng.standard_normal((n_out, hidden)) * 0.05,
        "b_out": rng.standard_normal(n_out) * 0.1,
    }


def test_grid_positions_brute_force():
    got = D.grid_positions(2, 3, 4)
    want = [(t, h, w) for t in range(2) for h in range(3) for w in range(4)]
    assert got.tolist() == [list(p) for p in want]


@pytest.mark.parametrize("T,pt,frames", [(0, 4, 0), (1, 4, 1), (2, 4, 5), (5, 4, 17), (6, 4, 21), (6, 1, 6)])
def test_decoder_frame_count(T, pt, frames):
    assert D.decoder_frames(T, pt) == frames


@pytest.mark.parametrize("T,H,W,c,pt,ps", [(3, 2, 3, 2, 2, 2), (2, 3, 2, 3, 4, 4), (1, 2, 2, 1, 3, 2)])
def test_unpatchify_matches_elementwise_placement(T, H, W, c, pt, ps):
    rng = np.random.default_rng(0)
    y = rng.standard_normal((T * H * W, c * pt * ps * ps))
    got = D.unpatchify(y, T, H, W, c, pt, ps)
    F = D.decoder_frames(T, pt)
    want = np.full((F, c, H * ps, W * ps), np.nan)
    dropped = 0
    for t in range(T):
        for h in range(H):
            for w in range(W):
                row = (t * H + h) * W + w
                for ch in range(c):
                    for dt in range(pt):
                        f = t * pt + dt - (pt - 1)
                        for dy in range(ps):
                            for dx in range(ps):
                                col = ((ch * pt + dt) * ps + dy) * ps + dx
                                if f < 0:
                                    dropped += 1
                                    continue
                                assert np.isnan(want[f, ch, h * ps + dy, w * ps + dx])  # written once
                                want[f, ch, h * ps + dy, w * ps + dx] = y[row, col]
    assert not np.isnan(want).any()                      # every pixel written
    assert dropped == (pt - 1) * H * W * c * ps * ps     # only latent frame 0's leading slices drop
    np.testing.assert_array_equal(got, want)


def test_head_column_order_dx_fastest():
    assert D.head_column(0, 0, 0, 1, 4, 16) == 1
    assert D.head_column(0, 0, 1, 0, 4, 16) == 16
    assert D.head_column(0, 1, 0, 0, 4, 16) == 256
    assert D.head_column(1, 0, 0, 0, 4, 16) == 1024
    assert D.head_column(2, 3, 15, 15, 4, 16) == 3 * 4 * 256 - 1


def test_zero_block_decoder_with_index_bias_is_closed_form():
    # w_out = 0 and b_out[col] = col: pixel (f, c, y, x) holds the column of
    # (c, dt, y mod ps, x mod ps) with dt = (f + pt - 1) mod pt
    T, H, W, c, pt, ps = 3, 2, 3, 3, 4, 4
    rng = np.random.default_rng(1)
    io = _io(rng, 64, 8, c, pt, ps)
    io["w_out"] = np.zeros_like(io["w_out"])
    io["b_out"] = np.arange(c * pt * ps * ps, dtype=np.float64)
    px = D.decoder_forward(rng.standard_normal((T * H * W, 8)), [], io, T, H, W, 1, 128, c, pt, ps)
    F = D.decoder_frames(T, pt)
    f, ch, yy, xx = np.meshgrid(np.arange(F), np.arange(c), np.arange(H * ps), np.arange(W * ps), indexing="ij")
    want = D.head_column(ch, (f + pt - 1) % pt, yy % ps, xx % ps, pt, ps)
    np.testing.assert_array_equal(px, want)


def test_zero_block_decoder_is_local_to_each_cell():
    # without blocks a latent cell reaches only its own patch: its pt frames
    # (one for latent frame 0), its ps x ps pixels, every channel
    T, H, W, c, pt, ps, c_lat = 3, 3, 4, 3, 4, 4, 8
    rng = np.random.default_rng(2)
    io = _io(rng, 64, c_lat, c, pt, ps)
    lat = rng.standard_normal((T * H * W, c_lat))
    base = D.decoder_forward(lat, [], io, T, H, W, 1, 128, c, pt, ps)
    for (t, h, w) in [(0, 0, 0), (1, 2, 3), (2, 1, 0)]:
        lat2 = lat.copy()
        lat2[(t * H + h) * W + w] += 1.0
        moved = D.decoder_forward(lat2, [], io, T, H, W, 1, 128, c, pt, ps) != base
        f0 = max(0, pt * t - pt + 1)
        expect = np.zeros_like(moved)
        expect[f0:pt * t + 1, :, h * ps:(h + 1) * ps, w * ps:(w + 1) * ps] = True
        np.testing.assert_array_equal(moved, expect)


def test_zero_block_decoder_token_is_norm_then_head():
    # one cell, no blocks: the head sees rmsnorm(W_in z + b_in) -- compare
    # with the RMSNorm written out on that single row
    rng = np.random.default_rng(3)
    io = _io(rng, 32, 4, 1, 1, 2)
    z = rng.standard_normal((1, 4))
    px = D.decoder_forward(z, [], io, 1, 1, 1, 1, 128, 1, 1, 2)
    e = io["w_in"] @ z[0] + io["b_in"]
    n = e / np.sqrt(np.mean(e * e) + 1e-6) * io["g_out"]
    want = (io["w_out"] @ n + io["b_out"]).reshape(1, 1, 2, 2)
    np.testing.assert_allclose(px, want, rtol=1e-12, atol=0)


def test_blocks_with_silent_outputs_reduce_to_the_zero_block_decoder():
    # blocks whose output projections are zero leave x unchanged, so the
    # decoder equals the decoder without blocks; with live outputs it differs
    T, H, W, c, pt, ps, hidden = 2, 3, 2, 3, 4, 2, 256
    rng = np.random.default_rng(4)
    io = _io(rng, hidden, 8, c, pt, ps)
    lat = rng.standard_normal((T * H * W, 8))

    def block(silent):
        w = {"w_qkv": rng.standard_normal((3 * 256, hidden)) * 0.05, "b_qkv": rng.standard_normal(3 * 256) * 0.02,
             "w_o": rng.standard_normal((hidden, 256)) * 0.05, "b_o": rng.standard_normal(hidden) * 0.02,
             "w_1": rng.standard_normal((4 * hidden, hidden)) * 0.05, "b_1": rng.standard_normal(4 * hidden) * 0.02,
             "w_2": rng.standard_normal((hidden, 4 * hidden)) * 0.05, "b_2": rng.standard_normal(hidden) * 0.02,
             "g_attn": np.ones(hidden), "g_ffn": np.ones(hidden)}
        if silent:
            for k in ("w_o", "b_o", "w_2", "b_2"):
                w[k] = np.zeros_like(w[k])
        return w

    base = D.decoder_forward(lat, [], io, T, H, W, 2, 128, c, pt, ps)
    quiet = D.decoder_forward(lat, [block(True), block(True)], io, T, H, W, 2, 128, c, pt, ps)
    np.testing.assert_allclose(quiet, base, rtol=1e-13, atol=1e-13)
    live = D.decoder_forward(lat, [block(False)], io, T, H, W, 2, 128, c, pt, ps)
    assert O.rel_l2(live, base) > 1e-3


def test_full_clip_shapes():
    # the 540p workload: 6 x 34 x 60 latents -> 21 frames of 544 x 960 RGB
    assert D.decoder_frames(6, 4) == 21
    assert (34 * 16, 60 * 16) == (544, 960)
    y = np.zeros((6 * 2 * 3, 3 * 4 * 16 * 16))
    assert D.unpatchify(y, 6, 2, 3, 3, 4, 16).shape == (21, 3, 32, 48)


def test_rgb8_closed_form_values():
    v = np.array([-1.0, 1.0, 0.0, -2.0, 3.0, np.float32(1 / 127.5 - 1), -1 + 3 / 127.5], dtype=np.float32)
    # -1 -> 0, 1 -> 255, 0 -> 127.5 -> 128 (tie to even), out of range clamps,
    # one code step above -1 -> 1, three steps -> 3
    np.testing.assert_array_equal(D.to_rgb8(v), [0, 255, 128, 0, 255, 1, 3])


def test_rgb8_ties_go_to_even_codes():
    # v = (k + 0.5) / 127.5 - 1 lands (in fp32) exactly on k + 0.5 only where
    # that is representable after the two roundings; check those cases
    k = np.arange(0, 255)
    v = ((k + 0.5) / 127.5 - 1).astype(np.float32)
    t = (v * np.float32(127.5)).astype(np.float32) + np.float32(127.5)
    exact = t.astype(np.float64) == k + 0.5
    assert exact.sum() > 50
    got = D.to_rgb8(v)[exact].astype(int)
    want = np.where(k[exact] % 2 == 0, k[exact], k[exact] + 1)
    np.testing.assert_array_equal(got, want)


def test_rgb8_is_monotone_and_within_half_a_code_of_the_exact_map():
    v = np.linspace(-1.2, 1.2, 200001).astype(np.float32)
    q = D.to_rgb8(v).astype(int)
    assert (np.diff(q) >= 0).all()
    exact = np.clip(127.5 * (v.astype(np.float64) + 1), 0, 255)
    assert (np.abs(q - exact) <= 0.5 + 1e-4).all()


def test_decoder_tokens_without_blocks_is_the_latent_projection():
    # no blocks: the hidden state of every cell is W_in z + b_in, cells in
    # (t, h, w) row-major order; a zero block leaves it unchanged
    rng = np.random.default_rng(8)
    io = _io(rng, 256, 5, 3, 1, 2)
    z = rng.standard_normal((2 * 3 * 2, 5))
    x = D.decoder_tokens(z, [], io, 2, 3, 2, 2, 128)
    np.testing.assert_allclose(x, z @ io["w_in"].T + io["b_in"], rtol=1e-13, atol=1e-13)
    zero = {"w_qkv": np.zeros((768, 256)), "b_qkv": np.zeros(768), "w_o": np.zeros((256, 256)),
            "b_o": np.zeros(256), "w_1": np.zeros((64, 256)), "b_1": np.zeros(64), "w_2": np.zeros((256, 64)),
            "b_2": np.zeros(256), "g_attn": np.ones(256), "g_ffn": np.ones(256)}
    np.testing.assert_array_equal(D.decoder_tokens(z, [zero], io, 2, 3, 2, 2, 128), x)


def test_pixel_head_on_one_hot_rows():
    # a row c e_j normalizes (eps = 0) to sign(c) sqrt(H) g_j e_j, so the head
    # returns sign(c) sqrt(H) g_j W_out[:, j] + b_out; a missing gain or the
    # head applied before the norm fails
    rng = np.random.default_rng(9)
    H = 16
    io = _io(rng, H, 4, 3, 1, 2)
    j, c = np.array([0, 7, 15]), np.array([3.0, -0.2, 40.0])
    x = np.zeros((3, H))
    x[np.arange(3), j] = c
    got = D.pixel_head(x, io, eps=0.0)
    for r in range(3):
        want = np.sign(c[r]) * np.sqrt(H) * io["g_out"][j[r]] * io["w_out"][:, j[r]] + io["b_out"]
        np.testing.assert_allclose(got[r], want, rtol=1e-12, atol=1e-12)
