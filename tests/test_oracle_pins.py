"""Pins of the oracle against facts the pages fix and against mathematics.

No test here re-types an oracle formula and compares: each checks a printed
value (tests/golden/, with its citation), a closed form, an invariant, a
special case that reduces to something known, or brute force on tiny inputs.
"""

import itertools
import math

import numpy as np
import pytest

import oracle as O
from tests.conftest import golden_path


def _read_golden(name):
    rows = []
    with open(golden_path(name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


# ---------------------------------------------------------------- keep map


def test_keep_map_9x10_matches_printed_rows_and_cols():
    g = {r[0]: r[1:] for r in _read_golden("keep_map_9x10.txt")}
    H, W = int(g["H"][0]), int(g["W"][0])
    rows = [int(v) for v in g["rows"]]
    cols = [int(v) for v in g["cols"]]
    assert O.axis_keep(H) == rows
    assert O.axis_keep(W) == cols
    keep_idx, near_idx = O.keep_map(1, H, W)
    assert keep_idx.tolist() == [h * W + w for h in rows for w in cols]
    assert near_idx.shape == (H * W,)


def test_keep_counts_match_printed_counts():
    for r in _read_golden("keep_counts.txt"):
        if r[0] == "axis":
            assert len(O.axis_keep(int(r[1]))) == int(r[2])
        elif r[0] == "grid":
            T, H, W, total, kept = map(int, r[1:])
            keep_idx, near_idx = O.keep_map(T, H, W)
            assert near_idx.shape[0] == total
            assert keep_idx.shape[0] == kept


@pytest.mark.parametrize("T,H,W", [(1, 1, 1), (1, 2, 2), (2, 3, 4), (2, 9, 10),
                                   (1, 7, 5), (3, 6, 11), (1, 17, 30)])
def test_near_idx_is_bruteforce_euclidean_nearest_in_same_frame(T, H, W):
    keep_idx, near_idx = O.keep_map(T, H, W)
    kept = [(int(p) // (H * W), (int(p) // W) % H, int(p) % W) for p in keep_idx]
    # kept ids strictly increasing, inside the grid
    assert all(a < b for a, b in zip(keep_idx[:-1], keep_idx[1:]))
    for t, h, w in itertools.product(range(T), range(H), range(W)):
        best = None
        for c, (tk, hk, wk) in enumerate(kept):
            if tk != t:
                continue
            d2 = (h - hk) ** 2 + (w - wk) ** 2
            key = (d2, hk, wk)          # ties: lower h, then lower w
            if best is None or key < best[0]:
                best = (key, c)
        assert near_idx[t * H * W + h * W + w] == best[1]


def test_kept_positions_map_to_themselves():
    keep_idx, near_idx = O.keep_map(2, 9, 10)
    assert (keep_idx[near_idx[keep_idx]] == keep_idx).all()


# ---------------------------------------------------------------- attention


def _bruteforce_attention(q, k, v):
    n, nh, d = q.shape
    out = np.zeros((n, nh, d))
    for h in range(nh):
        for i in range(n):
            logits = [sum(q[i, h, c] * k[j, h, c] for c in range(d)) / math.sqrt(d)
                      for j in range(n)]
            m = max(logits)
            ws = [math.exp(s - m) for s in logits]
            z = sum(ws)
            for c in range(d):
                out[i, h, c] = sum(ws[j] * v[j, h, c] for j in range(n)) / z
    return out.reshape(n, nh * d)


def test_attention_equals_bruteforce_on_tiny_inputs():
    rng = np.random.default_rng(7)
    q, k, v = (rng.standard_normal((6, 2, 4)) * 2 for _ in range(3))
    np.testing.assert_allclose(O.attention(q, k, v), _bruteforce_attention(q, k, v),
                               rtol=1e-12, atol=1e-12)


def test_attention_is_asymmetric_in_q_and_k_roles():
    # a transposed score matrix (keys as queries) must not pass
    rng = np.random.default_rng(8)
    q, k, v = (rng.standard_normal((5, 1, 4)) for _ in range(3))
    good = _bruteforce_attention(q, k, v)
    assert np.abs(O.attention(q, k, v) - good).max() < 1e-12
    assert np.abs(O.attention(k, q, v) - good).max() > 1e-3


def test_attention_with_equal_keys_averages_values():
    rng = np.random.default_rng(9)
    n = 11
    q = rng.standard_normal((n, 2, 8))
    k = np.tile(rng.standard_normal((1, 2, 8)), (n, 1, 1))
    v = rng.standard_normal((n, 2, 8))
    out = O.attention(q, k, v).reshape(n, 2, 8)
    np.testing.assert_allclose(out, np.broadcast_to(v.mean(axis=0), out.shape),
                               rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- RoPE


def test_rope_pair_rotation_closed_form():
    d = 128
    x = np.zeros((1, 1, d))
    x[0, 0, 0] = 1.0                       # pair 0 of the t chunk, inv_freq = 1
    y = O.apply_rope(x, np.array([[1, 0, 0]]))
    assert y[0, 0, 0] == pytest.approx(math.cos(1.0), abs=1e-15)
    assert y[0, 0, 1] == pytest.approx(math.sin(1.0), abs=1e-15)
    # pair 1 of the t chunk turns by theta^(-2/32)
    x = np.zeros((1, 1, d))
    x[0, 0, 3] = 1.0
    y = O.apply_rope(x, np.array([[2, 0, 0]]))
    ang = 2 * 10000.0 ** (-2.0 / 32)
    assert y[0, 0, 2] == pytest.approx(-math.sin(ang), abs=1e-15)
    assert y[0, 0, 3] == pytest.approx(math.cos(ang), abs=1e-15)


def test_rope_axis_chunks_32_48_48():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((1, 1, 128))
    for axis, (lo, hi) in enumerate([(0, 32), (32, 80), (80, 128)]):
        pos = np.zeros((1, 3), np.int64)
        pos[0, axis] = 3
        y = O.apply_rope(x, pos)
        changed = np.nonzero(np.abs(y - x)[0, 0] > 1e-14)[0]
        assert changed.min() >= lo and changed.max() < hi
        # the first pair of the chunk turns by exactly pos (inv_freq 1)
        a, b = x[0, 0, lo], x[0, 0, lo + 1]
        assert y[0, 0, lo] == pytest.approx(a * math.cos(3) - b * math.sin(3), abs=1e-14)
    assert sum((32, 48, 48)) == 128


def test_rope_matches_complex_multiplication():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((5, 3, 128))
    pos = rng.integers(0, 40, size=(5, 3))
    y = O.apply_rope(x, pos)
    z = x[..., 0::2] + 1j * x[..., 1::2]
    freqs = np.concatenate([10000.0 ** (-np.arange(0, da, 2) / da) for da in (32, 48, 48)])
    axis_of_pair = np.repeat([0, 1, 2], [16, 24, 24])
    theta = pos[:, axis_of_pair] * freqs[None, :]
    zr = z * np.exp(1j * theta)[:, None, :]
    np.testing.assert_allclose(y[..., 0::2], zr.real, atol=1e-12)
    np.testing.assert_allclose(y[..., 1::2], zr.imag, atol=1e-12)


def test_rope_preserves_norm():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((9, 4, 128))
    pos = rng.integers(0, 60, size=(9, 3))
    y = O.apply_rope(x, pos)
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1),
                               rtol=1e-13)


def test_attention_invariant_to_common_position_shift():
    rng = np.random.default_rng(4)
    n, nh = 10, 2
    q, k, v = (rng.standard_normal((n, nh, 128)) for _ in range(3))
    pos = rng.integers(0, 20, size=(n, 3))
    a0 = O.attention(O.apply_rope(q, pos), O.apply_rope(k, pos), v)
    shift = np.array([[16, 3, -2]])
    a1 = O.attention(O.apply_rope(q, pos + shift), O.apply_rope(k, pos + shift), v)
    np.testing.assert_allclose(a1, a0, rtol=1e-10, atol=1e-12)
    # a relative offset between two groups does change it
    pos2 = pos.copy()
    pos2[:5, 0] += 16
    a2 = O.attention(O.apply_rope(q, pos2), O.apply_rope(k, pos2), v)
    assert np.abs(a2 - a0).max() > 1e-3


# ---------------------------------------------------------------- GELU / RMSNorm


def test_gelu_tanh_special_values_and_erf_bound():
    assert O.gelu_tanh(0.0) == 0.0
    xs = np.linspace(-8, 8, 4001)
    g = O.gelu_tanh(xs)
    np.testing.assert_allclose(g - O.gelu_tanh(-xs), xs, atol=1e-12)
    exact = np.array([0.5 * x * (1 + math.erf(x / math.sqrt(2))) for x in xs])
    # the tanh form approximates the exact GELU to a few 1e-4
    assert np.abs(g - exact).max() < 1e-3
    assert O.gelu_tanh(1.0) == pytest.approx(0.8411919906, abs=1e-9)


def test_rmsnorm_constant_row_and_scale_invariance():
    g = np.array([0.5, 2.0, -1.0, 1.0])
    y = O.rms_norm(np.full(4, -3.0), g, eps=0.0)
    np.testing.assert_allclose(y, -g, rtol=1e-15)
    rng = np.random.default_rng(5)
    x = rng.standard_normal((3, 64))
    gg = rng.standard_normal(64)
    np.testing.assert_allclose(O.rms_norm(7.5 * x, gg, 0.0), O.rms_norm(x, gg, 0.0),
                               rtol=1e-13)
    y = O.rms_norm(x, np.ones(64), 0.0)
    np.testing.assert_allclose(np.mean(y * y, axis=1), 1.0, rtol=1e-13)
    # eps enters inside the root
    assert O.rms_norm(np.array([1e-3]), np.ones(1), 1e-6)[0] == pytest.approx(
        1e-3 / math.sqrt(1e-6 + 1e-6), rel=1e-12)


# ---------------------------------------------------------------- block structure


def _tiny_weights(rng, H, F, zero=()):
    w = {
        "w_qkv": rng.standard_normal((3 * H, H)) * 0.2,
        "b_qkv": rng.standard_normal(3 * H) * 0.2,
        "w_o": rng.standard_normal((H, H)) * 0.2,
        "b_o": rng.standard_normal(H) * 0.2,
        "w_1": rng.standard_normal((F, H)) * 0.2,
        "b_1": rng.standard_normal(F) * 0.2,
        "w_2": rng.standard_normal((H, F)) * 0.2,
        "b_2": rng.standard_normal(H) * 0.2,
        "g_attn": 1 + rng.standard_normal(H) * 0.2,
        "g_ffn": 1 + rng.standard_normal(H) * 0.2,
    }
    for k in zero:
        w[k] = np.zeros_like(w[k])
    return w


def _tiny_tokens(rng, n, grid=None):
    pos = rng.integers(0, 9, size=(n, 3))
    return pos


def test_block_with_zero_projections_is_identity():
    rng = np.random.default_rng(10)
    H, F = 256, 64
    w = _tiny_weights(rng, H, F, zero=("w_qkv", "b_qkv", "w_o", "b_o", "w_1", "b_1",
                                       "w_2", "b_2"))
    x = rng.standard_normal((7, H))
    np.testing.assert_array_equal(O.dit_block(x, w, _tiny_tokens(rng, 7), 2, 128), x)


def test_block_biases_only_adds_them():
    rng = np.random.default_rng(11)
    H, F = 256, 64
    w = _tiny_weights(rng, H, F, zero=("w_qkv", "w_o", "w_1", "b_1"))
    x = rng.standard_normal((5, H))
    # W_o = 0 -> h = x + b_o ; W_1 = 0, b_1 = 0 -> gelu(0) = 0 -> y = h + b_2
    np.testing.assert_allclose(O.dit_block(x, w, _tiny_tokens(rng, 5), 2, 128),
                               x + w["b_o"] + w["b_2"], rtol=1e-14, atol=1e-14)


def test_block_attention_branch_with_equal_keys_is_mean_of_values():
    # W_k = 0 and b_k = 0 -> every key is 0 (RoPE keeps 0 at 0) -> uniform
    # softmax over ALL rows (joint attention, no mask): attn = mean of v rows.
    rng = np.random.default_rng(12)
    H, F, n = 256, 64, 9
    w = _tiny_weights(rng, H, F, zero=("w_1", "b_1", "w_2", "b_2"))
    w["w_qkv"][H:2 * H] = 0
    w["b_qkv"][H:2 * H] = 0
    x = rng.standard_normal((n, H))
    xn = x / np.sqrt(np.mean(x * x, axis=1, keepdims=True) + 1e-6) * w["g_attn"]
    v = xn @ w["w_qkv"][2 * H:].T + w["b_qkv"][2 * H:]
    expect = x + v.mean(axis=0) @ w["w_o"].T + w["b_o"]
    np.testing.assert_allclose(O.dit_block(x, w, _tiny_tokens(rng, n), 2, 128), expect,
                               rtol=1e-12, atol=1e-12)


def test_block_is_prenorm_residual_scale_invariant_update():
    # with the FFN off, y(a x) - a x == y(x) - x (pre-norm + residual)
    rng = np.random.default_rng(13)
    H, F, n = 256, 64, 8
    w = _tiny_weights(rng, H, F, zero=("w_1", "b_1", "w_2", "b_2"))
    x = rng.standard_normal((n, H))
    pos = _tiny_tokens(rng, n)
    d1 = O.dit_block(x, w, pos, 2, 128, eps=0.0) - x
    d2 = O.dit_block(5.0 * x, w, pos, 2, 128, eps=0.0) - 5.0 * x
    np.testing.assert_allclose(d2, d1, rtol=1e-11, atol=1e-11)
    # same for the FFN branch with the attention branch off
    w = _tiny_weights(rng, H, F, zero=("w_qkv", "b_qkv", "w_o", "b_o"))
    d1 = O.dit_block(x, w, pos, 2, 128, eps=0.0) - x
    d2 = O.dit_block(5.0 * x, w, pos, 2, 128, eps=0.0) - 5.0 * x
    np.testing.assert_allclose(d2, d1, rtol=1e-11, atol=1e-11)


def test_block_single_token_attention_returns_its_value():
    rng = np.random.default_rng(14)
    H, F = 256, 64
    w = _tiny_weights(rng, H, F, zero=("w_1", "b_1", "w_2", "b_2"))
    x = rng.standard_normal((1, H))
    xn = x / np.sqrt(np.mean(x * x) + 1e-6) * w["g_attn"]
    v = xn @ w["w_qkv"][2 * H:].T + w["b_qkv"][2 * H:]
    expect = x + v @ w["w_o"].T + w["b_o"]
    np.testing.assert_allclose(O.dit_block(x, w, np.array([[3, 4, 5]]), 2, 128), expect,
                               rtol=1e-12, atol=1e-12)


def test_block_is_permutation_equivariant():
    rng = np.random.default_rng(15)
    H, F, n = 256, 64, 12
    w = _tiny_weights(rng, H, F)
    x = rng.standard_normal((n, H))
    pos = _tiny_tokens(rng, n)
    perm = rng.permutation(n)
    y = O.dit_block(x, w, pos, 2, 128)
    yp = O.dit_block(x[perm], w, pos[perm], 2, 128)
    np.testing.assert_allclose(yp, y[perm], rtol=1e-11, atol=1e-11)


# ---------------------------------------------------------------- compression


def _grid_case(rng, T, Hg, Wg, n_other, H=256, F=64):
    V = T * Hg * Wg
    n = V + n_other
    x = rng.standard_normal((n, H))
    tt, hh, ww = np.meshgrid(np.arange(T), np.arange(Hg), np.arange(Wg), indexing="ij")
    pos = np.zeros((n, 3), np.int64)
    pos[:V] = np.stack([tt.ravel(), hh.ravel(), ww.ravel()], 1)
    return x, pos, V, _tiny_weights(rng, H, F)


def test_keep_all_compressed_block_equals_plain_block_bit_exactly():
    rng = np.random.default_rng(20)
    x, pos, V, w = _grid_case(rng, 2, 3, 4, 5)
    keep_all = np.arange(V, dtype=np.int32)
    y_plain = O.dit_block(x, w, pos, 2, 128)
    y_comp = O.dit_block_compressed(x, w, pos, 2, 128, keep_all, keep_all, V)
    np.testing.assert_array_equal(y_comp, y_plain)


def test_compressed_block_kept_rows_equal_block_on_gathered_rows():
    rng = np.random.default_rng(21)
    T, Hg, Wg = 2, 5, 4
    x, pos, V, w = _grid_case(rng, T, Hg, Wg, 6)
    keep_idx, near_idx = O.keep_map(T, Hg, Wg)
    y = O.dit_block_compressed(x, w, pos, 2, 128, keep_idx, near_idx, V)
    sel = np.concatenate([keep_idx, np.arange(V, x.shape[0])])
    y_c = O.dit_block(x[sel], w, pos[sel], 2, 128)
    np.testing.assert_array_equal(y[keep_idx], y_c[:len(keep_idx)])
    np.testing.assert_array_equal(y[V:], y_c[len(keep_idx):])


def test_broadcast_dropped_rows_carry_nearest_kept_update():
    rng = np.random.default_rng(22)
    T, Hg, Wg = 2, 9, 10
    x, pos, V, w = _grid_case(rng, T, Hg, Wg, 3)
    keep_idx, near_idx = O.keep_map(T, Hg, Wg)
    y = O.dit_block_compressed(x, w, pos, 2, 128, keep_idx, near_idx, V)
    delta = y[:V] - x[:V]
    src = keep_idx[near_idx]
    np.testing.assert_allclose(delta, delta[src], rtol=0, atol=1e-12)
    # dropped rows are not equal to their kept source (full-res residual survives)
    dropped = np.nonzero(src != np.arange(V))[0]
    assert dropped.size == V - len(keep_idx)
    assert np.abs(y[dropped] - y[src[dropped]]).min() > 0


def test_row_restricted_block_equals_full_block_rows():
    rng = np.random.default_rng(24)
    T, Hg, Wg = 2, 5, 6
    x, pos, V, w = _grid_case(rng, T, Hg, Wg, 5)
    rows = np.array([0, 3, 7, 13, V - 1, V, x.shape[0] - 1])
    full = O.dit_block(x, w, pos, 2, 128)
    np.testing.assert_allclose(O.dit_block_rows(x, w, pos, 2, 128, rows), full[rows], rtol=1e-12,
                               atol=1e-12)
    keep_idx, near_idx = O.keep_map(T, Hg, Wg)
    comp = O.dit_block_compressed(x, w, pos, 2, 128, keep_idx, near_idx, V)
    np.testing.assert_allclose(
        O.dit_block_compressed_rows(x, w, pos, 2, 128, keep_idx, near_idx, V, rows), comp[rows],
        rtol=1e-12, atol=1e-12)


def test_segment_form_equals_per_layer_form():
    rng = np.random.default_rng(23)
    T, Hg, Wg = 2, 5, 6
    x, pos, V, _ = _grid_case(rng, T, Hg, Wg, 4)
    H, F = 256, 64
    layers = [_tiny_weights(rng, H, F) for _ in range(4)]
    keep_idx, near_idx = O.keep_map(T, Hg, Wg)
    # per-layer: broadcast after each compressed layer
    xa = x.copy()
    for w in layers:
        xa = O.dit_block_compressed(xa, w, pos, 2, 128, keep_idx, near_idx, V)
    # segment: one gather, four blocks, one broadcast
    sel = np.concatenate([keep_idx, np.arange(V, x.shape[0])])
    xc = x[sel]
    for w in layers:
        xc = O.dit_block(xc, w, pos[sel], 2, 128)
    xb = O.broadcast_residual(x, xc, keep_idx, near_idx, V)
    np.testing.assert_array_equal(xa[keep_idx], xb[keep_idx])
    np.testing.assert_array_equal(xa[V:], xb[V:])
    np.testing.assert_allclose(xa, xb, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- flow matching


def test_clocks_match_printed_values():
    g = {r[0]: [float(v) for v in r[1:]] for r in _read_golden("clocks.txt")}
    assert sorted(O.FLASH_VIDEO_CLOCK) == g["video"]
    assert sorted(O.FLASH_AUDIO_CLOCK) == g["audio"]
    assert list(O.FLASH_VIDEO_CLOCK) == sorted(g["video"], reverse=True)
    assert list(O.STANDARD_VIDEO_CLOCK[1:]) == sorted(g["video"], reverse=True)
    assert list(O.STANDARD_AUDIO_CLOCK[1:]) == sorted(g["audio"], reverse=True)


def test_flash_schedule_matches_printed_split():
    g = {r[0]: int(r[1]) for r in _read_golden("flash_schedule.txt")}
    flags = O.flash_layer_compress()
    assert len(flags) == g["total"]
    assert flags[:g["full_head"]] == [0] * g["full_head"]
    assert flags[g["full_head"]:g["full_head"] + g["compressed"]] == [1] * g["compressed"]
    assert flags[-g["full_tail"]:] == [0] * g["full_tail"]


def test_flow_matching_closed_form_and_euler_recovery():
    rng = np.random.default_rng(30)
    x0 = rng.standard_normal((7, 24))
    eps = rng.standard_normal((7, 24))
    for t in (0.2, 0.0769, 0.5, 1.0):
        xt = O.flow_interpolate(x0, eps, t)
        assert np.allclose(xt, (1 - t) * x0 + t * eps, atol=0, rtol=1e-15)
        v = O.flow_velocity(x0, eps)
        x_rec = O.euler_step(xt, v, np.full(7, O.MOD_VIDEO), np.ones(7),
                             [0, t, 0, 0], [0, 0, 0, 0])
        np.testing.assert_allclose(x_rec, x0, atol=1e-14)
    # endpoints
    np.testing.assert_allclose(O.flow_interpolate(x0, eps, 0.0), x0)
    np.testing.assert_allclose(O.flow_interpolate(x0, eps, 1.0), eps)


def test_euler_chain_over_dual_clocks_recovers_both_modalities():
    rng = np.random.default_rng(31)
    n_v, n_a = 6, 4
    x0 = rng.standard_normal((n_v + n_a, 8))
    eps = rng.standard_normal((n_v + n_a, 8))
    mods = np.array([O.MOD_VIDEO] * n_v + [O.MOD_AUDIO] * n_a)
    tv, ta = O.FLASH_VIDEO_CLOCK, O.FLASH_AUDIO_CLOCK
    x = np.where((mods == O.MOD_VIDEO)[:, None], O.flow_interpolate(x0, eps, tv[0]),
                 O.flow_interpolate(x0, eps, ta[0]))
    v = O.flow_velocity(x0, eps)
    for e in range(3):
        x = O.euler_step(x, v, mods, np.ones(n_v + n_a), [0, tv[e], ta[e], 0],
                         [0, tv[e + 1], ta[e + 1], 0])
        # after each step each modality sits on its own clock
        for m, clk in ((O.MOD_VIDEO, tv), (O.MOD_AUDIO, ta)):
            rows = mods == m
            np.testing.assert_allclose(x[rows],
                                       O.flow_interpolate(x0, eps, clk[e + 1])[rows],
                                       atol=1e-13)
    np.testing.assert_allclose(x, x0, atol=1e-13)


def test_euler_leaves_unmarked_rows():
    rng = np.random.default_rng(32)
    x = rng.standard_normal((5, 3))
    v = rng.standard_normal((5, 3))
    mask = np.array([1, 0, 1, 0, 0])
    mods = np.array([1, 3, 2, 0, 1])
    y = O.euler_step(x, v, mods, mask, [0, 0.2, 0.5, 0], [0, 0.1, 0.25, 0])
    np.testing.assert_array_equal(y[mask == 0], x[mask == 0])
    np.testing.assert_allclose(y[0], x[0] - 0.1 * v[0], rtol=1e-15)
    np.testing.assert_allclose(y[2], x[2] - 0.25 * v[2], rtol=1e-15)


# ---------------------------------------------------------------- embedding / heads


def test_timestep_features_closed_form():
    f0 = O.timestep_features(0.0)
    np.testing.assert_array_equal(f0[:128], 1.0)
    np.testing.assert_array_equal(f0[128:], 0.0)
    f = O.timestep_features(0.2)
    assert f[0] == pytest.approx(math.cos(200.0), abs=1e-12)
    assert f[128] == pytest.approx(math.sin(200.0), abs=1e-12)
    assert f[127] == pytest.approx(math.cos(200.0 * 10000.0 ** (-127 / 128)), abs=1e-12)


def test_embed_routes_rows_by_modality():
    rng = np.random.default_rng(40)
    H = 16
    io = {
        "w_vin": np.eye(H, 3), "b_vin": np.zeros(H),
        "w_tin": 2 * np.eye(H, 5), "b_tin": np.zeros(H),
        "w_ain": 3 * np.eye(H, 4), "b_ain": np.zeros(H),
        "mod_emb": np.zeros((4, H)),
        "w_t1": np.zeros((H, 256)), "b_t1": np.zeros(H),
        "w_t2": np.zeros((H, H)), "b_t2": np.arange(H, dtype=float),
    }
    io["mod_emb"][2] = 100.0
    modality = np.array([1, 1, 3, 0, 2, 0])
    time_id = np.array([1, 1, 0, 0, 2, 0])
    vl = rng.standard_normal((3, 3))
    te = rng.standard_normal((2, 5))
    al = rng.standard_normal((1, 4))
    x = O.embed(io, modality, time_id, [0.0, 0.3, 0.7], vl, te, al)
    base = np.arange(H, dtype=float)
    np.testing.assert_allclose(x[0, :3], vl[0] + base[:3])
    np.testing.assert_allclose(x[2, :3], vl[2] + base[:3])
    np.testing.assert_allclose(x[3, :5], 2 * te[0] + base[:5])
    np.testing.assert_allclose(x[5, :5], 2 * te[1] + base[:5])
    np.testing.assert_allclose(x[4, :4], 3 * al[0] + 100 + base[:4])
    np.testing.assert_allclose(x[4, 4:], 100 + base[4:])


def test_axis_nearest_printed_axes():
    # the 9 x 10 example: rows keep {0,2,4,6,8}, columns {0,2,4,6,8,9}; every
    # dropped index takes the kept index just below it (ties -> lower)
    assert O.axis_nearest(9) == [0, 0, 2, 2, 4, 4, 6, 6, 8]
    assert O.axis_nearest(10) == [0, 0, 2, 2, 4, 4, 6, 6, 8, 9]
    assert O.axis_nearest(1) == [0] and O.axis_nearest(2) == [0, 1]


def test_rope_angles_per_axis_frequencies():
    # position (1, 0, 0) turns only the t chunk (16 pairs) by theta^(-2j/32);
    # (0, 1, 0) only the h chunk (24 pairs) by theta^(-2j/48); (0, 0, 2) the w
    # chunk by 2 theta^(-2j/48)
    ang = O.rope_angles(np.array([[1, 0, 0], [0, 1, 0], [0, 0, 2]]))
    assert ang.shape == (3, 64)
    jt, jh = np.arange(16), np.arange(24)
    np.testing.assert_allclose(ang[0, :16], 10000.0 ** (-2 * jt / 32), rtol=1e-14)
    np.testing.assert_array_equal(ang[0, 16:], 0)
    np.testing.assert_array_equal(ang[1, :16], 0)
    np.testing.assert_allclose(ang[1, 16:40], 10000.0 ** (-2 * jh / 48), rtol=1e-14)
    np.testing.assert_array_equal(ang[1, 40:], 0)
    np.testing.assert_allclose(ang[2, 40:], 2 * 10000.0 ** (-2 * jh / 48), rtol=1e-14)
