"""Pins of the oracle's composite functions: the timestep MLP, the output
heads, the backbone stack and the few-step sampler.

Each test sets weights that reduce the composite to a closed form the test
writes out by hand (one-hot rows, selection matrices, zero blocks) or to
pieces pinned elsewhere (``embed``, ``dit_block``, ``dit_block_compressed``),
and each docstring names a plausible wiring mistake it would catch.

Sources: [tokendh] backbone section (one forward predicts video and audio
velocity; every row carries its own noise time) and training section (flow
matching, the dual clocks, the Flash layer schedule); [PaperDaily] section 一
(video and audio keep separate noise clocks).
"""

import math

import numpy as np
import pytest
from scipy.special import expit

import oracle as O

# ---------------------------------------------------------------- SiLU


def test_silu_closed_forms():
    """x*sigmoid(x): zero at zero, odd part equal to x/2 (silu(x) - silu(-x) = x),
    slope 1/2 at zero, tends to x for large x and to 0 for large negative x,
    and equals x * scipy's logistic function.  Catches a sigmoid in place of
    silu, a sign error in the exponent, or tanh in place of the logistic."""
    x = np.linspace(-30, 30, 601)
    assert O.silu(0.0) == 0.0
    np.testing.assert_allclose(O.silu(x) - O.silu(-x), x, rtol=0, atol=1e-12)
    h = 1e-7
    assert O.silu(h) / h == pytest.approx(0.5, abs=1e-6)
    assert O.silu(40.0) == pytest.approx(40.0, rel=1e-15)
    assert abs(O.silu(-40.0)) < 1e-15
    np.testing.assert_allclose(O.silu(x), x * expit(x), rtol=1e-13, atol=1e-300)


# ---------------------------------------------------------------- timestep MLP


def _feature(t, i, dim=256, max_period=10000.0):
    """Feature i of the sinusoidal embedding of 1000 t, written per element:
    cos for the first half, sin for the second, frequency max_period^(-j/half)."""
    half = dim // 2
    j = i % half
    arg = 1000.0 * t * max_period ** (-j / half)
    return math.cos(arg) if i < half else math.sin(arg)


def _silu1(v):
    return v / (1.0 + math.exp(-v))


@pytest.mark.parametrize("t", [0.0, 0.0769, 0.2, 0.5, 1.0])
def test_time_embedding_with_identity_layers_is_silu_of_features(t):
    """Identity weights, zero biases: temb(t) = silu(features(t)), element by
    element.  Catches a missing SiLU, SiLU after the second layer, or sin/cos
    halves swapped."""
    io = {"w_t1": np.eye(256), "b_t1": np.zeros(256), "w_t2": np.eye(256), "b_t2": np.zeros(256)}
    got = O.time_embedding(t, io)
    want = np.array([_silu1(_feature(t, i)) for i in range(256)])
    np.testing.assert_allclose(got, want, rtol=1e-11, atol=1e-11)  # arguments up to 1000: ~1e-13 apart


def test_time_embedding_bias_placement():
    """W1 = 0 and b1 = beta: temb = W2 silu(beta) + b2, whatever t is.  Catches
    b1 added after the SiLU (gives W2 beta + b2) or b2 inside it."""
    rng = np.random.default_rng(5)
    H = 8
    beta = rng.standard_normal(H) * 2
    w2 = rng.standard_normal((H, H))
    b2 = rng.standard_normal(H)
    io = {"w_t1": np.zeros((H, 256)), "b_t1": beta, "w_t2": w2, "b_t2": b2}
    want = w2 @ np.array([_silu1(v) for v in beta]) + b2
    for t in (0.0, 0.3, 0.9):
        np.testing.assert_allclose(O.time_embedding(t, io), want, rtol=1e-13, atol=1e-13)


def test_time_embedding_selection_weights_pick_features():
    """W1 selects features (row r reads feature idx[r]), W2 is diagonal d:
    temb_r = d_r silu(f_idx[r](t)).  Catches the two layers applied in the
    wrong order or W1 used transposed."""
    H = 6
    idx = [0, 5, 127, 128, 200, 255]
    w1 = np.zeros((H, 256))
    for r, i in enumerate(idx):
        w1[r, i] = 1.0
    d = np.array([1.0, -2.0, 0.5, 3.0, -1.0, 4.0])
    io = {"w_t1": w1, "b_t1": np.zeros(H), "w_t2": np.diag(d), "b_t2": np.zeros(H)}
    t = 0.027
    want = np.array([d[r] * _silu1(_feature(t, i)) for r, i in enumerate(idx)])
    np.testing.assert_allclose(O.time_embedding(t, io), want, rtol=1e-11, atol=1e-11)


# ---------------------------------------------------------------- output heads


def _head_io(rng, H, c_v=24, c_a=64):
    return {"g_out": 1.0 + rng.uniform(0.2, 1.5, H) * rng.choice([-1, 1], H),
            "w_vout": rng.standard_normal((c_v, H)), "b_vout": rng.standard_normal(c_v),
            "w_aout": rng.standard_normal((c_a, H)), "b_aout": rng.standard_normal(c_a)}


def test_output_heads_on_one_hot_rows():
    """A row c * e_j has RMS |c| / sqrt(H), so with eps = 0 its normalized row
    is sign(c) sqrt(H) g_j e_j and the head returns sign(c) sqrt(H) g_j W[:, j]
    + b.  Video and control rows (modality 1, 3) go to the video head in row
    order, audio rows (2) to the audio head, text rows (0) to neither.
    Catches a missing or misindexed gain, heads applied before the norm,
    control rows dropped, or the two heads swapped."""
    rng = np.random.default_rng(50)
    H = 16
    io = _head_io(rng, H)
    modality = np.array([1, 1, 3, 0, 2, 1, 0, 2])
    j = np.array([0, 5, 9, 3, 15, 7, 2, 4])
    c = np.array([2.5, -0.3, 7.0, 1.0, -4.0, 0.01, 9.0, 3.0])
    x = np.zeros((len(j), H))
    x[np.arange(len(j)), j] = c
    v_vid, v_aud = O.output_heads(x, io, modality, eps=0.0)
    vid_rows = [r for r, m in enumerate(modality) if m in (1, 3)]
    aud_rows = [r for r, m in enumerate(modality) if m == 2]
    assert v_vid.shape == (len(vid_rows), 24) and v_aud.shape == (len(aud_rows), 64)
    for out, rows, w, b in ((v_vid, vid_rows, io["w_vout"], io["b_vout"]),
                            (v_aud, aud_rows, io["w_aout"], io["b_aout"])):
        for k, r in enumerate(rows):
            want = math.copysign(1.0, c[r]) * math.sqrt(H) * io["g_out"][j[r]] * w[:, j[r]] + b
            np.testing.assert_allclose(out[k], want, rtol=1e-12, atol=1e-12)


def test_output_heads_are_invariant_to_row_scale():
    """Norm first: scaling a row by a > 0 leaves its velocity unchanged (eps =
    0).  Catches a head applied to the unnormalized row."""
    rng = np.random.default_rng(51)
    H = 32
    io = _head_io(rng, H)
    modality = np.array([1, 2, 3, 0, 2])
    x = rng.standard_normal((5, H))
    a = np.array([3.0, 0.1, 17.0, 2.0, 1e3])[:, None]
    for u, w in zip(O.output_heads(x, io, modality, 0.0), O.output_heads(a * x, io, modality, 0.0)):
        np.testing.assert_allclose(w, u, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- stack and sampler


def _zero_block(H, F, A):
    return {"w_qkv": np.zeros((3 * A, H)), "b_qkv": np.zeros(3 * A), "w_o": np.zeros((H, A)), "b_o": np.zeros(H),
            "w_1": np.zeros((F, H)), "b_1": np.zeros(F), "w_2": np.zeros((H, F)), "b_2": np.zeros(H),
            "g_attn": np.ones(H), "g_ffn": np.ones(H)}


def _rand_block(rng, H, F, A, s=0.1):
    return {"w_qkv": rng.standard_normal((3 * A, H)) * s, "b_qkv": rng.standard_normal(3 * A) * s,
            "w_o": rng.standard_normal((H, A)) * s, "b_o": rng.standard_normal(H) * s,
            "w_1": rng.standard_normal((F, H)) * s, "b_1": rng.standard_normal(F) * s,
            "w_2": rng.standard_normal((H, F)) * s, "b_2": rng.standard_normal(H) * s,
            "g_attn": 1 + rng.standard_normal(H) * s, "g_ffn": 1 + rng.standard_normal(H) * s}


def _sequence(T=2, Hg=5, Wg=6, n_ctrl=4, n_text=3, n_audio=5):
    """Packed tags: target grid rows, control rows, text, audio (the pages' row
    order), with the sampler's per-row time slots 1 (video clock), 2 (audio
    clock), 0 (clean: text and controls)."""
    V = T * Hg * Wg
    n_v = V + n_ctrl
    n = n_v + n_text + n_audio
    mod = np.array([1] * V + [3] * n_ctrl + [0] * n_text + [2] * n_audio)
    tid = np.array([1] * V + [0] * n_ctrl + [0] * n_text + [2] * n_audio)
    tt, hh, ww = np.meshgrid(np.arange(T), np.arange(Hg), np.arange(Wg), indexing="ij")
    pos = np.zeros((n, 3), np.int64)
    pos[:V] = np.stack([tt.ravel() + 16, hh.ravel(), ww.ravel()], 1)
    pos[V:n_v, 1] = np.arange(n_ctrl) % Hg
    pos[n_v + n_text:, 0] = np.arange(n_audio) * T // n_audio + 16
    keep_idx, near_idx = O.keep_map(T, Hg, Wg)
    return {"modality": mod, "time_id": tid, "pos": pos, "n_video": V, "keep_idx": keep_idx,
            "near_idx": near_idx, "video_modality": mod[:n_v], "video_out": (mod[:n_v] == 1).astype(np.uint8),
            "audio_out": np.ones(n_audio, np.uint8), "n_vrows": n_v, "n_text": n_text, "n_audio": n_audio}


def _io(rng, H, c_text=12, s=0.1):
    return {"w_vin": rng.standard_normal((H, 24)) * s, "b_vin": rng.standard_normal(H) * s,
            "w_tin": rng.standard_normal((H, c_text)) * s, "b_tin": rng.standard_normal(H) * s,
            "w_ain": rng.standard_normal((H, 64)) * s, "b_ain": rng.standard_normal(H) * s,
            "mod_emb": rng.standard_normal((4, H)) * s,
            "w_t1": rng.standard_normal((H, 256)) * s, "b_t1": rng.standard_normal(H) * s,
            "w_t2": rng.standard_normal((H, H)) * s, "b_t2": rng.standard_normal(H) * s,
            "g_out": 1 + rng.standard_normal(H) * s,
            "w_vout": rng.standard_normal((24, H)) * s, "b_vout": rng.standard_normal(24) * s,
            "w_aout": rng.standard_normal((64, H)) * s, "b_aout": rng.standard_normal(64) * s}


def _inputs(rng, tok, c_text=12):
    return (rng.standard_normal((tok["n_vrows"], 24)), rng.standard_normal((tok["n_text"], c_text)),
            rng.standard_normal((tok["n_audio"], 64)))


H_S, F_S, HEADS, HD = 256, 64, 2, 128
A_S = HEADS * HD


def test_stack_of_zero_blocks_is_heads_of_embedding():
    """Zero blocks are exact identities, compressed or not (kept rows take y =
    x, dropped rows x + 0), so the stack returns output_heads(embed(...)) bit
    for bit under any compression schedule.  Catches the heads reading
    anything but the last residual, or a compressed segment that changes rows
    it should not."""
    rng = np.random.default_rng(60)
    tok = _sequence()
    io = _io(rng, H_S)
    vl, te, al = _inputs(rng, tok)
    table = [0.0, 0.2, 0.5]
    x = O.embed(io, tok["modality"], tok["time_id"], table, vl, te, al)
    want = O.output_heads(x, io, tok["modality"])
    layers = [_zero_block(H_S, F_S, A_S) for _ in range(6)]
    for flags in ([0] * 6, [0, 1, 1, 1, 0, 0], [1] * 6):
        for segment in (False, True):
            got = O.dit_stack(layers, flags, io, tok, table, vl, te, al, HEADS, HD, segment=segment)
            for g, w in zip(got, want):
                np.testing.assert_array_equal(g, w)


@pytest.mark.parametrize("layer", [1, 2, 27, 28])
def test_flash_schedule_compresses_exactly_layers_3_to_28(layer):
    """42 layers on the Flash schedule, all zero but one random block at
    0-based index `layer`: the stack equals the heads of that block applied to
    the embedding, compressed (gather, block, nearest-kept broadcast) when the
    page's 1-based layer number layer+1 lies in 3..28 and plain otherwise.
    Catches an off-by-one in the schedule's use (layers 2..27 compressed),
    compression applied to the head or tail layers, or layers run out of
    order."""
    rng = np.random.default_rng(61 + layer)
    tok = _sequence()
    io = _io(rng, H_S)
    vl, te, al = _inputs(rng, tok)
    table = [0.0, 0.0769, 0.25]
    flags = O.flash_layer_compress()
    layers = [_zero_block(H_S, F_S, A_S) for _ in range(42)]
    layers[layer] = _rand_block(rng, H_S, F_S, A_S)
    x = O.embed(io, tok["modality"], tok["time_id"], table, vl, te, al)
    compressed = 3 <= layer + 1 <= 28
    if compressed:
        y = O.dit_block_compressed(x, layers[layer], tok["pos"], HEADS, HD, tok["keep_idx"], tok["near_idx"],
                                   tok["n_video"])
    else:
        y = O.dit_block(x, layers[layer], tok["pos"], HEADS, HD)
    want = O.output_heads(y, io, tok["modality"])
    got = O.dit_stack(layers, flags, io, tok, table, vl, te, al, HEADS, HD)
    for g, w in zip(got, want):
        np.testing.assert_allclose(g, w, rtol=1e-12, atol=1e-12)
    # and the two forms of a block differ on this input, so the test can tell them apart
    other = (O.dit_block(x, layers[layer], tok["pos"], HEADS, HD) if compressed else
             O.dit_block_compressed(x, layers[layer], tok["pos"], HEADS, HD, tok["keep_idx"], tok["near_idx"],
                                    tok["n_video"]))
    assert np.abs(O.output_heads(other, io, tok["modality"])[0] - want[0]).max() > 1e-6


def test_sampler_with_bias_only_velocity_moves_each_modality_by_its_clock_span():
    """Zero blocks and zero head weights: the velocity is the head bias on
    every row, so after the three evaluations target-video latents are x -
    0.2 b_vout, audio latents x - 0.5 b_aout, and control rows are untouched.
    Catches the two clocks swapped, the Euler step's sign, a missing or extra
    evaluation, or control rows being moved."""
    rng = np.random.default_rng(70)
    tok = _sequence()
    io = _io(rng, H_S)
    for k in ("w_vout", "w_aout"):
        io[k] = np.zeros_like(io[k])
    vl, te, al = _inputs(rng, tok)
    layers = [_zero_block(H_S, F_S, A_S) for _ in range(4)]
    flags = [0, 1, 1, 0]
    v_out, a_out = O.flow_sample(layers, flags, io, tok, O.FLASH_VIDEO_CLOCK, O.FLASH_AUDIO_CLOCK, vl, te, al,
                                 HEADS, HD)
    V = tok["n_video"]
    np.testing.assert_allclose(v_out[:V], vl[:V] - 0.2 * io["b_vout"], rtol=0, atol=1e-14)
    np.testing.assert_array_equal(v_out[V:], vl[V:])
    np.testing.assert_allclose(a_out, al - 0.5 * io["b_aout"], rtol=0, atol=1e-14)


@pytest.mark.parametrize("clocks", ["flash", "standard"])
def test_sampler_time_slots_closed_form(clocks):
    """Zero blocks; input projections, biases and modality embeddings zero;
    the timestep MLP routes feature 255, sin(1000 t 10000^(-127/128)), through
    the SiLU into channel j alone.  Each row is then s(t) e_j with s(t) =
    silu(sin(...)) at its own slot's time, its RMSNorm is s g_j /
    sqrt(s^2/H + eps) at j, and the velocity is that times W[:, j] plus b.
    The sampler's result is x + sum_e (t[e+1] - t[e]) v(t[e]) per modality:
    video rows on the video clock, audio rows on the audio clock, control
    rows fixed.  Catches the table's video and audio slots swapped (or the
    clocks read at e+1), cos features in place of sin, the gain or eps
    dropped from the final norm, and heads applied before it."""
    rng = np.random.default_rng(71)
    tok = _sequence()
    H, j, i_feat, eps = H_S, 37, 255, 1e-6
    io = _io(rng, H)
    for k in ("w_vin", "b_vin", "w_tin", "b_tin", "w_ain", "b_ain", "mod_emb", "b_t1", "b_t2", "w_t1", "w_t2"):
        io[k] = np.zeros_like(io[k])
    io["w_t1"][j, i_feat] = 1.0
    io["w_t2"][j, j] = 1.0
    g_j = io["g_out"][j]
    vl, te, al = _inputs(rng, tok)
    layers = [_zero_block(H_S, F_S, A_S) for _ in range(3)]
    flags = [0, 1, 0]
    tv, ta = ((O.FLASH_VIDEO_CLOCK, O.FLASH_AUDIO_CLOCK) if clocks == "flash" else
              (O.STANDARD_VIDEO_CLOCK, O.STANDARD_AUDIO_CLOCK))
    v_out, a_out = O.flow_sample(layers, flags, io, tok, tv, ta, vl, te, al, HEADS, HD, eps=eps)

    def velocity(t, w, b):
        s = _silu1(math.sin(1000.0 * t * 10000.0 ** (-127.0 / 128.0)))
        return s * g_j / math.sqrt(s * s / H + eps) * w[:, j] + b

    want_v, want_a = vl.copy(), al.copy()
    for e in range(len(tv) - 1):
        want_v[:tok["n_video"]] += (tv[e + 1] - tv[e]) * velocity(tv[e], io["w_vout"], io["b_vout"])
        want_a += (ta[e + 1] - ta[e]) * velocity(ta[e], io["w_aout"], io["b_aout"])
    np.testing.assert_allclose(v_out, want_v, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(a_out, want_a, rtol=1e-12, atol=1e-12)
    # the two clocks give different velocities here, so swapped slots would fail
    assert max(abs(velocity(tv[e], io["w_vout"], 0)[0] - velocity(ta[e], io["w_vout"], 0)[0])
               for e in range(len(tv) - 1)) > 1e-3


def test_sampler_segment_form_equals_per_layer_form_through_three_evaluations():
    """The stack's segment form (one gather and one broadcast per run of
    compressed layers) against the per-layer form through a whole 3-evaluation
    sample with random blocks: equal to rounding.  Catches a segment that
    gathers from the wrong residual or broadcasts against the wrong base."""
    rng = np.random.default_rng(72)
    tok = _sequence()
    io = _io(rng, H_S)
    vl, te, al = _inputs(rng, tok)
    layers = [_rand_block(rng, H_S, F_S, A_S, 0.05) for _ in range(5)]
    flags = [0, 1, 1, 1, 0]
    a = O.flow_sample(layers, flags, io, tok, O.FLASH_VIDEO_CLOCK, O.FLASH_AUDIO_CLOCK, vl, te, al, HEADS, HD,
                      segment=False)
    b = O.flow_sample(layers, flags, io, tok, O.FLASH_VIDEO_CLOCK, O.FLASH_AUDIO_CLOCK, vl, te, al, HEADS, HD,
                      segment=True)
    for u, w in zip(a, b):
        np.testing.assert_allclose(u, w, rtol=1e-11, atol=1e-11)


# ---------------------------------------------------------------- small helpers


def test_linear_gather_and_rel_l2_special_cases():
    """linear with the identity is x + b and picks columns for one-hot rows;
    gather_rows puts the kept grid rows first (keep order) and every non-grid
    row after them unchanged; rel_l2 of a 1e-3 relative perturbation is
    1e-3.  Catches W used untransposed, non-grid rows dropped or reordered."""
    rng = np.random.default_rng(80)
    x = rng.standard_normal((4, 6))
    b = rng.standard_normal(6)
    np.testing.assert_array_equal(O.linear(x, np.eye(6), b), x + b)
    w = rng.standard_normal((3, 6))
    np.testing.assert_array_equal(O.linear(np.eye(6)[[2]], w)[0], w[:, 2])
    rows = np.arange(20)[:, None] * np.ones((1, 3))
    g = O.gather_rows(rows, np.array([0, 2, 9]), 12)
    np.testing.assert_array_equal(g[:, 0], [0, 2, 9] + list(range(12, 20)))
    assert O.rel_l2(b * (1 + 1e-3), b) == pytest.approx(1e-3, rel=1e-9)
    assert O.rel_l2(np.zeros(3), np.zeros(3)) == 0.0


def test_every_oracle_function_is_called_by_a_pin():
    """Each public function of the oracle is called by name in some
    tests/test_oracle_*.py file (its pin), so none is trusted unchecked."""
    import glob
    import inspect
    import os
    import re

    from oracle import decoder, dit, fp8, long_video

    here = os.path.dirname(os.path.abspath(__file__))
    text = "".join(open(f, encoding="utf-8").read() for f in glob.glob(os.path.join(here, "test_oracle_*.py")))
    missing = [f"{m.__name__}.{name}" for m in (dit, fp8, long_video, decoder)
               for name, obj in vars(m).items()
               if not name.startswith("_") and inspect.isfunction(obj) and obj.__module__ == m.__name__
               and not re.search(r"\b%s\(" % name, text)]
    assert not missing, missing
