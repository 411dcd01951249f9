"""Pins of the FP8 (E4M3) projection oracle: the rounding against torch's own
float8_e4m3fn / bfloat16 casts and hand-checked special values, the
quantizer's invariants, an exactly representable GEMM, and the quantized
block against the full-precision block.  CPU only."""

import numpy as np
import torch

import oracle as O
from oracle import fp8 as Q


def _torch_e4m3(x):
    return torch.tensor(np.asarray(x, np.float32)).to(torch.float8_e4m3fn).to(torch.float64).numpy()


def test_e4m3_matches_torch_cast_on_random_and_boundary_values():
    rng = np.random.default_rng(1)
    x = np.concatenate([
        rng.uniform(-448, 448, 20000),
        rng.standard_normal(20000) * 2.0 ** rng.integers(-12, 8, 20000),   # every binade incl. subnormals
        rng.uniform(-2.0 ** -6, 2.0 ** -6, 5000),                         # subnormal range
    ]).astype(np.float32)
    np.testing.assert_array_equal(Q.e4m3(x), _torch_e4m3(x))


def test_e4m3_every_code_and_midpoint():
    # all finite positive E4M3 values, from the format's own definition via torch
    codes = torch.arange(0, 127, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert codes.max() == 448.0
    np.testing.assert_array_equal(Q.e4m3(codes), codes)                    # representable values are fixed
    np.testing.assert_array_equal(Q.e4m3(-codes), -codes)
    mids = (codes[1:] + codes[:-1]) / 2                                      # exact ties
    np.testing.assert_array_equal(Q.e4m3(mids), _torch_e4m3(mids))


def test_e4m3_special_values():
    assert Q.e4m3(448.0) == 448.0
    assert Q.e4m3(500.0) == 448.0 and Q.e4m3(1e9) == 448.0 and Q.e4m3(-1e9) == -448.0   # saturation
    assert Q.e4m3(2.0 ** -9) == 2.0 ** -9                                   # smallest subnormal
    assert Q.e4m3(2.0 ** -10) == 0.0                                        # half of it: tie to even 0
    assert Q.e4m3(3 * 2.0 ** -10) == 2.0 ** -8                              # 1.5 quanta: tie to even 2
    assert Q.e4m3(1.0 + 1.0 / 16) == 1.0 and Q.e4m3(1.0 + 3.0 / 16) == 1.25  # ties to even mantissa
    assert Q.e4m3(0.0) == 0.0


def test_bf16_round_matches_torch():
    rng = np.random.default_rng(2)
    x = (rng.standard_normal(50000) * 10.0 ** rng.uniform(-5, 5, 50000)).astype(np.float32)
    ref = torch.tensor(x).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(Q.bf16_round(x), ref)


def test_quantize_rows_invariants():
    rng = np.random.default_rng(3)
    a = (rng.standard_normal((40, 300)) * rng.uniform(0.01, 50, (40, 1))).astype(np.float32)
    a[7] = 0.0
    q, s = Q.quantize_rows(a)
    np.testing.assert_array_equal(Q.e4m3(q), q)                             # codes are E4M3 values
    assert s[7] == 1.0 and not q[7].any()                                    # zero row
    nz = np.arange(40) != 7
    assert (np.abs(q[nz]).max(axis=1) == 448.0).all()                        # the row max lands on 448
    # dequantized error: half an ulp, <= 2^-4 relative (normal) or s * 2^-10 (subnormal)
    err = np.abs(q * s[:, None] - a)
    assert (err <= np.maximum(np.abs(a) * 2.0 ** -4, s[:, None] * 2.0 ** -10) * (1 + 1e-6)).all()
    # scales are fp32 numbers
    np.testing.assert_array_equal(s.astype(np.float32).astype(np.float64), s)


def test_quantize_rows_is_the_plain_quotient():
    # the definition itself on values whose quotient is exact: a row whose
    # amax is 448 has scale 1, and its codes are the E4M3 roundings of the
    # values themselves
    a = np.array([[448.0, 1.0, -3.3, 0.0137, 100.0, -448.0, 5e-4, 17.25]], dtype=np.float32)
    q, s = Q.quantize_rows(a)
    assert s[0] == 1.0
    np.testing.assert_array_equal(q[0], Q.e4m3(a[0].astype(np.float64)))
    # scale 2^k: dividing by a power of two is exact, codes shift by binades
    q2, s2 = Q.quantize_rows(a * np.float32(8.0))
    assert s2[0] == 8.0
    np.testing.assert_array_equal(q2, q)


def test_linear_fp8_exact_on_representable_operands():
    rng = np.random.default_rng(4)
    # entries from E4M3 integers; each row holds 448 so its scale is exactly 1
    vals = np.array([0, 1, 2, 3, 4, 6, 8, 12, 16, 24, 32, 448, -448, -3, -7, 20])
    a = rng.choice(vals, (9, 64)).astype(np.float64); a[:, 0] = 448
    w = rng.choice(vals, (5, 64)).astype(np.float64); w[:, 1] = -448
    qa, sa = Q.quantize_rows(a.astype(np.float32))
    qw, sw = Q.quantize_rows(w.astype(np.float32))
    assert (sa == 1).all() and (sw == 1).all()
    np.testing.assert_array_equal(qa, a)
    b = rng.standard_normal(5)
    np.testing.assert_array_equal(Q.linear_fp8(qa, sa, qw, sw, b), a @ w.T + b)
    # a scaled row: scale s, and the product picks up s exactly
    qa2, sa2 = Q.quantize_rows((a * 0.25).astype(np.float32))
    np.testing.assert_array_equal(qa2, qa)
    np.testing.assert_allclose(Q.linear_fp8(qa2, sa2, qw, sw), 0.25 * (a @ w.T), rtol=1e-15)


def _tiny(rng, H=256, F=512):
    w = {"w_qkv": rng.standard_normal((3 * H, H)) * 0.05, "b_qkv": rng.standard_normal(3 * H) * 0.05,
         "w_o": rng.standard_normal((H, H)) * 0.05, "b_o": rng.standard_normal(H) * 0.05,
         "w_1": rng.standard_normal((F, H)) * 0.05, "b_1": rng.standard_normal(F) * 0.05,
         "w_2": rng.standard_normal((H, F)) * 0.05, "b_2": rng.standard_normal(H) * 0.05,
         "g_attn": 1 + rng.standard_normal(H) * 0.05, "g_ffn": 1 + rng.standard_normal(H) * 0.05}
    return w


def test_fp8_block_stays_within_e4m3_error_of_full_precision_block():
    rng = np.random.default_rng(6)
    n = 24
    w = _tiny(rng)
    x = rng.standard_normal((n, 256))
    pos = rng.integers(0, 9, (n, 3))
    ref = O.dit_block(x, w, pos, 2, 128)
    got = Q.dit_block_fp8(x, w, pos, 2, 128)
    upd = O.rel_l2(got - x, ref - x)
    # E4M3 keeps 3 mantissa bits: the rounding error of one operand is uniform
    # in +-2^-4 relative, 2^-4/sqrt(3) = 3.6% RMS, and each GEMM quantizes two
    # operands (~5.1%); the block update moves by about that (5.3-5.6% on these
    # seeds), not by more than twice it.  A dropped bias, RoPE or scale moves it
    # by O(1).
    assert 1e-3 < upd < 0.1, upd
    # the quantized path is deterministic and its codes come from fp32 inputs
    np.testing.assert_array_equal(Q.dit_block_fp8(x, w, pos, 2, 128), got)


def test_fp8_block_decisions_use_fp32_inputs():
    # perturbing x below fp32 resolution cannot change any quantization code
    rng = np.random.default_rng(7)
    n = 12
    w = _tiny(rng)
    x = rng.standard_normal((n, 256)).astype(np.float32).astype(np.float64)
    pos = rng.integers(0, 9, (n, 3))
    xn = O.rms_norm(x, w["g_attn"], 1e-6)
    q1, s1 = Q.quantize_rows(xn.astype(np.float32))
    q2, s2 = Q.quantize_rows((xn * (1 + 1e-12)).astype(np.float32))
    np.testing.assert_array_equal(q1, q2)
    np.testing.assert_array_equal(s1, s2)


def test_fp8_block_row_restriction_equals_the_block():
    # the row-restricted E4M3 block reproduces the full block's rows (each
    # quantization depends on its own row), also through the compressed form
    rng = np.random.default_rng(12)
    n = 40
    w = _tiny(rng)
    x = rng.standard_normal((n, 256)).astype(np.float32).astype(np.float64)
    pos = rng.integers(0, 9, (n, 3))
    rows = np.array([0, 3, 17, 39])
    full = Q.dit_block_fp8(x, w, pos, 2, 128)
    np.testing.assert_allclose(Q.dit_block_fp8_rows(x, w, pos, 2, 128, rows), full[rows], rtol=1e-10, atol=1e-12)
    # compressed: a 2 x 4 x 5 grid (40 rows, no text/audio)
    k, nn = O.keep_map(2, 4, 5)
    pos_g = np.stack(np.meshgrid(np.arange(2), np.arange(4), np.arange(5), indexing="ij"), -1).reshape(-1, 3)
    fullc = O.dit_block_compressed(x, w, pos_g, 2, 128, k, nn, n, block_fn=Q.dit_block_fp8)
    got = O.dit_block_compressed_rows(x, w, pos_g, 2, 128, k, nn, n, rows, rows_fn=Q.dit_block_fp8_rows)
    np.testing.assert_allclose(got, fullc[rows], rtol=1e-10, atol=1e-12)


def test_quantize_block_weights_quantizes_each_projection_per_output_channel():
    # the four projections, each row (output channel) with its own scale; a
    # row whose largest magnitude is 448 keeps scale 1 and its values' codes
    rng = np.random.default_rng(12)
    w = {"w_qkv": rng.standard_normal((6, 4)), "w_o": rng.standard_normal((4, 2)),
         "w_1": rng.standard_normal((3, 4)), "w_2": rng.standard_normal((4, 3)), "b_o": np.zeros(4)}
    w["w_o"][1] = [448.0, -5.0]
    wq = Q.quantize_block_weights(w)
    assert sorted(wq) == ["w_1", "w_2", "w_o", "w_qkv"]
    for k, (q, s) in wq.items():
        assert q.shape == w[k].shape and s.shape == (w[k].shape[0],)
        np.testing.assert_array_equal(s, np.abs(w[k]).max(axis=1).astype(np.float32) / np.float32(448.0))
    assert wq["w_o"][1][1] == 1.0
    np.testing.assert_array_equal(wq["w_o"][0][1], Q.e4m3(np.array([448.0, -5.0])))
