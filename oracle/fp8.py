"""fp64 CPU oracle of the low-bit (FP8 E4M3) block projections (test
infrastructure only; see the package docstring).

Source: [PaperDaily] section 二 "Flash怎么把22帧压到377毫秒", third step: the
model switches suitable projection layers to low-bit weights and activations
and fuses normalization, quantization, RoPE and the residual update into the
surrounding computation.  The pages give no format or scaling, so every choice
below is a reading:

* Format: FP8 E4M3 (OCP "E4M3FN": 1 sign, 4 exponent bits with bias 7, 3
  mantissa bits, subnormals, no infinity, largest finite 448).  Rounding is to
  nearest with ties to even; magnitudes beyond 448 saturate to 448.
* Scaling: one fp32 scale per row of the operand that is quantized -- per
  token for activations, per output channel for weights: s = amax / 448
  (rounded to fp32, as a stored scale is; 1 for an all-zero row) and
  q = E4M3(value / s), the quotient of the fp32 value by the fp32 scale taken
  in float64 and rounded once to E4M3 (ties to even).
* Which projections: the four of every block (QKV, O, FFN up, FFN down); the
  input/output embeddings, the time MLP and the heads stay as they are.
* GEMM: out = (sum_k q_a q_w) * s_a[row] * s_w[col] + bias, then the
  projection's own epilogue (RoPE, GELU or residual).
* What each quantizer sees: the fp32 RMSNorm output (x * rstd * gain) for the
  QKV and FFN-up inputs; the attention output and the GELU output rounded to
  bf16 (the kernels store them in bf16 before quantizing them).
"""

from __future__ import annotations

import numpy as np

from .dit import apply_rope, attention, gelu_tanh, rms_norm

F64 = np.float64
F32 = np.float32
E4M3_MAX = 448.0


def e4m3(x):
    """Nearest E4M3 value of each element (ties to even, saturating at 448),
    returned in float64."""
    x = np.asarray(x, dtype=F64)
    a = np.abs(x)
    _, ex = np.frexp(np.where(a > 0, a, 1.0))  # a = m 2^ex, m in [0.5, 1)
    e = np.maximum(ex - 1, -6)                  # binade exponent; subnormals share -6
    quantum = np.ldexp(1.0, e - 3)              # 3 mantissa bits
    r = np.round(a / quantum) * quantum         # exact scaling; round half to even
    r = np.minimum(r, E4M3_MAX)
    return np.where(x < 0, -r, r)


def bf16_round(x):
    """Round to the nearest bfloat16 (ties to even), returned in float64."""
    x32 = np.asarray(x, dtype=F32)
    b = x32.view(np.uint32).astype(np.uint64)
    b = (b + 0x7FFF + ((b >> 16) & 1)) & 0xFFFF0000
    return b.astype(np.uint32).view(F32).astype(F64)


def quantize_rows(a):
    """Per-row E4M3 quantization of a [R, K] operand given in fp32.

    Returns (q [R, K] float64 holding E4M3 values, s [R] float64 holding the
    fp32 scales) with a ~= q * s[:, None]: s = fp32(amax / 448), q = E4M3(a / s)."""
    a32 = np.asarray(a, dtype=F32)
    amax = np.max(np.abs(a32), axis=1) if a32.shape[1] else np.zeros(a32.shape[0], F32)
    s = np.where(amax > 0, amax / F32(E4M3_MAX), F32(1.0)).astype(F32)
    q = e4m3(a32.astype(F64) / s.astype(F64)[:, None])
    return q, s.astype(F64)


def linear_fp8(qa, sa, qw, sw, b=None):
    """(qa qw^T) * sa[row] * sw[col] + b, in float64."""
    y = (np.asarray(qa, F64) @ np.asarray(qw, F64).T) * np.asarray(sa, F64)[:, None] * np.asarray(sw, F64)[None, :]
    if b is not None:
        y = y + np.asarray(b, F64)
    return y


def quantize_block_weights(w):
    """The four projection weights of a block, quantized per output channel
    from their stored values.  Returns {name: (q, s)}."""
    return {k: quantize_rows(np.asarray(w[k], F64).astype(F32)) for k in ("w_qkv", "w_o", "w_1", "w_2")}


def dit_block_fp8(x, w, pos, heads, head_dim, rope_split=(32, 48, 48), eps=1e-6, theta=10000.0, wq=None):
    """One block with E4M3 projections (see the module docstring), in the
    same order as ``dit_block``: h = x + O(attn(RoPE(QKV(norm x)))),
    y = h + FFN(norm h)."""
    x = np.asarray(x, dtype=F64)
    if wq is None:
        wq = quantize_block_weights(w)
    A = heads * head_dim
    n = x.shape[0]
    xn = rms_norm(x, w["g_attn"], eps)
    qa, sa = quantize_rows(xn.astype(F32))
    qkv = linear_fp8(qa, sa, *wq["w_qkv"], w["b_qkv"])
    q = apply_rope(qkv[:, :A].reshape(n, heads, head_dim), pos, rope_split, theta)
    k = apply_rope(qkv[:, A:2 * A].reshape(n, heads, head_dim), pos, rope_split, theta)
    v = qkv[:, 2 * A:].reshape(n, heads, head_dim)
    o = attention(q, k, v).reshape(n, A)
    qo, so = quantize_rows(bf16_round(o).astype(F32))
    h = x + linear_fp8(qo, so, *wq["w_o"], w["b_o"])
    hn = rms_norm(h, w["g_ffn"], eps)
    qh, sh = quantize_rows(hn.astype(F32))
    u = gelu_tanh(linear_fp8(qh, sh, *wq["w_1"], w["b_1"]))
    qu, su = quantize_rows(bf16_round(u).astype(F32))
    return h + linear_fp8(qu, su, *wq["w_2"], w["b_2"])


def dit_block_fp8_rows(x, w, pos, heads, head_dim, rows, rope_split=(32, 48, 48), eps=1e-6, theta=10000.0,
                       wq=None):
    """``dit_block_fp8(x, ...)[rows]`` for the requested rows only.  Every
    row's normalized input is quantized (its own scale) and projected to keys
    and values; queries, the output projection and the FFN only for ``rows``.
    Each quantization depends on its own row alone, so the restriction is
    exact -- used to check full-size E4M3 blocks one row at a time."""
    x = np.asarray(x, dtype=F64)
    rows = np.asarray(rows, dtype=np.int64)
    if wq is None:
        wq = quantize_block_weights(w)
    A = heads * head_dim
    n, r = x.shape[0], len(rows)
    qa, sa = quantize_rows(rms_norm(x, w["g_attn"], eps).astype(F32))
    qw, sw = wq["w_qkv"]
    b = np.asarray(w["b_qkv"], dtype=F64)
    q = linear_fp8(qa[rows], sa[rows], qw[:A], sw[:A], b[:A]).reshape(r, heads, head_dim)
    k = linear_fp8(qa, sa, qw[A:2 * A], sw[A:2 * A], b[A:2 * A]).reshape(n, heads, head_dim)
    v = linear_fp8(qa, sa, qw[2 * A:], sw[2 * A:], b[2 * A:]).reshape(n, heads, head_dim)
    q = apply_rope(q, np.asarray(pos)[rows], rope_split, theta)
    k = apply_rope(k, pos, rope_split, theta)
    o = attention(q, k, v)
    qo, so = quantize_rows(bf16_round(o).astype(F32))
    h = x[rows] + linear_fp8(qo, so, *wq["w_o"], w["b_o"])
    qh, sh = quantize_rows(rms_norm(h, w["g_ffn"], eps).astype(F32))
    u = gelu_tanh(linear_fp8(qh, sh, *wq["w_1"], w["b_1"]))
    qu, su = quantize_rows(bf16_round(u).astype(F32))
    return h + linear_fp8(qu, su, *wq["w_2"], w["b_2"])
