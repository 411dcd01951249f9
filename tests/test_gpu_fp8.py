"""FP8 (E4M3) projections on the GPU against the oracle.

* Per-row quantization: scales and codes bit-exact.  Both sides take the
  scale s = amax / 448 in fp32 and the code of the exact quotient value / s
  (the oracle divides in float64; the kernel reads the side of the E4M3
  midpoint from the sign of an exact fused multiply-add), so every rounding
  decision, ties included, is the same.
* RMSNorm fused with quantization: the kernel's fp32 RMSNorm rounds a little
  differently from the fp64 oracle rounded to fp32, so at most 1e-3 of the
  codes may move, by one E4M3 step.
* E4M3 GEMM on identical quantized operands: fp32 outputs rel-L2 <= 1e-5,
  bf16 outputs <= 5e-3 (one bf16 rounding, 2^-9).
* Whole block with E4M3 projections: rel-L2 <= 3e-2 on the output and 5e-2 on
  the update y - x.  Derivation: the GPU attention runs in bf16 and differs
  from the fp64 oracle by ~2e-3; near an E4M3 rounding boundary such a
  difference moves a code by a whole step (12.5%), and a CPU simulation of
  that (the oracle's FP8 block with 2e-3 to 5e-3 relative noise on the
  attention output) moves the update by 2.3-2.8% and the output by 1.2-1.4%;
  the bounds are about twice that.
"""

import numpy as np
import pytest
import torch

import oracle as O
from oracle import fp8 as Q
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


def _codes_to_values(q):
    return q.cpu().view(torch.float8_e4m3fn).to(torch.float64).numpy()


def _values_to_codes(v):
    return torch.tensor(np.asarray(v), dtype=torch.float64).to(torch.float8_e4m3fn).view(torch.uint8).to(DEV)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("rows,cols", [(7, 256), (300, 5376), (33, 14336), (1, 16), (4, 4096), (3, 16400)])
def test_quantize_rows_matches_definition(dtype, rows, cols):
    g = torch.Generator().manual_seed(1)
    a = torch.randn(rows, cols, generator=g) * torch.exp(torch.randn(rows, 1, generator=g) * 2)
    a[0, :5] = torch.tensor([300.0, -1e-6, 0.0, 7e-3, -2.5])  # wide dynamic range in one row
    if rows > 3:
        a[3] = 0.0                                              # all-zero row: scale 1, codes 0
    a = a.to(dtype)
    q, s = api.quantize_rows(a.to(DEV))
    torch.cuda.synchronize()
    ref_q, ref_s = Q.quantize_rows(a.float().numpy())
    np.testing.assert_array_equal(s.cpu().double().numpy(), ref_s)
    np.testing.assert_array_equal(_codes_to_values(q), ref_q)


@pytest.mark.parametrize("amax", [1.75, 1.3125, 3.0, 0.7])
def test_quantize_rows_ties_and_near_ties_of_bf16_rows(amax):
    # bf16 rows whose largest magnitude is amax: for 1.75 or 1.3125 the scale
    # amax / 448 is a short binary number and many quotients land exactly on
    # E4M3 midpoints (ties to even); for the others they land within an ulp
    # of them, where multiplying by a rounded reciprocal would round every
    # such value of a row the same way
    g = torch.Generator().manual_seed(int(amax * 64))
    a = (torch.randn(64, 4096, generator=g) * 0.5).clamp(-amax, amax)
    a[:, 0] = amax
    a = a.bfloat16()
    q, s = api.quantize_rows(a.to(DEV))
    torch.cuda.synchronize()
    ref_q, ref_s = Q.quantize_rows(a.float().numpy())
    np.testing.assert_array_equal(s.cpu().double().numpy(), ref_s)
    np.testing.assert_array_equal(_codes_to_values(q), ref_q)


@pytest.mark.parametrize("rows,hidden", [(9, 256), (300, 5376)])
def test_rmsnorm_quant_matches_oracle(rows, hidden):
    g = torch.Generator().manual_seed(2)
    x = torch.randn(rows, hidden, generator=g) * 3
    gain = (1 + 0.02 * torch.randn(hidden, generator=g)).bfloat16()
    q, s = api.rmsnorm_quant(x.to(DEV), gain.to(DEV))
    torch.cuda.synchronize()
    ref_q, ref_s = Q.quantize_rows(O.rms_norm(x.double().numpy(), gain.double().numpy(), 1e-6).astype(np.float32))
    np.testing.assert_allclose(s.cpu().double().numpy(), ref_s, rtol=1e-6, atol=0)
    got = _codes_to_values(q)
    diff = got != ref_q
    assert diff.mean() <= 1e-3, diff.mean()
    # a moved code is at most one E4M3 step away (1/8 of the value, or the
    # subnormal step 2^-9)
    assert (np.abs(got[diff] - ref_q[diff]) <= np.abs(ref_q[diff]) / 8 + 2.0 ** -9).all()


def _ref_epilogue(y, epi, resid=None, pos=None, A=None):
    if epi == L.EPI_GELU:
        return O.gelu_tanh(y)
    if epi == L.EPI_RESIDUAL:
        return resid + y
    if epi == L.EPI_QKV_ROPE:
        M = y.shape[0]
        q = O.apply_rope(y[:, :A].reshape(M, A // 128, 128), pos).reshape(M, A)
        k = O.apply_rope(y[:, A:2 * A].reshape(M, A // 128, 128), pos).reshape(M, A)
        return np.concatenate([q, k, y[:, 2 * A:]], axis=1)
    return y


FP8_CASES = [
    (300, 512, 256, L.EPI_BIAS),
    (1, 256, 64, L.EPI_BIAS),
    (257, 768, 256, L.EPI_QKV_ROPE),
    (200, 512, 256, L.EPI_GELU),
    (200, 256, 512, L.EPI_RESIDUAL),
    (77, 256, 528, L.EPI_BIAS_F32),
    (513, 352, 144, L.EPI_BIAS),          # ragged last K step (144 = 128 + 16), half column tile past N
    (2600, 2048, 256, L.EPI_GELU),        # more pair tiles than resident CTA pairs
    (3668, 5376, 7168, L.EPI_RESIDUAL),   # O-projection of a compressed layer, full size
]


@pytest.mark.parametrize("M,N,K,epi", FP8_CASES)
def test_linear_fp8_on_identical_quantized_operands(M, N, K, epi):
    rng = np.random.default_rng(4)
    a = (rng.standard_normal((M, K)) * rng.uniform(0.1, 10, (M, 1))).astype(np.float32)
    w = (rng.standard_normal((N, K)) * 0.05).astype(np.float32)
    qa, sa = Q.quantize_rows(a)
    qw, sw = Q.quantize_rows(w)
    b = torch.tensor(rng.standard_normal(N) * 0.05).bfloat16()
    A = N // 3 if epi == L.EPI_QKV_ROPE else 256
    dims = api.make_dims(A, A // 128, 512, L.BF16, proj_fp8=True)
    resid = rng.standard_normal((M, N)).astype(np.float32) if epi == L.EPI_RESIDUAL else None
    pos = rng.integers(0, 40, (M, 3)).astype(np.int32) if epi == L.EPI_QKV_ROPE else None
    out = api.linear_fp8(dims, _values_to_codes(qa), torch.tensor(sa, dtype=torch.float32).to(DEV),
                         _values_to_codes(qw), torch.tensor(sw, dtype=torch.float32).to(DEV), b.to(DEV), epi,
                         resid=torch.tensor(resid).to(DEV) if resid is not None else None,
                         pos=torch.tensor(pos).to(DEV) if pos is not None else None)
    torch.cuda.synchronize()
    y = Q.linear_fp8(qa, sa, qw, sw, b.double().numpy())
    ref = _ref_epilogue(y, epi, resid.astype(np.float64) if resid is not None else None, pos, A)
    err = O.rel_l2(out.double().cpu().numpy(), ref)
    bound = 1e-5 if out.dtype == torch.float32 else 5e-3
    assert err < bound, err


def _fp8_block_case(w, compress):
    layers, _ = S.make_weights(w, n_layers=1)
    inp = S.make_inputs(w)
    tags = S.pack_tokens(w)
    seq = api.Sequence.from_workload(w, tags, DEV, compress=True)
    bw = api.BlockWeights(api.quantize_block_weights({k: v.to(DEV) for k, v in layers[0].items()}))
    x = inp["x"].float()
    out = api.block_forward(api.dims_of(w, proj_fp8=True), bw, seq, x.to(DEV), compress=compress)
    torch.cuda.synchronize()
    wn = S.to_numpy64(layers[0])
    xn = x.double().numpy()
    k, n = O.keep_map(*w.grid)
    if compress:
        # the compressed block: gather kept rows, FP8 block, nearest-kept broadcast
        sel = np.concatenate([k, np.arange(w.n_video, w.n_tokens)])
        yc = Q.dit_block_fp8(xn[sel], wn, tags["pos"][sel], w.heads, w.head_dim)
        ref = O.broadcast_residual(xn, yc, k, n, w.n_video)
    else:
        ref = Q.dit_block_fp8(xn, wn, tags["pos"], w.heads, w.head_dim)
    return out.double().cpu().numpy(), ref, xn


@pytest.mark.parametrize("compress", [True, False])
@pytest.mark.parametrize("grid", [(2, 9, 10), (3, 6, 7)])
def test_fp8_block_matches_fp8_oracle(grid, compress):
    w = S.scaled(S.WORKLOADS["flash_block_6x34x60"], hidden=256, heads=2, ffn=512, grid=grid, n_text=16, n_audio=8)
    got, ref, x = _fp8_block_case(w, compress)
    assert O.rel_l2(got, ref) < 3e-2
    assert O.rel_l2(got - x, ref - x) < 5e-2


@pytest.mark.parametrize("compress", [True, False])
def test_fp8_full_width_block_sampled_rows(compress):
    # the bench's E4M3 configuration at full size (6x34x60, hidden 5376, 56
    # heads, FFN 14336) on sampled rows the oracle's row-restricted E4M3
    # block computes one by one.  At full width the update is as large as the
    # output (|y - x| ~ |y|), so the output inherits the update's code-flip
    # bound (5e-2) instead of the small-width output bound
    w = S.WORKLOADS["flash_block_6x34x60"]
    layers, _ = S.make_weights(w, n_layers=1)
    inp = S.make_inputs(w)
    tags = S.pack_tokens(w)
    seq = api.Sequence.from_workload(w, tags, DEV, compress=True)
    bw = api.BlockWeights(api.quantize_block_weights({k: v.to(DEV) for k, v in layers[0].items()}))
    x = inp["x"].float()
    y = api.block_forward(api.dims_of(w, proj_fp8=True), bw, seq, x.to(DEV), compress=compress)
    torch.cuda.synchronize()
    V, N = w.n_video, w.n_tokens
    T, H, W = w.grid
    rows = np.unique(np.concatenate([[0, 1, W, W + 1, H * W - 1, V - 1, V, V + w.n_text - 1, N - 1],
                                     np.random.default_rng(13).integers(0, N, 24)]))
    got = y[torch.as_tensor(rows, device=DEV)].double().cpu().numpy()
    wn = S.to_numpy64(layers[0])
    xn = x.double().numpy()
    if compress:
        k, n = O.keep_map(*w.grid)
        ref = O.dit_block_compressed_rows(xn, wn, tags["pos"], w.heads, w.head_dim, k, n, V, rows,
                                          rows_fn=Q.dit_block_fp8_rows)
    else:
        ref = Q.dit_block_fp8_rows(xn, wn, tags["pos"], w.heads, w.head_dim, rows)
    upd = ref - xn[rows]
    assert float(np.linalg.norm(upd) / np.linalg.norm(ref)) > 0.5
    assert O.rel_l2(got, ref) < 5e-2
    assert O.rel_l2(got - xn[rows], upd) < 5e-2


def test_fp8_full_width_block_stays_within_e4m3_error_of_bf16_block():
    # full 6x34x60 width: the E4M3 block's update differs from the bf16 block's
    # by the quantization error scale (~5% per GEMM, see the oracle pins), not more
    w = S.WORKLOADS["flash_block_6x34x60"]
    layers, _ = S.make_weights(w, device=DEV, n_layers=1)
    inp = S.make_inputs(w, device=DEV)
    seq = api.Sequence.from_workload(w, S.pack_tokens(w), DEV, compress=True)
    x = inp["x"].float()
    y16 = api.block_forward(api.dims_of(w), api.BlockWeights(layers[0]), seq, x)
    y8 = api.block_forward(api.dims_of(w, proj_fp8=True), api.BlockWeights(api.quantize_block_weights(layers[0])),
                           seq, x)
    torch.cuda.synchronize()
    d16, d8 = (y16 - x).double(), (y8 - x).double()
    rel = float((d8 - d16).norm() / d16.norm())
    assert torch.isfinite(y8).all() and 1e-3 < rel < 0.1, rel


def test_fp8_sampler_matches_fp8_oracle():
    # three evaluations of a 6-layer stack (two full, three compressed, one
    # full) with E4M3 projections, against the oracle sampler running the
    # oracle's E4M3 block; the per-block discrepancy above (code flips next to
    # bf16 attention) feeds the velocities, so the bounds are the block's
    w = S.scaled(S.WORKLOADS["flash_backbone_6x34x60"], hidden=256, heads=2, ffn=512, grid=(2, 9, 10),
                 n_text=16, n_audio=8, n_layers=6, compress=(0, 1, 1, 1, 0, 0))
    layers, io = S.make_weights(w)
    inp = S.make_inputs(w)
    tags = S.pack_tokens(w)
    seq = api.Sequence.from_workload(w, tags, DEV)
    bb = api.Backbone(api.dims_of(w, proj_fp8=True),
                      [api.BlockWeights(api.quantize_block_weights({k: v.to(DEV) for k, v in l.items()}))
                       for l in layers],
                      api.IOWeights({k: v.to(DEV) for k, v in io.items()}), w.compress)
    vl, al = inp["video_lat"].to(DEV).clone(), inp["audio_lat"].to(DEV).clone()
    bb.sample(seq, w.video_clock, w.audio_clock, vl, inp["text_emb"].to(DEV), al)
    torch.cuda.synchronize()
    tok = dict(tags)
    tok["keep_idx"], tok["near_idx"] = O.keep_map(*w.grid)
    v0, a0 = inp["video_lat"].double().numpy(), inp["audio_lat"].double().numpy()
    rv, ra = O.flow_sample([S.to_numpy64(l) for l in layers], w.compress, S.to_numpy64(io), tok, w.video_clock,
                           w.audio_clock, v0, inp["text_emb"].double().numpy(), inp["audio_lat"].double().numpy(),
                           w.heads, w.head_dim, block_fn=Q.dit_block_fp8)
    gv, ga = vl.double().cpu().numpy(), al.double().cpu().numpy()
    assert O.rel_l2(gv, rv) < 3e-2 and O.rel_l2(ga, ra) < 3e-2
    assert O.rel_l2(gv - v0, rv - v0) < 5e-2 and O.rel_l2(ga - a0, ra - a0) < 5e-2
