"""Per-kernel parity of the CUDA path (through the C ABI) against the oracle.

Index work is compared bit-exactly; floating point within the bounds stated
next to each test (fp32: relative L2 1e-5; bf16 GEMM operands: relative L2
1e-2, the block/denoise bound).
"""

import numpy as np
import pytest
import torch

import oracle as O
from few_step_dit_b200 import api, build, lib as L

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    L.load()
    yield
    torch.cuda.synchronize()
    api.device_error()


def _t(a, dtype=torch.float32):
    return torch.as_tensor(np.ascontiguousarray(a)).to(DEV, dtype)


def _np(t):
    return t.detach().to("cpu", torch.float64).numpy()


def _rng(seed):
    g = torch.Generator().manual_seed(seed)
    return g


# ---------------------------------------------------------------- index maps


@pytest.mark.parametrize("grid", [(2, 9, 10), (6, 34, 60), (12, 34, 60), (6, 17, 30), (1, 1, 1),
                                  (3, 7, 5), (1, 2, 2), (4, 1, 9)])
def test_keep_map_bit_exact(grid):
    k_ref, n_ref = O.keep_map(*grid)
    k, n = api.keep_map(*grid)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(k.cpu().numpy(), k_ref)
    np.testing.assert_array_equal(n.cpu().numpy(), n_ref)


@pytest.mark.parametrize("grid,n_other,hidden", [((2, 9, 10), 24, 256), ((6, 34, 60), 320, 5376),
                                                 ((1, 3, 3), 0, 64)])
def test_gather_bit_exact(grid, n_other, hidden):
    T, H, W = grid
    V = T * H * W
    g = _rng(1)
    x = torch.randn(V + n_other, hidden, generator=g)
    pos = torch.randint(0, 50, (V + n_other, 3), generator=g, dtype=torch.int32)
    keep_idx, near_idx = O.keep_map(T, H, W)
    k_dev, _ = api.keep_map(T, H, W)
    xc, posc = api.gather_rows(x.to(DEV), pos.to(DEV), k_dev, V)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(xc.cpu().numpy(), O.gather_rows(x.numpy(), keep_idx, V))
    np.testing.assert_array_equal(posc.cpu().numpy(), O.gather_rows(pos.numpy(), keep_idx, V))


@pytest.mark.parametrize("in_place", [False, True])
@pytest.mark.parametrize("grid,n_other,hidden", [((2, 9, 10), 24, 256), ((6, 34, 60), 320, 5376)])
def test_broadcast_residual(grid, n_other, hidden, in_place):
    T, H, W = grid
    V = T * H * W
    g = _rng(2)
    keep_idx, near_idx = O.keep_map(T, H, W)
    n_c = len(keep_idx) + n_other
    x = torch.randn(V + n_other, hidden, generator=g)
    yc = torch.randn(n_c, hidden, generator=g)
    ref = O.broadcast_residual(x.numpy(), yc.numpy(), keep_idx, near_idx, V)
    k_dev, n_dev = api.keep_map(T, H, W)
    xd = x.to(DEV)
    out = api.broadcast_residual(xd, yc.to(DEV), k_dev, n_dev, grid, out=xd if in_place else None)
    torch.cuda.synchronize()
    got = out.cpu().numpy()
    kept = np.zeros(V, bool)
    kept[keep_idx] = True
    # kept grid rows and non-grid rows are copies: bit-exact
    np.testing.assert_array_equal(got[:V][kept], ref[:V][kept].astype(np.float32))
    np.testing.assert_array_equal(got[V:], ref[V:].astype(np.float32))
    # dropped rows: x + (y - x_k) in fp32, two roundings from the fp64 value
    d = ~kept
    np.testing.assert_allclose(got[:V][d], ref[:V][d], rtol=0, atol=4 * np.finfo(np.float32).eps * 8)


# ---------------------------------------------------------------- RMSNorm


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("rows,hidden", [(7, 256), (300, 5376), (1, 64)])
def test_rmsnorm_cast(dtype, rows, hidden):
    g = _rng(3)
    x = torch.randn(rows, hidden, generator=g) * 3
    gain = (1 + 0.02 * torch.randn(hidden, generator=g)).to(dtype)
    xn = api.rmsnorm_cast(x.to(DEV), gain.to(DEV))
    ref = O.rms_norm(x.numpy(), gain.double().numpy(), 1e-6)
    tol = 1e-6 if dtype == torch.float32 else 4e-3
    assert O.rel_l2(_np(xn), ref) < tol


# ---------------------------------------------------------------- projections


def _ref_linear(a, w, b, epi, resid=None, pos=None, hidden=None):
    y = O.linear(a, w, b)
    if epi == L.EPI_GELU:
        y = O.gelu_tanh(y)
    elif epi == L.EPI_RESIDUAL:
        y = resid + y
    elif epi == L.EPI_QKV_ROPE:
        M = y.shape[0]
        nh = hidden // 128
        q = O.apply_rope(y[:, :hidden].reshape(M, nh, 128), pos).reshape(M, hidden)
        k = O.apply_rope(y[:, hidden:2 * hidden].reshape(M, nh, 128), pos).reshape(M, hidden)
        y = np.concatenate([q, k, y[:, 2 * hidden:]], axis=1)
    return y


LIN_CASES = [
    # (M, N, K, epilogue)
    (300, 512, 256, L.EPI_BIAS),
    (128, 256, 64, L.EPI_BIAS),
    (1, 256, 64, L.EPI_BIAS),
    (257, 768, 256, L.EPI_QKV_ROPE),
    (200, 512, 256, L.EPI_GELU),
    (200, 256, 512, L.EPI_RESIDUAL),
    (77, 256, 520, L.EPI_BIAS_F32),
    # 256 x 256 pair tiles: the second column tile's upper half (cols 384..511)
    # lies wholly past N, K = 136 ends in a partial 64-wide step
    (513, 352, 136, L.EPI_BIAS),
    # 11 x 8 = 88 pair tiles, more than the CTA pairs resident on a B200, so
    # pairs run several tiles and reuse both accumulator buffers
    (2600, 2048, 256, L.EPI_GELU),
    (3668, 5376, 5376, L.EPI_RESIDUAL),
]


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("M,N,K,epi", LIN_CASES)
def test_linear(dtype, M, N, K, epi):
    if dtype == torch.float32 and M * N * K > 3e9:
        pytest.skip("exact-fp32 path is exercised at the small sizes")
    g = _rng(4)
    hidden = N // 3 if epi == L.EPI_QKV_ROPE else 256
    dims = api.make_dims(hidden, hidden // 128, 512, dtype)
    a = torch.randn(M, K, generator=g).to(dtype)
    w = (0.05 * torch.randn(N, K, generator=g)).to(dtype)
    b = (0.05 * torch.randn(N, generator=g)).to(dtype)
    resid = torch.randn(M, N, generator=g) if epi == L.EPI_RESIDUAL else None
    pos = torch.randint(0, 40, (M, 3), generator=g, dtype=torch.int32) if epi == L.EPI_QKV_ROPE else None
    out = api.linear(dims, a.to(DEV), w.to(DEV), b.to(DEV), epi,
                     resid=resid.to(DEV) if resid is not None else None,
                     pos=pos.to(DEV) if pos is not None else None)
    torch.cuda.synchronize()
    ref = _ref_linear(a.double().numpy(), w.double().numpy(), b.double().numpy(), epi,
                      resid.double().numpy() if resid is not None else None,
                      pos.numpy() if pos is not None else None, hidden)
    err = O.rel_l2(_np(out), ref)
    if dtype == torch.float32:
        assert err < 1e-5, err
    else:
        # fp32 accumulation of exact bf16 products; bf16 outputs round once (2^-9)
        bound = 1e-4 if out.dtype == torch.float32 else 5e-3
        assert err < bound, err


@pytest.mark.parametrize("split", [(34, 46, 48), (30, 50, 48), (32, 48, 48)])
def test_linear_rope_chunks_with_odd_pair_boundaries(split):
    # rope_split widths whose pair counts are odd put an axis boundary between
    # the two pairs one lane rotates in the coalesced epilogue
    g = _rng(12)
    M, A, K = 300, 256, 256
    dims = api.make_dims(A, A // 128, 512, torch.bfloat16, rope_split=split)
    a = torch.randn(M, K, generator=g).bfloat16()
    w = (0.05 * torch.randn(3 * A, K, generator=g)).bfloat16()
    b = (0.05 * torch.randn(3 * A, generator=g)).bfloat16()
    pos = torch.randint(0, 40, (M, 3), generator=g, dtype=torch.int32)
    out = api.linear(dims, a.to(DEV), w.to(DEV), b.to(DEV), L.EPI_QKV_ROPE, pos=pos.to(DEV))
    torch.cuda.synchronize()
    y = O.linear(a.double().numpy(), w.double().numpy(), b.double().numpy())
    q = O.apply_rope(y[:, :A].reshape(M, A // 128, 128), pos.numpy(), split).reshape(M, A)
    k = O.apply_rope(y[:, A:2 * A].reshape(M, A // 128, 128), pos.numpy(), split).reshape(M, A)
    ref = np.concatenate([q, k, y[:, 2 * A:]], axis=1)
    assert O.rel_l2(_np(out), ref) < 5e-3
    # the same split with the default one differs: the split reached the kernel
    if split != (32, 48, 48):
        ref0 = np.concatenate([O.apply_rope(y[:, :A].reshape(M, A // 128, 128), pos.numpy()).reshape(M, A),
                               O.apply_rope(y[:, A:2 * A].reshape(M, A // 128, 128), pos.numpy()).reshape(M, A),
                               y[:, 2 * A:]], axis=1)
        assert O.rel_l2(_np(out), ref0) > 1e-2


# ---------------------------------------------------------------- attention


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("n,heads", [(204, 2), (84, 2), (1, 1), (129, 3), (1000, 2)])
def test_attention(dtype, n, heads):
    g = _rng(5)
    hidden = heads * 128
    dims = api.make_dims(hidden, heads, 512, dtype)
    qkv = (torch.randn(n, 3 * hidden, generator=g) * 1.5).to(dtype)
    out = api.attention(dims, qkv.to(DEV))
    torch.cuda.synchronize()
    q = qkv[:, :hidden].double().numpy().reshape(n, heads, 128)
    k = qkv[:, hidden:2 * hidden].double().numpy().reshape(n, heads, 128)
    v = qkv[:, 2 * hidden:].double().numpy().reshape(n, heads, 128)
    ref = O.attention(q, k, v)
    err = O.rel_l2(_np(out), ref)
    assert err < (1e-5 if dtype == torch.float32 else 1e-2), err


@pytest.mark.parametrize("n,heads,check_heads", [(3668, 56, (0, 17, 55)), (12560, 56, (3, 42))])
def test_attention_full_size_sampled_heads(n, heads, check_heads):
    # the Flash sequence lengths (compressed and full) at the 56-head width;
    # the oracle runs on a few heads, the kernel on all of them
    g = _rng(8)
    A = heads * 128
    dims = api.make_dims(5376, heads, 14336, torch.bfloat16)
    qkv = (torch.randn(n, 3 * A, generator=g) * 1.5).bfloat16()
    out = api.attention(dims, qkv.to(DEV))
    torch.cuda.synchronize()
    got = out.float().cpu().numpy()
    for h in check_heads:
        q = qkv[:, h * 128:(h + 1) * 128].double().numpy()[:, None, :]
        k = qkv[:, A + h * 128:A + (h + 1) * 128].double().numpy()[:, None, :]
        v = qkv[:, 2 * A + h * 128:2 * A + (h + 1) * 128].double().numpy()[:, None, :]
        ref = O.attention(q, k, v)
        err = O.rel_l2(got[:, h * 128:(h + 1) * 128], ref)
        assert err < 1e-2, (h, err)


# ---------------------------------------------------------------- Euler


def test_euler_step_per_modality_clocks():
    g = _rng(6)
    n, wdt = 300, 24
    x = torch.randn(n, wdt, generator=g)
    v = torch.randn(n, wdt, generator=g)
    mod = torch.randint(0, 4, (n,), generator=g, dtype=torch.uint8)
    mask = torch.randint(0, 2, (n,), generator=g, dtype=torch.uint8)
    tc, tn = [0.0, 0.2, 0.5, 0.0], [0.0, 0.0769, 0.25, 0.0]
    xd = x.to(DEV)
    api.euler_step(xd, v.to(DEV), mod.to(DEV), mask.to(DEV), tc, tn)
    torch.cuda.synchronize()
    ref = O.euler_step(x.numpy(), v.numpy(), mod.numpy(), mask.numpy(), tc, tn)
    np.testing.assert_allclose(xd.cpu().numpy(), ref, rtol=1e-6, atol=1e-6)
    np.testing.assert_array_equal(xd.cpu().numpy()[mask.numpy() == 0], x.numpy()[mask.numpy() == 0])
