"""The projections' tail cut (fsdit_linear_ws / fsdit_linear_fp8_ws) against
the oracle, on shapes whose last wave of 256 x 256 pair tiles leaves most CTA
pairs idle, so those tiles run as K-split units whose fp32 parts the last unit
sums: bf16 rel-L2 <= 1e-4 (fp32 out) / 5e-3 (bf16 out) as for fsdit_linear;
E4M3 on identical quantized operands 1e-5 / 5e-3.  With and without the cut
the results agree within 1e-5 (only the grouping of the K sum differs), the
cut is deterministic (two runs bit-identical), the residual epilogue works in
place, and where the plan cuts an fp32-output GEMM the two results differ in
the last bits -- evidence that the cut path ran."""

import numpy as np
import pytest
import torch

import oracle as O
from oracle import fp8 as Q
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


@pytest.fixture(scope="module")
def scratch():
    return api.gemm_scratch(DEV)


def _cuts(M, N, K, k_elems_per_step):
    """Whether the host plan cuts the tail (same rule as the launcher; the
    pair count assumes every SM pair holds one CTA pair)."""
    pairs = torch.cuda.get_device_properties(0).multi_processor_count // 2
    tiles = -(-M // 256) * -(-N // 256)
    kb = -(-K // k_elems_per_step)
    R = tiles % pairs
    if R == 0 or kb < 32:
        return False
    S = min(pairs // R, kb // 12, 8)
    return R <= 64 and S >= 2


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


TAIL_CASES = [
    (3668, 5376, 7168, L.EPI_RESIDUAL),   # 315 tiles: 19 in the last wave, cut in 3
    (256, 5376, 5120, L.EPI_BIAS_F32),    # 21 tiles, all in one partial wave, cut in 3
    (300, 768, 6144, L.EPI_QKV_ROPE),     # 6 tiles, cut in 4 (48 K steps)
    (1000, 2048, 4096, L.EPI_GELU),       # 32 tiles, cut in 2
    (700, 32, 12288, L.EPI_BIAS),         # 3 tiles, N far below the tile width, cut in 8
    (300, 512, 2048, L.EPI_BIAS_F32),     # 16 K steps: too short to cut (the plain path)
]


@pytest.mark.parametrize("M,N,K,epi", TAIL_CASES)
def test_linear_tail_cut_matches_oracle(scratch, M, N, K, epi):
    g = torch.Generator().manual_seed(6)
    A = N // 3 if epi == L.EPI_QKV_ROPE else 256
    dims = api.make_dims(A, A // 128, 512, L.BF16)
    a = torch.randn(M, K, generator=g).bfloat16()
    w = (0.05 * torch.randn(N, K, generator=g)).bfloat16()
    b = (0.05 * torch.randn(N, generator=g)).bfloat16()
    resid = torch.randn(M, N, generator=g) if epi == L.EPI_RESIDUAL else None
    pos = torch.randint(0, 40, (M, 3), generator=g, dtype=torch.int32) if epi == L.EPI_QKV_ROPE else None
    args = (dims, a.to(DEV), w.to(DEV), b.to(DEV), epi)
    kw = dict(resid=resid.to(DEV) if resid is not None else None, pos=pos.to(DEV) if pos is not None else None)
    cut = api.linear(*args, scratch=scratch, **kw)
    cut2 = api.linear(*args, scratch=scratch, **kw)
    whole = api.linear(*args, **kw)
    torch.cuda.synchronize()
    assert torch.equal(cut, cut2)                        # the part order is fixed
    y = O.linear(a.double().numpy(), w.double().numpy(), b.double().numpy())
    ref = _ref_epilogue(y, epi, resid.double().numpy() if resid is not None else None,
                        pos.numpy() if pos is not None else None, A)
    got = cut.double().cpu().numpy()
    bound = 1e-4 if cut.dtype == torch.float32 else 5e-3
    assert O.rel_l2(got, ref) < bound
    if cut.dtype == torch.float32:
        # the tensor core rounds its fp32 sums along K; cutting K regroups
        # them (measured 1.3e-6 at K = 7168)
        assert O.rel_l2(got, whole.double().cpu().numpy()) < 1e-5
        if _cuts(M, N, K, 128):
            assert not torch.equal(cut, whole)           # the K sum ran in parts


def test_linear_tail_cut_residual_in_place(scratch):
    # out == resid: every element is read and written once, by the unit that
    # completes its tile region
    g = torch.Generator().manual_seed(7)
    M, N, K = 200, 256, 12288                             # one tile, cut in 8
    dims = api.make_dims(256, 2, 512, L.BF16)
    a = torch.randn(M, K, generator=g).bfloat16()
    w = (0.02 * torch.randn(N, K, generator=g)).bfloat16()
    b = (0.05 * torch.randn(N, generator=g)).bfloat16()
    x = torch.randn(M, N, generator=g)
    xd = x.to(DEV)
    api.linear(dims, a.to(DEV), w.to(DEV), b.to(DEV), L.EPI_RESIDUAL, resid=xd, out=xd, scratch=scratch)
    torch.cuda.synchronize()
    ref = x.double().numpy() + O.linear(a.double().numpy(), w.double().numpy(), b.double().numpy())
    assert O.rel_l2(xd.double().cpu().numpy(), ref) < 1e-4


@pytest.mark.parametrize("M,N,K,epi", [(1000, 2048, 8192, L.EPI_RESIDUAL), (300, 512, 8192, L.EPI_BIAS),
                                       (300, 768, 8192, L.EPI_QKV_ROPE)])
def test_fp8_tail_cut_on_identical_quantized_operands(scratch, M, N, K, epi):
    rng = np.random.default_rng(8)
    a = (rng.standard_normal((M, K)) * rng.uniform(0.1, 10, (M, 1))).astype(np.float32)
    w = (rng.standard_normal((N, K)) * 0.05).astype(np.float32)
    qa, sa = Q.quantize_rows(a)
    qw, sw = Q.quantize_rows(w)
    b = torch.tensor(rng.standard_normal(N) * 0.05).bfloat16()
    resid = rng.standard_normal((M, N)).astype(np.float32) if epi == L.EPI_RESIDUAL else None
    pos = rng.integers(0, 40, (M, 3)).astype(np.int32) if epi == L.EPI_QKV_ROPE else None
    codes = lambda v: torch.tensor(v).to(torch.float8_e4m3fn).view(torch.uint8).to(DEV)  # noqa: E731
    A = N // 3 if epi == L.EPI_QKV_ROPE else 256
    dims = api.make_dims(A, A // 128, 512, L.BF16, proj_fp8=True)
    out = api.linear_fp8(dims, codes(qa), torch.tensor(sa, dtype=torch.float32).to(DEV), codes(qw),
                         torch.tensor(sw, dtype=torch.float32).to(DEV), b.to(DEV), epi,
                         resid=torch.tensor(resid).to(DEV) if resid is not None else None,
                         pos=torch.tensor(pos).to(DEV) if pos is not None else None, scratch=scratch)
    torch.cuda.synchronize()
    y = Q.linear_fp8(qa, sa, qw, sw, b.double().numpy())
    ref = _ref_epilogue(y, epi, resid.astype(np.float64) if resid is not None else None, pos, A)
    bound = 1e-5 if out.dtype == torch.float32 else 5e-3
    assert O.rel_l2(out.double().cpu().numpy(), ref) < bound
