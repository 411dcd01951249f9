"""Joint attention on score distributions that exercise the online softmax
(fsdit_attention; fp32 and bf16 paths) against the oracle's fp64 softmax:

* keys whose norm grows along the sequence, so the running row max rises by
  far more than the lazy-rescale threshold from one key tile to the next (the
  O and l rescale runs in most tiles);
* the same keys in falling order (the max sits in the first tile: no rescale);
* scores of a few hundred units (near one-hot rows: exponents far below the
  max must underflow cleanly to 0, never to inf or NaN);
* every valid score strongly negative, so the zero-filled key rows past the
  end of a ragged last tile would win every row if they were not masked;
* all keys equal: every row is the plain mean of V (closed form).

Bounds as for every attention test: rel-L2 <= 1e-5 (fp32), 1e-2 (bf16)."""

import numpy as np
import pytest
import torch

import oracle as O
from few_step_dit_b200 import api, build, lib as L

pytestmark = pytest.mark.gpu
DEV = "cuda"
HEADS = 2
A = HEADS * 128


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    L.load()
    yield
    torch.cuda.synchronize()
    api.device_error()


def _qkv(kind, n, g):
    q = torch.randn(n, A, generator=g)
    k = torch.randn(n, A, generator=g)
    v = torch.randn(n, A, generator=g)
    ramp = 1.0 + 6.0 * torch.arange(n, dtype=torch.float32)[:, None] / max(n - 1, 1)
    if kind == "growing":
        k = k * ramp
    elif kind == "falling":
        k = k * ramp.flip(0)
    elif kind == "huge":
        q, k = q * 8.0, k * 8.0
    elif kind == "negative":
        u = torch.randn(1, A, generator=g)
        q = 3.0 * u + 0.05 * q
        k = -3.0 * u + 0.05 * k
    elif kind == "equal_keys":
        k = k[:1].expand(n, A).clone()
    return torch.cat([q, k, v], dim=1)


def _oracle(qkv64, n):
    q = qkv64[:, :A].reshape(n, HEADS, 128)
    k = qkv64[:, A:2 * A].reshape(n, HEADS, 128)
    v = qkv64[:, 2 * A:].reshape(n, HEADS, 128)
    return O.attention(q, k, v)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("n", [1000, 300])
@pytest.mark.parametrize("kind", ["growing", "falling", "huge", "negative", "equal_keys"])
def test_attention_score_distributions(kind, n, dtype):
    g = torch.Generator().manual_seed(11)
    qkv = _qkv(kind, n, g).to(dtype)
    dims = api.make_dims(A, HEADS, 512, dtype)
    out = api.attention(dims, qkv.to(DEV))
    torch.cuda.synchronize()
    got = out.double().cpu().numpy()
    assert np.isfinite(got).all()
    qkv64 = qkv.double().numpy()
    ref = _oracle(qkv64, n)
    bound = 1e-5 if dtype == torch.float32 else 1e-2
    err = O.rel_l2(got, ref)
    assert err < bound, err
    if kind == "equal_keys":
        mean_v = qkv64[:, 2 * A:].mean(axis=0, keepdims=True)
        assert O.rel_l2(got, np.broadcast_to(mean_v, got.shape)) < bound
