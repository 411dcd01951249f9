"""The CTA-pair attention kernel (clusters of two CTAs, 256 queries per
cluster, Q and P in tensor memory) against the oracle's fp64 softmax and
against the single-CTA kernel, on ragged and full-size sequences and on the
score distributions that drive the online softmax ([tokendh] backbone
section: one joint sequence of text, video and audio tokens, no mask).

The kernel choice is a process-wide threshold; this module sets it to one
row (every bf16 attention runs on the pair kernel) and restores it after.
Bounds: rel-L2 <= 1e-2 against the oracle (bf16 operands, as for every bf16
attention test); against the single-CTA kernel <= 2e-3 (both round the same
fp32 softmax to bf16 P and output; only the order of the exponentials'
partial sums differs).
"""

import numpy as np
import pytest
import torch

import oracle as O
from few_step_dit_b200 import api, build, lib as L
from few_step_dit_b200 import synthetic as S

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _pair_everywhere():
    build.build()
    fs = L.load()
    old = fs.fsdit_attention_pair_min_rows()
    assert fs.fsdit_set_attention_pair_min_rows(1) == 0
    yield fs
    torch.cuda.synchronize()
    fs.fsdit_set_attention_pair_min_rows(old)
    api.device_error()


def _single_cta(fs, dims, qkv):
    old = fs.fsdit_attention_pair_min_rows()
    fs.fsdit_set_attention_pair_min_rows(1 << 30)
    try:
        out = api.attention(dims, qkv)
        torch.cuda.synchronize()
    finally:
        fs.fsdit_set_attention_pair_min_rows(old)
    return out


def _heads_ref(qkv, A, heads):
    n = qkv.shape[0]
    q = qkv[:, :A].double().numpy().reshape(n, heads, 128)
    k = qkv[:, A:2 * A].double().numpy().reshape(n, heads, 128)
    v = qkv[:, 2 * A:].double().numpy().reshape(n, heads, 128)
    return O.attention(q, k, v)


def test_threshold_knob_rejects_nonpositive(_pair_everywhere):
    fs = _pair_everywhere
    assert fs.fsdit_set_attention_pair_min_rows(0) == -2
    assert fs.fsdit_attention_pair_min_rows() == 1


@pytest.mark.parametrize("n", [1, 64, 128, 129, 300, 511, 512, 513, 1000, 1300, 3668])
def test_pair_attention_matches_oracle_and_single_cta_kernel(_pair_everywhere, n):
    # one cluster covers 256 queries (a 128-row tile per CTA); 300, 513 and
    # 1300 leave ragged clusters, 129 a ragged key block split across the pair
    heads = 2
    A = heads * 128
    g = torch.Generator().manual_seed(n)
    qkv = (torch.randn(n, 3 * A, generator=g) * 1.5).bfloat16()
    dims = api.make_dims(A, heads, 512, torch.bfloat16)
    out = api.attention(dims, qkv.to(DEV))
    torch.cuda.synchronize()
    got = out.double().cpu().numpy()
    assert np.isfinite(got).all()
    assert O.rel_l2(got, _heads_ref(qkv, A, heads)) < 1e-2
    single = _single_cta(_pair_everywhere, dims, qkv.to(DEV)).double().cpu().numpy()
    assert O.rel_l2(got, single) < 2e-3


def _stress_qkv(kind, n, A, g):
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


@pytest.mark.parametrize("n", [1000, 300])
@pytest.mark.parametrize("kind", ["growing", "falling", "huge", "negative", "equal_keys"])
def test_pair_attention_score_distributions(kind, n):
    # growing key norms (the lazy O rescale runs in most key blocks), falling
    # ones (no rescale), near one-hot rows, all valid scores strongly negative
    # (masked key rows past n must not win), equal keys (closed form: mean of V)
    heads = 2
    A = heads * 128
    g = torch.Generator().manual_seed(11)
    qkv = _stress_qkv(kind, n, A, g).bfloat16()
    dims = api.make_dims(A, heads, 512, torch.bfloat16)
    out = api.attention(dims, qkv.to(DEV))
    torch.cuda.synchronize()
    got = out.double().cpu().numpy()
    assert np.isfinite(got).all()
    ref = _heads_ref(qkv, A, heads)
    assert O.rel_l2(got, ref) < 1e-2
    if kind == "equal_keys":
        mean_v = qkv[:, 2 * A:].double().numpy().mean(axis=0, keepdims=True)
        assert O.rel_l2(got, np.broadcast_to(mean_v, got.shape)) < 1e-2


@pytest.mark.parametrize("n,check_heads", [(12560, (3, 42)), (24800, (7,))])
def test_pair_attention_full_size_sampled_heads(_pair_everywhere, n, check_heads):
    # the full-resolution Flash sequence (6x34x60 + 256 + 64) and the
    # 12x34x60 sweep grid at the 56-head width; the oracle runs on a few heads
    heads = 56
    A = heads * 128
    g = torch.Generator().manual_seed(8)
    qkv = (torch.randn(n, 3 * A, generator=g) * 1.5).bfloat16()
    dims = api.make_dims(5376, heads, 14336, torch.bfloat16)
    qd = qkv.to(DEV)
    out = api.attention(dims, qd)
    torch.cuda.synchronize()
    got = out.float().cpu().numpy()
    for h in check_heads:
        sl = slice(h * 128, (h + 1) * 128)
        q = qkv[:, h * 128:(h + 1) * 128].double().numpy()[:, None, :]
        k = qkv[:, A + h * 128:A + (h + 1) * 128].double().numpy()[:, None, :]
        v = qkv[:, 2 * A + h * 128:2 * A + (h + 1) * 128].double().numpy()[:, None, :]
        assert O.rel_l2(got[:, sl], O.attention(q, k, v)) < 1e-2, h
    single = _single_cta(_pair_everywhere, dims, qd).float().cpu().numpy()
    assert O.rel_l2(got, single) < 2e-3


def test_sampler_with_pair_attention_matches_oracle():
    # the 3-evaluation sampler with every attention on the pair kernel
    w = S.scaled(S.WORKLOADS["flash_backbone_6x34x60"], hidden=256, heads=2, ffn=512, grid=(2, 9, 10), n_text=16,
                 n_audio=8, n_layers=6, compress=(0, 1, 1, 1, 0, 0))
    layers, io = S.make_weights(w)
    inp = S.make_inputs(w)
    tags = S.pack_tokens(w)
    seq = api.Sequence.from_workload(w, tags, DEV)
    bb = api.Backbone(api.dims_of(w), [api.BlockWeights({k: v.to(DEV) for k, v in l.items()}) for l in layers],
                      api.IOWeights({k: v.to(DEV) for k, v in io.items()}), w.compress)
    vl, al = inp["video_lat"].to(DEV).clone(), inp["audio_lat"].to(DEV).clone()
    bb.sample(seq, w.video_clock, w.audio_clock, vl, inp["text_emb"].to(DEV), al)
    torch.cuda.synchronize()
    tok = dict(tags)
    tok["keep_idx"], tok["near_idx"] = O.keep_map(*w.grid)
    rv, ra = O.flow_sample([S.to_numpy64(l) for l in layers], w.compress, S.to_numpy64(io), tok, w.video_clock,
                           w.audio_clock, inp["video_lat"].double().numpy(), inp["text_emb"].double().numpy(),
                           inp["audio_lat"].double().numpy(), w.heads, w.head_dim)
    v0 = inp["video_lat"].double().numpy()
    got = vl.double().cpu().numpy()
    assert O.rel_l2(got, rv) < 1e-2
    assert O.rel_l2(got - v0, rv - v0) < 1e-2
    assert O.rel_l2(al.double().cpu().numpy(), ra) < 1e-2
