"""dit_block_forward_noalloc: the block forward for callers that cannot call
cudaMalloc (for example a host application whose device memory belongs to its
own pool allocator), with its scratch in a static device array inside the
library.  Its output must match dit_block_forward (which takes a workspace
from the caller) within the tests' usual bounds, on two calls in a row, and
the oracle on the tiny fp32 block; the largest blocks its header lists are
accepted and one row more is refused.

This file is collected last so that a run stopping at the first failure has
already run every other test; it also passes alone in a fresh process.
"""

import ctypes as C

import pytest
import torch

import oracle as O
from few_step_dit_b200 import api, build, lib as L
from few_step_dit_b200 import synthetic as S

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def fs():
    build.build()
    return L.load()


def _case(w):
    layers, _ = S.make_weights(w, n_layers=1)
    inp = S.make_inputs(w)
    tags = S.pack_tokens(w)
    seq = api.Sequence.from_workload(w, tags, DEV, compress=True)
    bw = api.BlockWeights({k: v.to(DEV) for k, v in layers[0].items()})
    return api.dims_of(w), bw, seq, inp["x"].float().to(DEV)


@pytest.mark.parametrize("name,kw,bound", [
    ("tiny_block_f32", {}, 1e-5),
    ("flash_block_6x34x60", dict(hidden=256, heads=2, ffn=512, grid=(3, 6, 7), n_text=16, n_audio=8), 1e-2),
])
@pytest.mark.parametrize("compress", [True, False])
def test_noalloc_matches_workspace_entry_point_twice(fs, name, kw, bound, compress):
    w = S.scaled(S.WORKLOADS[name], **kw)
    dims, bw, seq, x = _case(w)
    tok = seq.struct if compress else seq.struct_full
    ref = api.block_forward(dims, bw, seq, x, compress=compress)
    stream = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    for _ in range(2):
        out = torch.full_like(x, float("nan"))
        st = fs.dit_block_forward_noalloc(C.byref(dims), C.byref(bw.struct), C.byref(tok), L.ptr(x), L.ptr(out),
                                          stream)
        assert st == 0, L.last_error()
        torch.cuda.synchronize()
        got = out.double().cpu().numpy()
        assert O.rel_l2(got, ref.double().cpu().numpy()) <= bound
        assert O.rel_l2(got - x.double().cpu().numpy(), ref.double().cpu().numpy() - x.double().cpu().numpy()) <= bound
    api.device_error()


def test_noalloc_matches_the_oracle_on_the_tiny_fp32_block(fs):
    # directly against the oracle, not only against dit_block_forward:
    # compressed (gather, block, nearest-kept broadcast) and plain, <= 1e-5
    w = S.WORKLOADS["tiny_block_f32"]
    dims, bw, seq, x = _case(w)
    layers, _ = S.make_weights(w, n_layers=1)
    wts = S.to_numpy64(layers[0])
    tags = S.pack_tokens(w)
    keep_idx, near_idx = O.keep_map(*w.grid)
    xh = x.double().cpu().numpy()
    stream = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    for compress in (True, False):
        tok = seq.struct if compress else seq.struct_full
        out = torch.full_like(x, float("nan"))
        assert fs.dit_block_forward_noalloc(C.byref(dims), C.byref(bw.struct), C.byref(tok), L.ptr(x), L.ptr(out),
                                            stream) == 0, L.last_error()
        torch.cuda.synchronize()
        if compress:
            ref = O.dit_block_compressed(xh, wts, tags["pos"], w.heads, w.head_dim, keep_idx, near_idx, w.n_video)
        else:
            ref = O.dit_block(xh, wts, tags["pos"], w.heads, w.head_dim)
        got = out.double().cpu().numpy()
        assert O.rel_l2(got, ref) <= 1e-5
        assert O.rel_l2(got - xh, ref - xh) <= 1e-5
    api.device_error()


def _long_tokens(n_text, grid=(2, 9, 10)):
    """A compressed sequence of a small grid plus n_text extra rows."""
    T, H, W = grid
    V = T * H * W
    n = V + n_text
    tags = {"pos": torch.zeros(n, 3, dtype=torch.int32).numpy(),
            "modality": torch.tensor([1] * V + [0] * n_text, dtype=torch.uint8).numpy(),
            "time_id": torch.zeros(n, dtype=torch.uint8).numpy(),
            "out_mask": torch.zeros(n, dtype=torch.uint8).numpy()}
    tags["pos"][:V, 1] = torch.arange(V).numpy() // W % H
    tags["pos"][:V, 2] = torch.arange(V).numpy() % W
    return api.Sequence(tags, grid, V, n_text, 0, DEV, compress=True)


@pytest.mark.parametrize("compress,limit", [(False, 9362), (True, 7262)])
def test_noalloc_accepts_its_largest_block_and_refuses_one_row_more(fs, compress, limit):
    # bf16, hidden 256, 2 x 128 heads, FFN 512: the header's limits, 9,362
    # rows uncompressed and 7,262 compressed rows (60 kept grid rows + text)
    w = S.scaled(S.WORKLOADS["flash_block_6x34x60"], hidden=256, heads=2, ffn=512, grid=(2, 9, 10), n_text=16,
                 n_audio=8)
    layers, _ = S.make_weights(w, n_layers=1)
    bw = api.BlockWeights({k: v.to(DEV) for k, v in layers[0].items()})
    dims = api.dims_of(w)
    stream = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    kept = 2 * 5 * 6
    for extra, want in ((0, 0), (1, -6)):
        n_text = (limit - kept if compress else limit - 180) + extra
        seq = _long_tokens(n_text)
        tok = seq.struct if compress else seq.struct_full
        x = torch.randn(seq.n_tokens, 256, generator=torch.Generator().manual_seed(5)).to(DEV)
        out = torch.full_like(x, float("nan"))
        st = fs.dit_block_forward_noalloc(C.byref(dims), C.byref(bw.struct), C.byref(tok), L.ptr(x), L.ptr(out),
                                          stream)
        assert st == want, L.last_error()
        if want == 0:
            ref = api.block_forward(dims, bw, seq, x, compress=compress)
            torch.cuda.synchronize()
            assert O.rel_l2(out.double().cpu().numpy(), ref.double().cpu().numpy()) <= 1e-6
    api.device_error()


def test_noalloc_rejects_blocks_beyond_its_static_scratch(fs):
    # a full-width 12,560-token block needs far more than the 32 MiB array;
    # the call fails on the host before any launch (pointers are never used)
    dims = api.make_dims(5376, 56, 14336, L.BF16)
    tok = L.Tokens()
    tok.n_tokens, tok.n_vrows, tok.n_text, tok.n_audio = 12560, 12240, 256, 64
    tok.pos_thw = 0x10000
    fake = C.c_void_p(0x10000)
    w = L.BlockWeights(*([0x10000] * 10))
    st = fs.dit_block_forward_noalloc(C.byref(dims), C.byref(w), C.byref(tok), fake, fake, None)
    assert st == -6
    assert "static" in L.last_error()
