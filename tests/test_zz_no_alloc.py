"""dit_block_forward_noalloc: the block forward for callers that cannot call
cudaMalloc (for example a host application whose device memory belongs to its
own pool allocator), with its scratch in a static device array inside the
library.  Its output must match dit_block_forward (which takes a workspace
from the caller) within the tests' usual bounds, on two calls in a row.

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


def test_noalloc_rejects_blocks_beyond_its_static_scratch(fs):
    # a full-width 12,560-token block needs far more than the 32 MiB array;
    # the call fails on the host before any launch (pointers are never used)
    dims = api.make_dims(5376, 56, 14336, L.BF16)
    tok = L.Tokens()
    tok.n_tokens, tok.n_vrows, tok.n_text, tok.n_audio = 12560, 12240, 256, 64
    fake = C.c_void_p(0x10000)
    w = L.BlockWeights(*([0x10000] * 10))
    st = fs.dit_block_forward_noalloc(C.byref(dims), C.byref(w), C.byref(tok), fake, fake, None)
    assert st == -6
    assert "static" in L.last_error()
