"""The failure path of the library's bounded device waits, exercised without
a fault: a kernel waits, through the same bounded mbarrier wait the
tensor-core kernels use, on a barrier nothing arrives at; the wait gives up
after its limit, the host reads FSDIT_E_TIMEOUT from the device error word,
and the context keeps working (a projection afterwards is correct and the
word is clear again)."""

import pytest
import torch

import oracle as O
from few_step_dit_b200 import api, build, lib as L

pytestmark = pytest.mark.gpu
DEV = "cuda"


def test_bounded_wait_times_out_and_the_context_stays_usable():
    build.build()
    fs = L.load()
    torch.cuda.synchronize()
    api.device_error()                          # start from a clear word
    res = torch.full((2,), -1, dtype=torch.int32, device=DEV)
    assert fs.fsdit_check_bounded_wait(L.ptr(res), None) == 0
    assert fs.fsdit_device_error(None) == -7   # FSDIT_E_TIMEOUT, word cleared
    assert "timed out" in L.last_error()
    assert res.tolist() == [0, 1]              # not completed, abort flag set
    # the context still runs work correctly and the word stays clear
    g = torch.Generator().manual_seed(9)
    a = torch.randn(300, 512, generator=g).bfloat16()
    w = (0.05 * torch.randn(256, 512, generator=g)).bfloat16()
    b = (0.05 * torch.randn(256, generator=g)).bfloat16()
    out = api.linear(api.make_dims(256, 2, 512, torch.bfloat16), a.to(DEV), w.to(DEV), b.to(DEV), L.EPI_BIAS_F32)
    torch.cuda.synchronize()
    ref = O.linear(a.double().numpy(), w.double().numpy(), b.double().numpy())
    assert O.rel_l2(out.double().cpu().numpy(), ref) < 1e-4
    assert fs.fsdit_device_error(None) == 0


def test_check_rejects_null_result():
    build.build()
    fs = L.load()
    assert fs.fsdit_check_bounded_wait(None, None) == -1
