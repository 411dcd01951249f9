"""The end-to-end generate command on a small-width backbone and decoder:
one clip (sampler, then decoder) and a long video (chunks with the bounded
history, each decoded on its own without its boundary frame), bf16 and with
E4M3 projections.  The stages themselves are checked against the oracle in
their own tests; here the frame counts, shapes, value range and determinism."""

import pytest
import torch

from few_step_dit_b200 import generate as G

pytestmark = pytest.mark.gpu


def test_one_clip_frames():
    frames, t = G.run(tiny=True)
    wb, wd = G.tiny_workloads()
    T, H, W = wd.grid
    assert frames.dtype == torch.uint8
    assert tuple(frames.shape) == (1 + wd.patch_t * (T - 1), 3, H * wd.patch_s, W * wd.patch_s)
    assert frames.float().std() > 0 and t["sample_ms"] > 0 and t["decode_ms"] > 0
    again, _ = G.run(tiny=True)
    assert torch.equal(frames, again)


@pytest.mark.parametrize("fp8", [False, True])
def test_long_video_frames(fp8):
    frames, _ = G.run(tiny=True, chunks=3, proj_fp8=fp8)
    wb, wd = G.tiny_workloads()
    T, H, W = wd.grid
    first = 1 + wd.patch_t * (T - 1)
    assert tuple(frames.shape) == (first + 2 * wd.patch_t * (T - 1), 3, H * wd.patch_s, W * wd.patch_s)
    assert frames.float().std() > 0
