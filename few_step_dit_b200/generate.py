"""Generate and decode a clip end to end with seeded random weights.

  python -m few_step_dit_b200.generate --out clip.npy                 # Flash, 6x34x60 -> 21 frames
  python -m few_step_dit_b200.generate --chunks 4 --out long.npy      # long video: 4 chunks
  python -m few_step_dit_b200.generate --backbone standard_backbone_12x34x60 --out std.npy
  python -m few_step_dit_b200.generate --proj-fp8 --out clip8.npy     # E4M3 block projections

One clip: the few-step sampler of the backbone (dit_flow_sample) from seeded
noise, then the decoder (fsdit_decoder_forward) of the target grid's latents.
Long video (--chunks N): chunk after chunk with the bounded history store; every
chunk after the first starts from the previous chunk's last latent frame (its
boundary), is decoded on its own and loses the boundary's frame, so the clip
grows by 4 x (T - 1) frames a chunk.  Frames are written as uint8 RGB
[frames, 3, height, width]: the decoder's pixel head converts its values from
[-1, 1] to 8-bit codes on the GPU (fsdit_decoder_forward, FSDIT_PIXELS_RGB8).
No trained weights are available, so the frames are noise-like: the command
exercises and times the path (one JSON line with the stage times on stdout).
"""

from __future__ import annotations

import argparse
import json
import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from few_step_dit_b200 import api, build as B, lib as L  # noqa: E402
from few_step_dit_b200 import synthetic as S  # noqa: E402


def tiny_workloads():
    """A small-width backbone and decoder with the same structure (for tests
    and quick runs)."""
    wb = S.scaled(S.WORKLOADS["flash_backbone_6x34x60"], hidden=256, heads=2, ffn=512, grid=(3, 6, 8),
                  n_text=16, n_audio=8, n_layers=4, compress=(0, 1, 1, 0))
    wd = S.scaled(S.DECODER_WORKLOADS["decoder_6x34x60"], hidden=256, heads=2, ffn=1024, n_layers=2,
                  grid=(3, 6, 8), patch_s=4)
    return wb, wd


def run(backbone="flash_backbone_6x34x60", proj_fp8=False, chunks=0, tiny=False, seed=S.SEED_INPUTS,
        device="cuda"):
    """Returns (uint8 frames [F, 3, H', W'] on the host, timings dict)."""
    B.build()
    L.load()
    if tiny:
        wb, wd = tiny_workloads()
    else:
        wb = S.WORKLOADS[backbone]
        wd = S.scaled(S.DECODER_WORKLOADS["decoder_6x34x60"], grid=wb.grid)
    if wd.c_lat != wb.video_ch:
        raise ValueError("decoder latent channels differ from the backbone's video channels")
    layers, io = S.make_weights(wb, device=device)
    if proj_fp8:
        layers = [api.quantize_block_weights(l) for l in layers]
    bb = api.Backbone(api.dims_of(wb, proj_fp8=proj_fp8), [api.BlockWeights(l) for l in layers],
                      api.IOWeights(io), wb.compress)
    dl, dio = S.make_decoder_weights(wd, device=device)
    if proj_fp8:
        dl = [api.quantize_block_weights(l) for l in dl]
    dec = api.Decoder(api.dims_of(wd, proj_fp8=proj_fp8), [api.BlockWeights(l) for l in dl],
                      api.DecoderIO(dio, wd.c_pix, wd.patch_t, wd.patch_s))
    g = torch.Generator(device=device).manual_seed(seed)
    text = torch.randn(wb.n_text, wb.text_dim, generator=g, device=device).to(wb.torch_dtype)
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    t_sample = t_decode = 0.0
    out = []
    if chunks <= 0:
        inp = S.make_inputs(wb, device=device, seed=seed)
        seq = api.Sequence.from_workload(wb, S.pack_tokens(wb), device)
        vl, al = inp["video_lat"].clone(), inp["audio_lat"].clone()
        e0, e1, e2 = ev(), ev(), ev()
        e0.record()
        bb.sample(seq, wb.video_clock, wb.audio_clock, vl, inp["text_emb"], al)
        e1.record()
        px = dec.forward(vl[:wb.n_video], wd.grid, rgb8=True)
        e2.record()
        e2.synchronize()
        t_sample, t_decode = e0.elapsed_time(e1), e1.elapsed_time(e2)
        out.append(px.cpu())
    else:
        lv = api.LongVideo(bb, wb.grid, wb.n_text, wb.n_audio, wb.video_ch, device=device)
        for k in range(chunks):
            noise_v = torch.randn(wb.n_video, wb.video_ch, generator=g, device=device)
            noise_a = torch.randn(wb.n_audio, wb.audio_dim, generator=g, device=device)
            e0, e1, e2 = ev(), ev(), ev()
            e0.record()
            lat, _ = lv.chunk(noise_v, text, noise_a, wb.video_clock, wb.audio_clock)
            e1.record()
            px = dec.forward(lat, wd.grid, rgb8=True)
            e2.record()
            e2.synchronize()
            t_sample += e0.elapsed_time(e1)
            t_decode += e1.elapsed_time(e2)
            out.append((px if k == 0 else px[1:]).cpu())  # drop the boundary's frame
    api.device_error()
    frames = torch.cat(out)
    return frames, {"sample_ms": t_sample, "decode_ms": t_decode}


def main():
    p = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    p.add_argument("--backbone", default="flash_backbone_6x34x60", choices=sorted(S.WORKLOADS))
    p.add_argument("--proj-fp8", action="store_true", help="E4M3 block projections (backbone and decoder)")
    p.add_argument("--chunks", type=int, default=0, help="long video: number of chunks (0: one clip)")
    p.add_argument("--tiny", action="store_true", help="small-width backbone and decoder")
    p.add_argument("--seed", type=int, default=S.SEED_INPUTS)
    p.add_argument("--out", default="", help=".npy file for the uint8 frames")
    a = p.parse_args()
    frames, t = run(a.backbone, a.proj_fp8, a.chunks, a.tiny, a.seed)
    if a.out:
        np.save(a.out, frames.numpy())
    print(json.dumps({"frames": int(frames.shape[0]), "shape": list(frames.shape), "out": a.out or None,
                      "backbone": "tiny" if a.tiny else a.backbone, "proj_fp8": bool(a.proj_fp8),
                      "chunks": a.chunks, **{k: round(v, 3) for k, v in t.items()}}), flush=True)


if __name__ == "__main__":
    main()
