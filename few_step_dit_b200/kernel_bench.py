"""Time single hot-path kernels through the C ABI (CUDA events, warm).

Examples:
  python -m few_step_dit_b200.kernel_bench attention --n 12560 --heads 56
  python -m few_step_dit_b200.kernel_bench gemm --M 12560 --N 21504 --K 5376 --epi qkv
  python -m few_step_dit_b200.kernel_bench block --workload flash_block_6x34x60
  python -m few_step_dit_b200.kernel_bench decoder [--grid 6x34x60] [--fp8]
  python -m few_step_dit_b200.kernel_bench generate   # 3-eval Flash pass + decoder
Inputs are seeded Gaussians; each case prints one JSON line.
"""

from __future__ import annotations

import argparse
import json
import os
import sys

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from few_step_dit_b200 import api, build as B, lib as L  # noqa: E402
from few_step_dit_b200 import synthetic as S  # noqa: E402

EPI = {"bias": L.EPI_BIAS, "bias_f32": L.EPI_BIAS_F32, "qkv": L.EPI_QKV_ROPE, "gelu": L.EPI_GELU,
       "residual": L.EPI_RESIDUAL}


def time_it(fn, iters, warmup):
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(iters):
        fn()
    e.record()
    e.synchronize()
    return s.elapsed_time(e) / iters


def case_attention(a):
    g = torch.Generator(device="cuda").manual_seed(1)
    A = a.heads * 128
    dims = api.make_dims(5376, a.heads, 14336, L.BF16)
    qkv = torch.randn(a.n, 3 * A, generator=g, device="cuda").mul_(1.5).bfloat16()
    out = torch.empty(a.n, A, dtype=torch.bfloat16, device="cuda")
    ms = time_it(lambda: api.attention(dims, qkv, out), a.iters, a.warmup)
    fl = 4.0 * a.n * a.n * A
    return {"case": "attention", "n": a.n, "heads": a.heads, "ms": ms, "tflops": fl / ms / 1e9}


def case_gemm(a):
    g = torch.Generator(device="cuda").manual_seed(2)
    epi = EPI[a.epi]
    heads = a.N // 3 // 128 if epi == L.EPI_QKV_ROPE else 56
    dims = api.make_dims(5376, heads, 14336, L.BF16)
    x = torch.randn(a.M, a.K, generator=g, device="cuda").bfloat16()
    w = torch.randn(a.N, a.K, generator=g, device="cuda").mul_(0.02).bfloat16()
    b = torch.randn(a.N, generator=g, device="cuda").mul_(0.02).bfloat16()
    resid = torch.randn(a.M, a.N, generator=g, device="cuda") if epi == L.EPI_RESIDUAL else None
    pos = torch.randint(0, 60, (a.M, 3), generator=g, device="cuda", dtype=torch.int32) \
        if epi == L.EPI_QKV_ROPE else None
    od = torch.float32 if epi in (L.EPI_RESIDUAL, L.EPI_BIAS_F32) else torch.bfloat16
    out = torch.empty(a.M, a.N, dtype=od, device="cuda")
    scr = api.gemm_scratch("cuda") if a.cut else None
    if a.fp8:
        dims8 = api.make_dims(5376, heads, 14336, L.BF16, proj_fp8=True)
        qx, sx = api.quantize_rows(x)
        qw, sw = api.quantize_rows(w)
        fn = lambda: api.linear_fp8(dims8, qx, sx, qw, sw, b, epi, resid=resid, pos=pos, out=out, scratch=scr)
    else:
        fn = lambda: api.linear(dims, x, w, b, epi, resid=resid, pos=pos, out=out, scratch=scr)
    ms = time_it(fn, a.iters, a.warmup)
    fl = 2.0 * a.M * a.N * a.K
    return {"case": "gemm", "M": a.M, "N": a.N, "K": a.K, "epi": a.epi, "fp8": bool(a.fp8), "tail_cut": bool(a.cut),
            "ms": ms, "tflops": fl / ms / 1e9}


def case_block(a):
    w = S.WORKLOADS[a.workload]
    layers, _ = S.make_weights(w, device="cuda", n_layers=1)
    tags = S.pack_tokens(w)
    seq = api.Sequence.from_workload(w, tags, "cuda", compress=True)
    bw = api.BlockWeights(layers[0])
    dims = api.dims_of(w)
    x = torch.randn(w.n_tokens, w.hidden, device="cuda")
    out = torch.empty_like(x)
    res = {"case": "block", "workload": a.workload, "tokens": w.n_tokens, "kept": seq.n_keep}
    for comp in (True, False):
        ms = time_it(lambda: api.block_forward(dims, bw, seq, x, out, compress=comp), a.iters, a.warmup)
        res["ms_compressed" if comp else "ms_full"] = ms
    return res


def case_memory(a):
    """Full-width gather, broadcast (in place) and RMSNorm-cast on a grid."""
    w = S.WORKLOADS[a.workload]
    T, H, W = w.grid
    n = w.n_tokens
    g = torch.Generator(device="cuda").manual_seed(3)
    x = torch.randn(n, w.hidden, generator=g, device="cuda")
    pos = torch.zeros(n, 3, dtype=torch.int32, device="cuda")
    keep_idx, near_idx = api.keep_map(T, H, W)
    n_keep = keep_idx.numel()
    xc, posc = api.gather_rows(x, pos, keep_idx, w.n_video)
    gain = torch.ones(w.hidden, dtype=torch.bfloat16, device="cuda")
    res = {"case": "memory", "workload": a.workload, "rows": n, "kept": n_keep}
    hb = w.hidden * 4.0
    ms = time_it(lambda: api.gather_rows(x, pos, keep_idx, w.n_video), a.iters, a.warmup)
    res["gather_ms"], res["gather_gbs"] = ms, xc.shape[0] * hb * 2 / ms / 1e6
    ms = time_it(lambda: api.broadcast_residual(x, xc, keep_idx, near_idx, w.grid, out=x), a.iters, a.warmup)
    res["broadcast_ms"] = ms
    res["broadcast_gbs"] = (w.n_video + xc.shape[0] + n) * hb / ms / 1e6
    ms = time_it(lambda: api.rmsnorm_cast(x, gain), a.iters, a.warmup)
    res["rmsnorm_ms"], res["rmsnorm_gbs"] = ms, n * w.hidden * 6.0 / ms / 1e6
    # E4M3 quantizers: the fused RMSNorm-quantizer (fp32 in, codes + scales out)
    # and the per-row quantizer of a bf16 attention output [n, A]
    ms = time_it(lambda: api.rmsnorm_quant(x, gain), a.iters, a.warmup)
    res["rmsnorm_quant_ms"], res["rmsnorm_quant_gbs"] = ms, n * (w.hidden * 5.0 + 4) / ms / 1e6
    att = torch.randn(n, w.attn_dim, generator=g, device="cuda").bfloat16()
    ms = time_it(lambda: api.quantize_rows(att), a.iters, a.warmup)
    res["quant_rows_ms"], res["quant_rows_gbs"] = ms, n * (w.attn_dim * 3.0 + 4) / ms / 1e6
    return res


def case_chunk(a):
    """One steady-state long-video chunk of the 42-layer Flash backbone: the
    target grid (default 6x34x60: boundary + 5 future latents) plus a full
    11-frame history (4,140 rows at 34x60), 3 evaluations, replayed from a
    CUDA graph."""
    w = S.WORKLOADS["flash_backbone_6x34x60"]
    if a.grid:
        w = S.scaled(w, grid=tuple(int(v) for v in a.grid.split("x")))
    T, H, W = w.grid
    layers, io = S.make_weights(w, device="cuda")
    if a.fp8:
        layers = [api.quantize_block_weights(l) for l in layers]
    bb = api.Backbone(api.dims_of(w, proj_fp8=a.fp8), [api.BlockWeights(l) for l in layers], api.IOWeights(io),
                      w.compress)
    inp = S.make_inputs(w, device="cuda")
    lv = api.LongVideo(bb, w.grid, w.n_text, w.n_audio, w.video_ch)
    g = torch.Generator(device="cuda").manual_seed(8)
    lv.store.push(torch.randn(21 * H * W, w.video_ch, generator=g, device="cuda"))
    seq, vl, has_b, base = lv.prepare()
    n_grid, hw = T * H * W, H * W
    vl[:n_grid].copy_(inp["video_lat"][:n_grid])
    lv.store.copy_frame(base, vl[:hw])
    v0, a0 = vl.clone(), inp["audio_lat"].clone()
    al = a0.clone()

    def step():
        vl.copy_(v0)
        al.copy_(a0)
        bb.sample(seq, w.video_clock, w.audio_clock, vl, inp["text_emb"], al)

    step()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    ms = time_it(graph.replay, a.iters, a.warmup)
    del graph
    plan, n = lv.store.plan(base)
    rows = lv.store.rows(plan, n)
    lat = torch.empty(rows, w.video_ch, device="cuda")
    pos = torch.empty(rows, 3, dtype=torch.int32, device="cuda")
    g_ms = time_it(lambda: lv.store.gather(plan, n, lat, pos), 50, 5)
    tokens = seq.n_tokens
    A, Hd, F = w.attn_dim, w.hidden, w.ffn

    def layer_flops(n):  # projections 2n(3AH + AH + 2HF) + attention 4n^2 A
        return 2.0 * n * (4 * A * Hd + 2 * Hd * F) + 4.0 * n * n * A

    per_eval = sum(layer_flops(seq.n_compressed if c else tokens) for c in w.compress)
    tflop = per_eval * w.n_evals / 1e12
    return {"case": "chunk", "tflop_per_chunk": tflop, "tflops": tflop / ms * 1e3, "fp8": bool(a.fp8),
            "workload": f"flash_chunk_{T}x{H}x{W}_history11", "history_rows": rows, "tokens": tokens,
            "compressed_tokens": seq.n_compressed, "ms_per_chunk": ms,
            "tokens_per_s": tokens * w.n_evals / ms * 1e3, "new_frames_per_s": 17 / ms * 1e3,
            "gather_ms": g_ms, "gather_gbs": rows * (w.video_ch * 8 + 12) / g_ms / 1e6}


def _decoder(a, device="cuda"):
    w = S.DECODER_WORKLOADS["decoder_6x34x60"]
    if a.grid:
        w = S.scaled(w, grid=tuple(int(v) for v in a.grid.split("x")))
    layers, io = S.make_decoder_weights(w, device=device)
    if a.fp8:
        layers = [api.quantize_block_weights(l) for l in layers]
    dec = api.Decoder(api.dims_of(w, proj_fp8=a.fp8), [api.BlockWeights(l) for l in layers],
                      api.DecoderIO(io, w.c_pix, w.patch_t, w.patch_s))
    return w, dec


def _decoder_flops(w):
    n, A, Hd, F = w.n_cells, w.attn_dim, w.hidden, w.ffn
    per_layer = 2.0 * n * (4 * A * Hd + 2 * Hd * F) + 4.0 * n * n * A
    return w.n_layers * per_layer + 2.0 * n * Hd * (w.c_lat + w.pixel_cols)


def _graph_ms(step, a):
    step()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    ms = time_it(graph.replay, a.iters, a.warmup)
    del graph
    return ms


def _profile(step):
    step()
    torch.cuda.synchronize()
    L.profile_start()
    step()
    prof = L.profile_stop()
    tot = sum(v["ms"] for v in prof.values())
    return {k: {"ms": round(v["ms"], 3), "share": round(v["ms"] / tot, 4),
                "tflops": round(v["flops"] / v["ms"] / 1e9, 1) if v["flops"] else None,
                "gbs": round(v["bytes"] / v["ms"] / 1e6, 1)} for k, v in prof.items()}


def case_decoder(a):
    """The 26-layer lightweight decoder (hidden 2048, 16 heads, FFN 8192) on
    a latent grid (default 6x34x60 -> 21 frames of 544x960), replayed from a
    CUDA graph; plus a per-kernel-class profile of one eager run."""
    w, dec = _decoder(a)
    lat = S.make_decoder_latents(w, device="cuda")
    px = torch.empty(w.pixel_shape, dtype=torch.uint8 if a.rgb8 else torch.float32, device="cuda")
    step = lambda: dec.forward(lat, w.grid, pixels=px, rgb8=a.rgb8)  # noqa: E731
    ms = _graph_ms(step, a)
    tflop = _decoder_flops(w) / 1e12
    T, H, W = w.grid
    return {"case": "decoder", "workload": f"decoder_{T}x{H}x{W}", "fp8": bool(a.fp8), "rgb8": bool(a.rgb8),
            "cells": w.n_cells,
            "frames": w.n_frames, "ms": ms, "tflop": tflop, "tflops": tflop / ms * 1e3,
            "frames_per_s": w.n_frames / ms * 1e3, "classes": _profile(step)}


def case_generate(a):
    """The pages' latency protocol on one GPU: a sampling pass of the backbone
    (default the 3-evaluation Flash pass, 42 layers, 6x34x60, text 256, audio
    64; --backbone standard_backbone_12x34x60 for the 4-evaluation standard
    model) followed by the 26-layer decoder of its target-grid video latents,
    one CUDA graph, warm."""
    wb = S.WORKLOADS[a.backbone]
    layers, io = S.make_weights(wb, device="cuda")
    if a.fp8:
        layers = [api.quantize_block_weights(l) for l in layers]
    bb = api.Backbone(api.dims_of(wb, proj_fp8=a.fp8), [api.BlockWeights(l) for l in layers], api.IOWeights(io),
                      wb.compress)
    seq = api.Sequence.from_workload(wb, S.pack_tokens(wb), "cuda")
    inp = S.make_inputs(wb, device="cuda")
    a.grid = "x".join(str(v) for v in wb.grid)
    wd, dec = _decoder(a)
    assert wd.grid == wb.grid and wd.c_lat == wb.video_ch
    vl, al = inp["video_lat"].clone(), inp["audio_lat"].clone()
    target = vl[:wb.n_video]  # the target grid's latents (control frames follow)
    px = torch.empty(wd.pixel_shape, device="cuda")

    def step():
        vl.copy_(inp["video_lat"])
        al.copy_(inp["audio_lat"])
        bb.sample(seq, wb.video_clock, wb.audio_clock, vl, inp["text_emb"], al)
        dec.forward(target, wd.grid, pixels=px)

    ms = _graph_ms(step, a)
    ms_dec = _graph_ms(lambda: dec.forward(target, wd.grid, pixels=px), a)
    T, H, W = wd.grid
    return {"case": "generate", "workload": f"{wb.name}+decoder_{T}x{H}x{W}", "fp8": bool(a.fp8),
            "ms": ms, "ms_decoder": ms_dec, "ms_backbone": ms - ms_dec, "frames": wd.n_frames,
            "frames_per_s": wd.n_frames / ms * 1e3}


def main():
    p = argparse.ArgumentParser()
    p.add_argument("case", choices=["attention", "gemm", "block", "memory", "chunk", "decoder", "generate"])
    p.add_argument("--n", type=int, default=12560)
    p.add_argument("--heads", type=int, default=56)
    p.add_argument("--M", type=int, default=12560)
    p.add_argument("--N", type=int, default=21504)
    p.add_argument("--K", type=int, default=5376)
    p.add_argument("--epi", default="qkv", choices=sorted(EPI))
    p.add_argument("--workload", default="flash_block_6x34x60")
    p.add_argument("--fp8", action="store_true",
                   help="gemm / chunk / decoder / generate: E4M3 projections (per-row scales)")
    p.add_argument("--grid", default="", help="chunk / decoder: latent grid TxHxW (default 6x34x60)")
    p.add_argument("--cut", action="store_true", help="gemm: cut the last wave's tiles along K (fsdit_linear_ws)")
    p.add_argument("--backbone", default="flash_backbone_6x34x60", help="generate: the backbone workload")
    p.add_argument("--rgb8", action="store_true", help="decoder: 8-bit RGB frames (fused colour conversion)")
    p.add_argument("--iters", type=int, default=10)
    p.add_argument("--warmup", type=int, default=3)
    a = p.parse_args()
    B.build()
    L.load()
    res = {"attention": case_attention, "gemm": case_gemm, "block": case_block,
           "memory": case_memory, "chunk": case_chunk, "decoder": case_decoder,
           "generate": case_generate}[a.case](a)
    api.device_error()
    print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
