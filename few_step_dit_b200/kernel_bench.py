"""Time single hot-path kernels through the C ABI (CUDA events, warm).

Examples:
  python -m few_step_dit_b200.kernel_bench attention --n 12560 --heads 56
  python -m few_step_dit_b200.kernel_bench gemm --M 12560 --N 21504 --K 5376 --epi qkv
  python -m few_step_dit_b200.kernel_bench block --workload flash_block_6x34x60
  python -m few_step_dit_b200.kernel_bench decoder [--grid 6x34x60] [--fp8]
  python -m few_step_dit_b200.kernel_bench generate   # 3-eval Flash pass + decoder
  python -m few_step_dit_b200.kernel_bench sweep      # compression sweep, 3 grids
  python -m few_step_dit_b200.kernel_bench layer --rows 3668,12560   # one layer's projections + attention
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
    kernel = "pair" if a.n >= L.load().fsdit_attention_pair_min_rows() else "single"
    return {"case": "attention", "n": a.n, "heads": a.heads, "kernel": kernel, "ms": ms, "tflops": fl / ms / 1e9}


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


SWEEP_GRIDS = ("6x17x30", "6x34x60", "12x34x60")


def case_sweep(a):
    """The compression sweep: one full-width Flash block (hidden 5376, 56 x
    128 heads, FFN 14336, bf16, 256 text + 64 audio rows) at each video grid,
    compressed (per-block form: gather, block on the kept rows, nearest-kept
    broadcast) and uncompressed.  Per grid: kept count, ms per block from a
    CUDA graph, and from one profiled run of each form the GEMM and attention
    TFLOP/s and the gather / broadcast GB/s.  Prints one JSON line per grid."""
    grids = a.grids.split(",") if a.grids else SWEEP_GRIDS
    out = []
    w0 = S.WORKLOADS["flash_block_6x34x60"]
    layers, _ = S.make_weights(w0, device="cuda", n_layers=1)
    bw = api.BlockWeights(layers[0])
    dims = api.dims_of(w0)
    for gname in grids:
        w = S.scaled(w0, grid=tuple(int(v) for v in gname.split("x")))
        seq = api.Sequence.from_workload(w, S.pack_tokens(w), "cuda", compress=True)
        g = torch.Generator(device="cuda").manual_seed(4)
        x = torch.randn(w.n_tokens, w.hidden, generator=g, device="cuda")
        y = torch.empty_like(x)
        res = {"case": "sweep", "workload": f"flash_block_{gname}", "tokens": w.n_tokens,
               "video_tokens": w.n_video, "kept_video_tokens": seq.n_keep, "compressed_tokens": seq.n_compressed}
        for comp in (False, True):
            tag = "compressed" if comp else "full"
            step = lambda: api.block_forward(dims, bw, seq, x, y, compress=comp)  # noqa: E731
            res[f"ms_{tag}"] = _graph_ms(step, a)
            prof = _profile(step)
            gm = {k: v for k, v in prof.items() if k.startswith("gemm")}
            g_ms = sum(v["ms"] for v in gm.values())
            g_fl = sum(v["tflops"] * v["ms"] * 1e9 for v in gm.values() if v["tflops"])
            res[f"gemm_tflops_{tag}"] = round(g_fl / g_ms / 1e9, 1) if g_ms else None
            if "attention" in prof:
                res[f"attention_tflops_{tag}"] = prof["attention"]["tflops"]
                res[f"attention_ms_{tag}"] = prof["attention"]["ms"]
            res[f"gemm_ms_{tag}"] = round(g_ms, 3)
            for k in ("gather", "broadcast", "rmsnorm_cast"):
                if k in prof:
                    res[f"{k}_gbs_{tag}"] = prof[k]["gbs"]
                    res[f"{k}_ms_{tag}"] = prof[k]["ms"]
        A, H, F = w.attn_dim, w.hidden, w.ffn

        def fl(n):
            return 2.0 * n * (4 * A * H + 2 * H * F) + 4.0 * n * n * A

        res["tflop_full"] = fl(w.n_tokens) / 1e12
        res["tflop_compressed"] = fl(seq.n_compressed) / 1e12
        res["tflops_full"] = res["tflop_full"] / res["ms_full"] * 1e3
        res["tflops_compressed"] = res["tflop_compressed"] / res["ms_compressed"] * 1e3
        res["speedup"] = res["ms_full"] / res["ms_compressed"]
        print(json.dumps(res), flush=True)
        out.append(res)
    return {"case": "sweep", "grids": list(grids), "speedups": [r["speedup"] for r in out]}


def case_embed(a):
    """The backbone's input side alone: a stack of zero layers (timestep MLP,
    text projection, the three embedding launches, final RMSNorm and heads) on
    the 6x34x60 sequence, replayed from a CUDA graph, plus a per-class profile:
    the small case for captures of the embedding kernel."""
    w = S.scaled(S.WORKLOADS["flash_backbone_6x34x60"], n_layers=0, compress=())
    _, io = S.make_weights(w, device="cuda", n_layers=0)
    bb = api.Backbone(api.dims_of(w), [], api.IOWeights(io), ())
    seq = api.Sequence.from_workload(w, S.pack_tokens(w), "cuda", compress=False)
    inp = S.make_inputs(w, device="cuda")
    table = [0.0, w.video_clock[0], w.audio_clock[0]]
    step = lambda: bb.forward(seq, table, inp["video_lat"], inp["text_emb"], inp["audio_lat"])  # noqa: E731
    ms = _graph_ms(step, a)
    return {"case": "embed", "tokens": w.n_tokens, "ms": ms, "classes": _profile(step)}


def case_layer(a):
    """The four projections of one Flash layer (QKV + RoPE, O + residual, FFN
    up + GELU, FFN down + residual) and its attention, on each row count of
    --rows (default: the compressed and full sequences of the three sweep
    grids), one launch each per iteration: the small case for per-launch
    ncu captures (DRAM traffic, tensor-pipe activity).  Prints one JSON line
    per row count."""
    w = S.WORKLOADS["flash_block_6x34x60"]
    H, A, F = w.hidden, w.attn_dim, w.ffn
    rows = [int(v) for v in a.rows.split(",")] if a.rows else [1184, 3380, 3668, 12560, 7016, 24800]
    Mx = max(rows)
    g = torch.Generator(device="cuda").manual_seed(6)
    dims = api.dims_of(w)
    layers, _ = S.make_weights(w, device="cuda", n_layers=1)
    l0 = layers[0]
    xh = torch.randn(Mx, H, generator=g, device="cuda").bfloat16()
    xa = torch.randn(Mx, A, generator=g, device="cuda").bfloat16()
    resid = torch.randn(Mx, H, generator=g, device="cuda")
    pos = torch.randint(0, 60, (Mx, 3), generator=g, device="cuda", dtype=torch.int32)
    qkv = torch.empty(Mx, 3 * A, dtype=torch.bfloat16, device="cuda")
    att = torch.empty(Mx, A, dtype=torch.bfloat16, device="cuda")
    u = torch.randn(Mx, F, generator=g, device="cuda").bfloat16()
    u_out = torch.empty(Mx, F, dtype=torch.bfloat16, device="cuda")

    def step(M):
        api.linear(dims, xh[:M], l0["w_qkv"], l0["b_qkv"], L.EPI_QKV_ROPE, pos=pos[:M], out=qkv[:M])
        api.attention(dims, qkv[:M], att[:M])
        api.linear(dims, xa[:M], l0["w_o"], l0["b_o"], L.EPI_RESIDUAL, resid=resid[:M], out=resid[:M])
        api.linear(dims, xh[:M], l0["w_1"], l0["b_1"], L.EPI_GELU, out=u_out[:M])
        api.linear(dims, u[:M], l0["w_2"], l0["b_2"], L.EPI_RESIDUAL, resid=resid[:M], out=resid[:M])

    for it in range(a.warmup + a.iters):
        for M in rows:
            step(M)
    torch.cuda.synchronize()
    out = []
    for M in rows:
        ms = time_it(lambda: step(M), a.iters, 0)
        fl = 2.0 * M * (4 * A * H + 2 * H * F) + 4.0 * M * M * A
        r = {"case": "layer", "M": M, "ms": ms, "tflops": fl / ms / 1e9, "launches": 5,
             "weight_bytes": 2.0 * (4 * A * H + 2 * H * F)}
        print(json.dumps(r), flush=True)
        out.append(r)
    return {"case": "layer", "rows": rows}


def main():
    p = argparse.ArgumentParser()
    p.add_argument("case", choices=["attention", "gemm", "block", "memory", "chunk", "decoder", "generate",
                                    "sweep", "layer", "embed"])
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
    p.add_argument("--grids", default="", help="sweep: comma-separated grids (default 6x17x30,6x34x60,12x34x60)")
    p.add_argument("--rows", default="", help="layer: comma-separated row counts")
    p.add_argument("--pair-min-rows", type=int, default=0,
                   help="attention: rows from which the CTA-pair kernel runs (0: the library default)")
    p.add_argument("--iters", type=int, default=10)
    p.add_argument("--warmup", type=int, default=3)
    a = p.parse_args()
    B.build()
    lib = L.load()
    if a.pair_min_rows > 0:
        L.check("fsdit_set_attention_pair_min_rows", lib.fsdit_set_attention_pair_min_rows(a.pair_min_rows))
    res = {"attention": case_attention, "gemm": case_gemm, "block": case_block,
           "memory": case_memory, "chunk": case_chunk, "decoder": case_decoder,
           "generate": case_generate, "sweep": case_sweep, "layer": case_layer, "embed": case_embed}[a.case](a)
    api.device_error()
    print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
