#!/usr/bin/env python
"""Benchmark of the Flash backbone hot path on B200.

One step = one few-step sampling pass: 3 flow-matching evaluations of the
42-layer Flash backbone (layers 1-2 full, 3-28 token-compressed, 29-42 full)
on a 6x34x60 video grid + 256 text + 64 audio tokens, each followed by the
per-modality Euler update, through dit_flow_sample.  Weights are random
(seeded) bf16; inputs are seeded Gaussian latents and text features.

Contract: `python bench.py --gpus N --steps K --warmup W`; N>1 runs under
torchrun with one independent replica per GPU (no collective on the data
path; weak scaling).  Rank 0 prints one JSON line.  `--impl reference` times
the fp64 CPU oracle on a bounded sample of the same workload instead.
"""

from __future__ import annotations

import argparse
import gc
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

from few_step_dit_b200 import api, build as B, lib as L, replicas as R  # noqa: E402
from few_step_dit_b200 import synthetic as S  # noqa: E402

METRIC = "Flash backbone ms/3-eval pass and tokens/s on 1 B200; % of bf16 tensor peak"


def metric_of(w):
    """The headline metric names the Flash backbone; other workloads name their own."""
    if w.name.startswith("flash_backbone"):
        return METRIC
    kind = "Standard" if w.name.startswith("standard") else w.name
    return f"{kind} backbone ms/{w.n_evals}-eval pass and tokens/s on 1 B200; % of bf16 tensor peak"
UNIT = "tokens/s"
PEAKS_PATH = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# NVIDIA's dense bf16 tensor-core figure for one B200 (context for the fractions)
NOMINAL_BF16_TFLOPS = 2250.0
GEMM_SOURCES = ["few_step_dit_b200/csrc/gemm_tc.cu", "few_step_dit_b200/csrc/common.cuh",
                "few_step_dit_b200/csrc/tc_ptx.cuh"]
TRAFFIC_PATH = os.path.join(ROOT, "profiles", "gemm_traffic_flash_backbone_6x34x60.json")


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=5)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", default="fsdit", choices=["fsdit", "reference"])
    p.add_argument("--workload", default="flash_backbone_6x34x60")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-full-compare", action="store_true",
                   help="skip timing the same backbone with compression off")
    p.add_argument("--eager", action="store_true", help="time eager launches instead of a CUDA graph")
    p.add_argument("--proj-fp8", action="store_true",
                   help="run the four block projections on E4M3 operands (per-row scales); a separate "
                        "configuration, not the bf16 headline")
    return p.parse_args()


def load_peaks():
    try:
        with open(PEAKS_PATH) as f:
            return json.load(f), "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def _code_lines(text):
    """Source text without // comments and blank lines: the hash follows code changes only."""
    out = []
    for line in text.splitlines():
        line = line.split("//", 1)[0].rstrip()
        if line.strip():
            out.append(line)
    return "\n".join(out)


def gemm_sources_sha256(read=None):
    h = hashlib.sha256()
    for rel in GEMM_SOURCES:
        if read is None:
            with open(os.path.join(ROOT, rel), encoding="utf-8") as f:
                text = f.read()
        else:
            text = read(rel)
        h.update(_code_lines(text).encode())
    return h.hexdigest()


def gemm_traffic(workload):
    """DRAM bytes per GEMM launch from the committed ncu capture of this
    workload, or None when there is none or the GEMM sources changed since."""
    try:
        with open(TRAFFIC_PATH) as f:
            d = json.load(f)
    except (OSError, ValueError):
        return None
    if d.get("workload") != workload or d.get("sources_sha256") != gemm_sources_sha256():
        return None
    return d.get("dram_bytes_per_launch")


def peak_fracs(achieved, sustained, burst, nominal=None):
    """A TFLOP/s figure as a fraction of each basis: the measured sustained
    (power-capped, seconds-long) cuBLAS rate, the measured burst rate, and the
    nominal dense peak."""
    nominal = NOMINAL_BF16_TFLOPS if nominal is None else nominal
    out = {"of_measured_sustained": achieved / sustained if sustained else None,
           "of_measured_burst": achieved / burst if burst else None,
           "of_nominal_dense": achieved / nominal if nominal else None}
    return out


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi clock / throttle-reason sampling during the timed region."""

    Q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, device_index):
        self.proc = None
        try:
            uuid = "GPU-" + str(torch.cuda.get_device_properties(device_index).uuid)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", uuid, f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, RuntimeError, AttributeError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons = [], None, set()
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 7:
                continue
            try:
                sm.append(float(f[0]))
                smax = float(f[1])
            except ValueError:
                continue
            for name, val in zip(self.NAMES, f[3:7]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------- work counts

def block_flops(w, n):
    """Algorithmic FLOPs of one block on n rows: qkv, output, two FFN
    projections and the two attention contractions (A = heads * head_dim)."""
    H, F, A = w.hidden, w.ffn, w.attn_dim
    return 2.0 * n * (3 * A * H + A * H + 2 * H * F) + 4.0 * n * n * A


def pass_flops(w, compressed=True):
    T, Hg, Wg = w.grid
    n_keep = T * (Hg // 2 + 1) * (Wg // 2 + 1)
    n_c = n_keep + w.n_tokens - w.n_video
    tot = 0.0
    for c in w.compress:
        tot += block_flops(w, n_c if (c and compressed) else w.n_tokens)
    return tot * w.n_evals


# ---------------------------------------------------------------- CPU oracle sample

def oracle_sample(w, reps=1):
    """Time the fp64 oracle on one token-compressed full-width block of the
    workload (its kept video rows + text + audio; the full sequence when the
    workload has no compressed layer) and project a full pass by FLOPs.

    Returns (tokens_per_s, seconds_per_pass, sample_description, threads)."""
    import numpy as np

    import oracle as O

    T, H, W = w.grid
    comp = any(w.compress)
    k, _ = O.keep_map(T, H, W)
    n_s = len(k) + w.n_tokens - w.n_video if comp else w.n_tokens
    g = torch.Generator().manual_seed(S.SEED_WEIGHTS)
    wts = S.to_numpy64(S.make_block_weights(w, g))
    rng = np.random.default_rng(S.SEED_INPUTS)
    x = rng.standard_normal((n_s, w.hidden))
    tags = S.pack_tokens(w)
    pos = O.gather_rows(tags["pos"], k, w.n_video) if comp else tags["pos"]
    times = []
    for _ in range(reps):
        t0 = time.perf_counter()
        O.dit_block(x, wts, pos, w.heads, w.head_dim)
        times.append(time.perf_counter() - t0)
    t_s = statistics.median(times)
    f_s = block_flops(w, n_s)
    n_comp = sum(1 for c in w.compress if c)
    per_pass = 0.0
    for c in w.compress:
        per_pass += t_s * block_flops(w, n_s if c else w.n_tokens) / f_s
    per_pass *= w.n_evals
    desc = (f"projected by FLOPs from one {'token-compressed ' if comp else ''}full-width block ({n_s} rows, "
            f"hidden {w.hidden}) timed in fp64 numpy ({t_s:.2f} s); pass = {w.n_evals} evals x "
            f"({n_comp} compressed + {len(w.compress) - n_comp} full layers)")
    return w.n_tokens * w.n_evals / per_pass, per_pass, desc, blas_threads()


def oracle_tiny(reps=3):
    """The oracle timed directly (no projection) on the tiny fp32 workload:
    one compressed block, one plain block and one Euler step (video
    0.2 -> 0.0769, audio 0.5 -> 0.25), median of `reps`."""
    import numpy as np

    import oracle as O

    w = S.WORKLOADS["tiny_block_f32"]
    g = torch.Generator().manual_seed(S.SEED_WEIGHTS)
    wts = S.to_numpy64(S.make_block_weights(w, g))
    tags = S.pack_tokens(w)
    inp = S.make_inputs(w)
    x = inp["x"].double().numpy()
    k, near = O.keep_map(*w.grid)
    vl = inp["video_lat"].double().numpy()
    v = np.ones_like(vl)
    mods = tags["modality"][:vl.shape[0]]
    mask = tags["out_mask"][:vl.shape[0]]

    def med(fn):
        ts = []
        for _ in range(reps):
            t0 = time.perf_counter()
            fn()
            ts.append(time.perf_counter() - t0)
        return statistics.median(ts) * 1e3

    comp = med(lambda: O.dit_block_compressed(x, wts, tags["pos"], w.heads, w.head_dim, k, near, w.n_video))
    plain = med(lambda: O.dit_block(x, wts, tags["pos"], w.heads, w.head_dim))
    eul = med(lambda: O.euler_step(vl, v, mods, mask, [0, 0.2, 0.5, 0], [0, 0.0769, 0.25, 0]))
    return {"workload": "tiny_block_f32", "tokens": w.n_tokens, "compressed_block_ms": comp,
            "block_ms": plain, "euler_step_ms": eul, "tokens_per_s_block": w.n_tokens / (plain / 1e3),
            "cores": blas_threads(), "timed": "directly, median of %d" % reps}


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:  # noqa: BLE001
        pass
    return len(os.sched_getaffinity(0))


# ---------------------------------------------------------------- reference arm

def run_reference(args, rank):
    if rank != 0:
        return
    w = S.WORKLOADS[args.workload]
    vals = []
    desc, threads = "", 1
    for i in range(args.warmup + args.steps):
        v, _, desc, threads = oracle_sample(w)
        if i >= args.warmup:
            vals.append(v)
    v = statistics.median(vals)
    sec = w.n_tokens * w.n_evals / v
    line = {
        "metric": metric_of(w), "value": v, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": sec * 1000.0, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "impl": "reference",
        "config": {"workload": args.workload, "layers": w.n_layers, "evals": w.n_evals,
                   "grid": "x".join(map(str, w.grid)), "tokens": w.n_tokens},
        "cpu_baseline": {"value": v, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": desc},
        "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- B200 arm

def build_backbone(w, device, rank, proj_fp8=False):
    dims = api.dims_of(w, proj_fp8=proj_fp8)
    layers, io = S.make_weights(w, device=device)
    if proj_fp8:
        layers = [api.quantize_block_weights(l) for l in layers]  # the bf16 projection weights are dropped
        torch.cuda.synchronize(device)
    bw = [api.BlockWeights(l) for l in layers]
    iow = api.IOWeights(io)
    tags = S.pack_tokens(w)
    seq = api.Sequence.from_workload(w, tags, device)
    bb = api.Backbone(dims, bw, iow, w.compress)
    inp = S.make_inputs(w, device="cpu", seed=R.input_seed(S.SEED_INPUTS, rank))
    return bb, seq, inp


def timed(fn, steps, stream, per_step=None):
    """Milliseconds for `steps` calls of fn on `stream` (events on both sides);
    with a list `per_step`, also an event after every call (appended: ms of
    each step), which adds no work between the steps."""
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    marks = [torch.cuda.Event(enable_timing=True) for _ in range(steps)] if per_step is not None else []
    start.record(stream)
    for i in range(steps):
        fn()
        if marks:
            marks[i].record(stream)
    end.record(stream)
    end.synchronize()
    prev = start
    for m in marks:
        per_step.append(prev.elapsed_time(m))
        prev = m
    return start.elapsed_time(end)


def run_fsdit(args, rank, world, local_rank):
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    B.build()
    L.load()
    w = S.WORKLOADS[args.workload]
    bb, seq, inp = build_backbone(w, device, rank, args.proj_fp8)
    vl0 = inp["video_lat"].to(device)
    al0 = inp["audio_lat"].to(device)
    text = inp["text_emb"].to(device)
    vl = torch.empty_like(vl0)
    al = torch.empty_like(al0)

    def step(compress=True):
        vl.copy_(vl0)
        al.copy_(al0)
        bb.sample(seq, w.video_clock, w.audio_clock, vl, text, al, compress=compress)

    gc.collect()
    torch.cuda.reset_peak_memory_stats(device)  # setup copies (e.g. weights before quantizing) do not count
    for _ in range(args.warmup):
        step()
    api.device_error()
    R.barrier(world, device)

    # Timed region: one pass captured in a CUDA graph with the library's
    # launch profiler off, replayed K times.  The per-kernel breakdown comes
    # from a second graph of the same pass captured with the profiler on (its
    # event pairs replay with every launch), replayed once after the timing.
    graph, launch_mode = None, "eager"
    if not args.eager:
        try:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                step()
            graph, launch_mode = g, "cuda_graph"
        except Exception as e:  # noqa: BLE001
            launch_mode = f"eager (graph capture failed: {type(e).__name__})"
            torch.cuda.synchronize()
    run = graph.replay if graph is not None else step
    if graph is not None:
        run()  # one untimed replay
    stream = torch.cuda.current_stream()
    clocks = ClockSampler(local_rank)
    R.barrier(world, device)
    step_ms = []
    t_ms = timed(run, args.steps, stream, step_ms)
    R.barrier(world, device)
    clk = clocks.stop()
    api.device_error()
    t_ms = R.max_over_ranks(t_ms, world, device)
    ms_per_step = t_ms / args.steps
    value = R.weak_scaling_value(w.n_tokens * w.n_evals, world, ms_per_step / 1000.0)
    del graph

    # the instrumented pass: per-kernel times, FLOPs and bytes
    L.profile_start(20000)
    prof_graph = None
    if launch_mode == "cuda_graph":
        prof_graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(prof_graph):
            step()
        prof_graph.replay()
    else:
        step()
    torch.cuda.synchronize()
    # the replay's own duration, next to the clean pass (the event pairs' cost)
    prof_ms = None
    if prof_graph is not None:
        prof_ms = timed(prof_graph.replay, 1, stream)
    prof = L.profile_stop()  # the last replay's launches
    prof_steps = 1
    del prof_graph
    api.device_error()

    # end to end through the public API: pinned host inputs -> device, sample, result -> host
    pin = {k: v.pin_memory() for k, v in inp.items() if k in ("video_lat", "audio_lat", "text_emb")}
    out_v = torch.empty_like(pin["video_lat"]).pin_memory()
    out_a = torch.empty_like(pin["audio_lat"]).pin_memory()

    def e2e_step():
        vl.copy_(pin["video_lat"], non_blocking=True)
        al.copy_(pin["audio_lat"], non_blocking=True)
        text.copy_(pin["text_emb"], non_blocking=True)
        bb.sample(seq, w.video_clock, w.audio_clock, vl, text, al)
        out_v.copy_(vl, non_blocking=True)
        out_a.copy_(al, non_blocking=True)

    e2e_step()
    R.barrier(world, device)
    e_ms = R.max_over_ranks(timed(e2e_step, args.steps, stream), world, device) / args.steps
    h2d = sum(t.numel() * t.element_size() for t in pin.values())
    d2h = out_v.numel() * 4 + out_a.numel() * 4

    # same backbone with compression off (the pages' ablation)
    full_ms = None
    if not args.no_full_compare and any(w.compress):
        step(compress=False)
        R.barrier(world, device)
        n_full = max(1, min(args.steps, 2))
        full_ms = R.max_over_ranks(timed(lambda: step(False), n_full, stream), world, device) / n_full

    peaks, peak_src = load_peaks()
    burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    gemm = {k: v for k, v in prof.items() if k.startswith("gemm")}
    g_ms = sum(v["ms"] for v in gemm.values())
    g_fl = sum(v["flops"] for v in gemm.values())
    g_n = sum(v["scopes"] for v in gemm.values())
    achieved = g_fl / (g_ms / 1e3) / 1e12 if g_ms > 0 else 0.0
    peak = float(peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops")))
    # an E4M3 contraction runs at twice the bf16 rate (nominal 4.5 vs 2.25 PFLOP/s dense)
    gemm_peak = 2.0 * peak if args.proj_fp8 else peak
    kernels = {}
    for k, v in sorted(prof.items(), key=lambda kv: -kv[1]["ms"]):
        e = {"launches_per_step": v["launches"] // prof_steps, "ms_per_step": v["ms"] / prof_steps}
        if v["flops"] > 0 and k.startswith(("gemm", "attention")):
            e["tflops"] = v["flops"] / (v["ms"] / 1e3) / 1e12
        if v["bytes"] > 0 and not k.startswith(("gemm", "attention")):
            e["gbs"] = v["bytes"] / (v["ms"] / 1e3) / 1e9
        kernels[k] = e
    launches_per_step = sum(v["launches"] for v in prof.values()) // prof_steps
    line = {
        "metric": metric_of(w), "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "e4m3 block projections (per-row scales), bf16 elsewhere" if args.proj_fp8 else "bf16",
        "data": "synthetic",
        "config": {"workload": args.workload + ("+fp8proj" if args.proj_fp8 else ""), "layers": w.n_layers,
                   "evals": w.n_evals,
                   "grid": "x".join(map(str, w.grid)), "tokens": w.n_tokens,
                   "kept_video_tokens": seq.n_keep, "parallelism": f"replicas x{world}",
                   "launch": launch_mode,
                   "l2": "inputs larger than L2: the bf16 weights (22.7 GB for 42 layers) stream from HBM "
                         "every evaluation"},
        "tensor_peak_frac": (pass_flops(w) / (ms_per_step / 1e3) / 1e12) / peak,
        "tensor_peak_fracs": peak_fracs(pass_flops(w) / (ms_per_step / 1e3) / 1e12, peak, burst),
        "roofline": {"bound": "tensor", "kernel": "tc_gemm_pair_kernel (all projections with M > 128)"
                     + (", E4M3 operands" if args.proj_fp8 else ""),
                     "achieved": achieved, "peak": gemm_peak, "unit": "TFLOP/s",
                     "frac": achieved / gemm_peak if gemm_peak else None,
                     "traffic": None if args.proj_fp8 else gemm_traffic(args.workload),
                     "peak_source": f"{peak_src} bf16_tflops_sustained" + (" x 2 (E4M3/bf16 nominal ratio)"
                                                                           if args.proj_fp8 else ""),
                     "launches_per_step": g_n // prof_steps,
                     "fracs": peak_fracs(achieved, gemm_peak, (2.0 if args.proj_fp8 else 1.0) * burst,
                                         (2.0 if args.proj_fp8 else 1.0) * NOMINAL_BF16_TFLOPS)},
        "kernels": kernels,
        "gpu_launches": launches_per_step * args.steps,
        "e2e": {"value": R.weak_scaling_value(w.n_tokens * w.n_evals, world, e_ms / 1000.0), "unit": UNIT,
                "ms_per_step": e_ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
    }
    if step_ms:
        srt = sorted(step_ms)
        line["step_ms"] = {"median": statistics.median(srt), "min": srt[0], "max": srt[-1],
                           "note": "this rank's timed steps, one event after each replay (the pages' protocol: "
                                   "median of repeated runs after warm-up)"}
    if prof_ms is not None:
        line["profiled_ms_per_step"] = prof_ms
    if full_ms is not None:
        line["uncompressed_ms_per_step"] = full_ms
        line["compression_speedup"] = full_ms / ms_per_step
    if clk is not None:
        line["clocks"] = clk
    # peak device memory of the warm-up, timed and comparison passes: every
    # device buffer (weights, latents, workspaces) is a torch allocation
    line["peak_mem_gb"] = round(torch.cuda.max_memory_allocated(device) / 1e9, 2)
    if args.proj_fp8:
        line["tensor_peak_basis"] = "bf16 sustained peak (attention still runs in bf16)"
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not args.proj_fp8:
        v, _, desc, threads = oracle_sample(w)
        line["cpu_baseline"] = {"value": v, "unit": UNIT, "cores": threads, "kind": "oracle",
                                "sample": desc, "projected": True, "tiny": oracle_tiny()}
    if rank == 0:
        print(json.dumps(line), flush=True)


def main():
    args = parse()
    rank, world, local_rank = R.env()
    if args.impl == "reference":
        run_reference(args, rank)
        return
    if world > 1:
        torch.cuda.set_device(local_rank)
    R.init(world, backend="nccl")
    try:
        run_fsdit(args, rank, world, local_rank)
    finally:
        R.shutdown(world)


if __name__ == "__main__":
    main()
