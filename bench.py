#!/usr/bin/env python
"""Benchmark of the fused W8A8 block-scaled MoE layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload prefill|decode|mid|tiny]
                    [--impl ours|reference]

One step = one full fused layer (routing/permutation, activation quant,
GEMM1 gate/up + SwiGLU + FP8 requant, GEMM2 down + weighted combine, bf16
output) through the C ABI on one batch of synthetic, seeded inputs already
resident in HBM.  With N GPUs (torchrun) every rank runs an independent
replica of the workload (weak scaling); time is the max over ranks.

Prints one JSON line (rank 0).  `value` is the effective throughput in
TFLOP/s of algorithmic work (6*T*k*H*I flops per layer); `ms_per_step` is the
layer latency.  The reference arm (--impl reference) times the CPU oracle on
a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "fused MoE layer µs & TFLOPS/GB/s as % of B200 FP8-tensor/HBM roofline"
FP8_OVER_BF16 = 2.0        # nominal dense FP8 / BF16 tensor ratio (4.5 / 2.25 PFLOP/s)
FP4_OVER_BF16 = 4.0        # nominal dense FP4 / BF16 tensor ratio (9 / 2.25 PFLOP/s)
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
ROUTE_CHUNK = 1024         # (token, slot) pairs per routing chunk
ROUTE_SMALL_CHUNKS = 8     # up to this many chunks, routing is one single-CTA launch


def kernels_per_layer(T: int, k: int, fused: bool = False) -> int:
    """Kernel launches of one fused layer: routing (one launch for inputs of
    at most 8 chunks of 1024 pairs, else histogram/scan/scatter), quant,
    GEMM1 and GEMM2 (one fused-expert launch when the plan fuses them) and
    the combine."""
    nchunks = (T * k + ROUTE_CHUNK - 1) // ROUTE_CHUNK
    return (1 if nchunks <= ROUTE_SMALL_CHUNKS else 3) + (3 if fused else 4)


# Slices of the prefill and decode workloads (same H, I, top-k and routing,
# 32 experts) that keep a profiler capture to a couple of GB on the device.
PROFILE_SLICES = {
    "prefill_slice": synth.MoEConfig("prefill_slice", 1024, 7168, 2048, 32, 8, "zipf"),
    "decode_slice": synth.MoEConfig("decode_slice", 64, 7168, 2048, 32, 8),
}


# DRAM bytes (read + write) per launch of the dominant kernel, GEMM1, taken
# from the one-pass ncu launch list of `bench.py --workload <name>` on the full
# workload (see the launch-list summaries under profiles/).  A figure is
# reported only while the GEMM sources still hash to the digest it was taken
# with.
GEMM_SOURCES = ("grouped_gemm.cu", "gemm_common.cuh", "ptx.cuh", "common.cuh")  # its code
MEASURED_TRAFFIC = {  # workload -> (source digest, bytes per GEMM1 launch)
    "prefill": ("705b532ef98dca09", 6003600000),
    "decode": ("705b532ef98dca09", 6525600000),
}


def gemm_source_digest() -> str:
    h = hashlib.sha256()
    for name in GEMM_SOURCES:
        with open(os.path.join(ROOT, "fp8_block_scaled_route_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def measured_traffic(workload: str):
    entry = MEASURED_TRAFFIC.get(workload)
    if entry is None:
        return None
    try:
        return entry[1] if gemm_source_digest() == entry[0] else None
    except OSError:
        return None


def workload_desc(cfg: synth.MoEConfig) -> str:
    r = "zipf(1.2)-biased routing" if cfg.routing == "zipf" else "logits ~N(0,1)"
    return (f"{cfg.name}: T={cfg.T} H={cfg.H} I={cfg.I} E={cfg.E} top-{cfg.k}, {r}, "
            f"FP8 e4m3 weights with fp32 128x128 block scales, bf16 in/out")


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p["bf16_tflops_sustained"]), \
            "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, FALLBACK_BF16_TFLOPS, "fallback"


FUSION_MODES = {"auto": 0, "on": 1, "off": 2}   # MOE_FUSION_AUTO / ON / OFF


def stage_dict(stage_ms, fused: bool) -> dict:
    """Per-stage device times (µs) from the layer's stage events (each
    interval includes one event record, ~2-3 µs)."""
    us = [float(v) * 1e3 for v in stage_ms]
    if fused:   # events 3 and 4 are recorded back to back after the fused launch
        return {"route": us[0], "quant": us[1], "experts": us[2], "finish": us[4]}
    return dict(zip(["route", "quant", "gemm1", "gemm2", "finish"], us))


def work_counts(cfg: synth.MoEConfig, topk_ids: torch.Tensor):
    """Algorithmic flops and bytes of the layer and of GEMM1, from the actual
    routing (only experts with at least one row are read)."""
    ids = topk_ids.flatten()
    valid = ids[(ids >= 0) & (ids < cfg.E)]
    R = int(valid.numel())
    touched = int(torch.unique(valid).numel())
    H, I = cfg.H, cfg.I
    w13_b = 2 * I * H + 4 * (2 * I // 128) * (H // 128)
    w2_b = H * I + 4 * (H // 128) * (I // 128)
    flops = 6.0 * R * H * I
    layer_bytes = touched * (w13_b + w2_b) + 2 * cfg.T * H * 2 + cfg.T * cfg.k * 8
    g1_flops = 4.0 * R * H * I
    # GEMM1 reads the touched gate/up weights, the FP8 activations and their
    # scales, and writes the FP8 intermediate with its scales
    g1_bytes = touched * w13_b + R * H + 4 * R * (H // 128) + R * I + 4 * R * (I // 128)
    # the fused-expert launch reads the touched weights of both GEMMs and the
    # grouped FP8 activation rows with their scales, and writes the fp32 pair rows
    fx_bytes = touched * (w13_b + w2_b) + R * H + 4 * R * (H // 128) + 4 * R * H
    return dict(R=R, touched=touched, flops=flops, bytes=layer_bytes, g1_flops=g1_flops,
                g1_bytes=g1_bytes, fx_bytes=fx_bytes)


class ClockSampler:
    """nvidia-smi clocks/throttle sampling while the timed region runs."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: str):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.index, f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out = ""
        self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
            except ValueError:
                continue
            for name, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": smax, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


def max_over_ranks(values, pg=None, device="cpu"):
    """Element-wise maximum of a list of floats over all ranks of the default
    process group (a collective: every rank must call it, in the same order);
    the values unchanged when there is no group."""
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    if pg is not None:
        pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return [float(v) for v in t.cpu()]


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def sample_tokens(cfg, n):
    step = max(1, cfg.T // max(1, n))
    return list(range(0, cfg.T, step))[:n]


def oracle_sample_rate(inp, cfg, n_tok, repeats=1):
    """Times the CPU oracle (per-token form) on n_tok tokens; returns
    (flops per sample, seconds per sample, threads)."""
    import oracle
    toks = sample_tokens(cfg, n_tok)
    sub = synth.compact_experts(inp, toks)
    args = (sub["x"], sub["topk_ids"], sub["topk_w"], sub["w13"], sub["w13_scale"], sub["w2"],
            sub["w2_scale"], np.arange(len(toks), dtype=np.int32))
    valid = int(((sub["topk_ids"] >= 0)).sum())
    flops = 6.0 * valid * cfg.H * cfg.I
    times = []
    for _ in range(repeats):
        t0 = time.perf_counter()
        oracle.moe_tokens(*args)
        times.append(time.perf_counter() - t0)
    return flops, times, oracle.num_threads(), len(toks)


def run_reference(args, cfg):
    world, rank, local = dist_env()
    if rank != 0:
        return 0
    import oracle
    oracle.build()
    dev = f"cuda:{local}" if torch.cuda.is_available() else "cpu"
    big = cfg.H * cfg.I * cfg.E > (1 << 30)
    inp = synth.make_moe_inputs(cfg, seed=0, device=dev if big else "cpu")
    threads = oracle.num_threads()
    # size one step to about two seconds of oracle work
    n = max(1, min(cfg.T, threads))
    f, t, _, _ = oracle_sample_rate(inp, cfg, n)
    n = int(max(1, min(cfg.T, n * max(1.0, 2.0 / max(t[0], 1e-3)))))
    flops, times, threads, ntok = oracle_sample_rate(inp, cfg, n, repeats=args.warmup + args.steps)
    timed = times[args.warmup:]
    sec = sum(timed) / len(timed)
    value = flops / sec / 1e12
    sample = f"{ntok} of {cfg.T} tokens per step (per-token oracle form), all top-{cfg.k} slots"
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": sec * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "fp32 (fp8 e4m3 operands)",
        "data": "synthetic", "impl": "reference",
        "config": {"workload": workload_desc(cfg), "sample": sample},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_ours(args, cfg):
    import fp8_block_scaled_route_b200 as moe
    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
        pg = dist
    moe.lib()
    moe.moe_set_expert_fusion(FUSION_MODES[args.fusion])
    inp = synth.make_moe_inputs(cfg, seed=rank, device=dev)
    T, H, I, E, k = cfg.T, cfg.H, cfg.I, cfg.E, cfg.k
    ws = torch.empty(moe.moe_workspace_size(T, H, I, E, k), dtype=torch.uint8, device=dev)
    out = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)
    counts = work_counts(cfg, inp["topk_ids"])
    plan = moe.moe_fp8_fused_plan(T, H, I, E, k)

    def step():
        moe.moe_fp8_fused(inp["x"], inp["topk_ids"], inp["topk_w"], inp["w13"], inp["w13_scale"],
                          inp["w2"], inp["w2_scale"], out, ws, stream=stream)

    # warm-up
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    st = moe.moe_get_device_status(ws, stream=stream)
    if st != moe.MOE_OK:
        raise RuntimeError(f"device status after warm-up: {moe.moe_status_string(st)}")

    # stage events for the dominant kernel (GEMM1) over the timed region
    stage_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(args.steps)]
    for evs in stage_ev:          # torch creates the CUDA event on its first record
        for e in evs:
            e.record(stream)
    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
    smi_index = vis.split(",")[local] if vis else str(local)
    clocks = ClockSampler(smi_index)
    clocks.start()
    time.sleep(0.3)
    if pg:
        pg.barrier()
    torch.cuda.synchronize(dev)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    # the timed region: K layers back to back; the library records only the two
    # events around the dominant kernel (GEMM1, or the fused-expert launch),
    # as each event record costs ~2-3 µs of GPU time
    dom_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    for evs in dom_ev:
        for e in evs:
            e.record(stream)
    torch.cuda.synchronize(dev)
    t_start.record(stream)
    for i in range(args.steps):
        moe.moe_set_stage_events([None, None, dom_ev[i][0], dom_ev[i][1], None, None])
        step()
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    moe.moe_set_stage_events(None)
    if pg:
        pg.barrier()
    elapsed_ms = t_start.elapsed_time(t_end)
    dom_ms = float(np.mean([a.elapsed_time(b) for a, b in dom_ev]))
    # the same K layers again with all six stage events, for the per-stage
    # breakdown only
    s_start = torch.cuda.Event(enable_timing=True)
    s_end = torch.cuda.Event(enable_timing=True)
    s_start.record(stream)
    for i in range(args.steps):
        moe.moe_set_stage_events(stage_ev[i])
        step()
    s_end.record(stream)
    torch.cuda.synchronize(dev)
    moe.moe_set_stage_events(None)
    staged_ms = s_start.elapsed_time(s_end) / args.steps
    if pg:
        pg.barrier()
    st = moe.moe_get_device_status(ws, stream=stream)
    if st != moe.MOE_OK:
        raise RuntimeError(f"device status after timing: {moe.moe_status_string(st)}")
    stages = np.array([[ev[j].elapsed_time(ev[j + 1]) for j in range(5)] for ev in stage_ev])
    stage_ms = stages.mean(axis=0)   # route, quant, gemm1, gemm2, finish

    # end to end through the C ABI with host buffers: every step uploads its
    # inputs from pinned host memory and downloads its output.  The copies of
    # neighbouring steps overlap the layer on a second stream (double-buffered
    # device inputs and outputs), as a serving loop would run them; the timed
    # region ends when the last step's output is on the host.
    x_h = inp["x"].cpu().pin_memory()
    ids_h = inp["topk_ids"].cpu().pin_memory()
    w_h = inp["topk_w"].cpu().pin_memory()
    out_h = [torch.empty(T, H, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    bufs = [dict(x=torch.empty_like(inp["x"]), ids=torch.empty_like(inp["topk_ids"]),
                 w=torch.empty_like(inp["topk_w"]), out=torch.empty_like(out)) for _ in range(2)]
    copy = torch.cuda.Stream(dev)

    def e2e_run(n):
        h2d_done = [torch.cuda.Event() for _ in range(2)]
        layer_done = [torch.cuda.Event() for _ in range(2)]
        d2h_done = [torch.cuda.Event() for _ in range(2)]
        used = [False, False]

        def upload(i):
            b = bufs[i % 2]
            if used[i % 2]:
                copy.wait_event(layer_done[i % 2])  # layer i-2 has read these inputs
            with torch.cuda.stream(copy):
                b["x"].copy_(x_h, non_blocking=True)
                b["ids"].copy_(ids_h, non_blocking=True)
                b["w"].copy_(w_h, non_blocking=True)
            h2d_done[i % 2].record(copy)

        copy.wait_stream(stream)
        upload(0)
        for i in range(n):
            b = bufs[i % 2]
            stream.wait_event(h2d_done[i % 2])
            if used[i % 2]:
                stream.wait_event(d2h_done[i % 2])  # output of step i-2 is on the host
            moe.moe_fp8_fused(b["x"], b["ids"], b["w"], inp["w13"], inp["w13_scale"], inp["w2"],
                              inp["w2_scale"], b["out"], ws, stream=stream)
            layer_done[i % 2].record(stream)
            used[i % 2] = True
            if i + 1 < n:
                upload(i + 1)
            copy.wait_event(layer_done[i % 2])
            with torch.cuda.stream(copy):
                out_h[i % 2].copy_(b["out"], non_blocking=True)
            d2h_done[i % 2].record(copy)
        stream.wait_stream(copy)

    e2e_run(args.warmup)
    if pg:
        pg.barrier()
    torch.cuda.synchronize(dev)
    e_start = torch.cuda.Event(enable_timing=True)
    e_end = torch.cuda.Event(enable_timing=True)
    e_start.record(stream)
    e2e_run(args.steps)
    e_end.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = e_start.elapsed_time(e_end)

    # the decode workload (weight-streaming, HBM-bound) in the same run: its
    # own seeded inputs, the same warm-up and number of timed steps
    dec = None
    if cfg.name == "prefill" and not args.no_decode:
        dcfg = synth.CONFIGS["decode"]
        dinp = synth.make_moe_inputs(dcfg, seed=rank, device=dev)
        dws = torch.empty(moe.moe_workspace_size(dcfg.T, dcfg.H, dcfg.I, dcfg.E, dcfg.k),
                          dtype=torch.uint8, device=dev)
        dout = torch.empty(dcfg.T, dcfg.H, dtype=torch.bfloat16, device=dev)
        if pg:
            pg.barrier()
        dec_ms, dec_stages = timed_layer(
            lambda: moe.moe_fp8_fused(dinp["x"], dinp["topk_ids"], dinp["topk_w"], dinp["w13"],
                                      dinp["w13_scale"], dinp["w2"], dinp["w2_scale"], dout, dws,
                                      stream=stream), args, dws, stream, dev)
        dec = (dcfg, work_counts(dcfg, dinp["topk_ids"]), dec_stages)
        del dinp, dws, dout
        # and the mid workload (the shape the fused-expert launch is chosen for)
        mcfg = synth.CONFIGS["mid"]
        minp = synth.make_moe_inputs(mcfg, seed=rank, device=dev)
        mws = torch.empty(moe.moe_workspace_size(mcfg.T, mcfg.H, mcfg.I, mcfg.E, mcfg.k),
                          dtype=torch.uint8, device=dev)
        mout = torch.empty(mcfg.T, mcfg.H, dtype=torch.bfloat16, device=dev)
        if pg:
            pg.barrier()
        mid_ms, mid_stages = timed_layer(
            lambda: moe.moe_fp8_fused(minp["x"], minp["topk_ids"], minp["topk_w"], minp["w13"],
                                      minp["w13_scale"], minp["w2"], minp["w2_scale"], mout, mws,
                                      stream=stream), args, mws, stream, dev)
        mid = (mcfg, work_counts(mcfg, minp["topk_ids"]), mid_stages,
               moe.moe_fp8_fused_plan(mcfg.T, mcfg.H, mcfg.I, mcfg.E, mcfg.k))
        del minp, mws, mout
    else:
        dec_ms = 0.0
        mid_ms = 0.0
        mid = None
    clocks.stop()

    # max over ranks
    elapsed_ms, e2e_ms, dec_ms, mid_ms = max_over_ranks([elapsed_ms, e2e_ms, dec_ms, mid_ms], pg,
                                                        dev)

    if rank == 0:
        ms_step = elapsed_ms / args.steps
        value = world * counts["flops"] / (ms_step * 1e-3) / 1e12
        e2e_value = world * counts["flops"] / (e2e_ms / args.steps * 1e-3) / 1e12
        hbm, bf16, bf16_sus, src = load_peaks()
        # the dominant kernel: GEMM1, or the fused-expert launch (both GEMMs;
        # it alone sits between stage events 2 and 3), timed in the timed region
        fused = plan["fused"]
        g1_ms = dom_ms
        k_flops = counts["flops"] if fused else counts["g1_flops"]
        k_bytes = counts["fx_bytes"] if fused else counts["g1_bytes"]
        g1_tflops = k_flops / (g1_ms * 1e-3) / 1e12
        g1_gbs = k_bytes / (g1_ms * 1e-3) / 1e9
        fp8_peak = bf16 * FP8_OVER_BF16
        t_tensor = k_flops / (fp8_peak * 1e12)
        t_hbm = k_bytes / (hbm * 1e9)
        if t_tensor >= t_hbm:
            roof = {"bound": "tensor", "achieved": g1_tflops, "peak": fp8_peak, "unit": "TFLOP/s",
                    "frac": g1_tflops / fp8_peak}
        else:
            roof = {"bound": "hbm", "achieved": g1_gbs, "peak": hbm, "unit": "GB/s",
                    "frac": g1_gbs / hbm}
        roof.update({"traffic": None if fused else measured_traffic(cfg.name),
                     "kernel": "fused expert (gate/up + SwiGLU + FP8 requant on chip + down)"
                     if fused else "grouped GEMM1 (gate/up + SwiGLU + FP8 requant)",
                     "peak_source": f"{src} (FP8 = bf16 burst x {FP8_OVER_BF16:g})"
                     if roof["bound"] == "tensor" else f"{src} copy bandwidth"})
        layer_gbs = counts["bytes"] / (ms_step * 1e-3) / 1e9
        layer_tflops = counts["flops"] / (ms_step * 1e-3) / 1e12
        layer_frac = max(counts["flops"] / (fp8_peak * 1e12), counts["bytes"] / (hbm * 1e9)) / \
            (ms_step * 1e-3)
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "fp8_e4m3 (fp32 accumulate)", "data": "synthetic",
            "config": {"workload": workload_desc(cfg), "l2": "inputs larger than L2 (no flush)"
                       if counts["touched"] * 3 * H * I > 126e6 else "working set fits L2",
                       "parallelism": f"replicas x{world}", "seed": "rank"},
            "layer": {"us": ms_step * 1e3, "tflops": layer_tflops, "gbs": layer_gbs,
                      "roofline_frac": layer_frac, "rows": counts["R"],
                      "experts_touched": counts["touched"], "alg_bytes": counts["bytes"],
                      "alg_flops": counts["flops"]},
            "stages_us": stage_dict(stage_ms, fused),
            "stages_note": "per-stage device times from a second pass of the same steps after "
                           "the timed region, with all six stage events; the roofline kernel is "
                           "timed inside the timed region",
            "ms_per_step_with_stage_events": staged_ms,
            "plan": plan,
            "roofline": roof,
            "e2e": {"value": e2e_value, "unit": "TFLOP/s",
                    "h2d_bytes_per_step": T * H * 2 + T * k * 8, "d2h_bytes_per_step": T * H * 2},
            "gpu_launches": kernels_per_layer(T, k, fused) * args.steps,
            "clocks": clocks.summary(),
        }
        if dec is not None:
            dcfg, dc, dst = dec
            d_gbs = dc["bytes"] / (dec_ms * 1e-3) / 1e9
            g1_gbs_d = dc["g1_bytes"] / (float(dst[2]) * 1e-3) / 1e9
            line["decode"] = {
                "workload": workload_desc(dcfg), "us": dec_ms * 1e3, "steps": args.steps,
                "tflops": dc["flops"] / (dec_ms * 1e-3) / 1e12, "gbs": d_gbs,
                "hbm_frac": d_gbs / hbm, "alg_bytes": dc["bytes"],
                "experts_touched": dc["touched"],
                "stages_us": {n: float(v) * 1e3 for n, v in
                              zip(["route", "quant", "gemm1", "gemm2", "finish"], dst)},
                "gemm1_gbs": g1_gbs_d, "gemm1_hbm_frac": g1_gbs_d / hbm,
                "gemm1_traffic": measured_traffic(dcfg.name),
                "peak_source": f"{src} copy bandwidth",
                "l2": "inputs larger than L2 (no flush)",
                "gpu_launches": kernels_per_layer(dcfg.T, dcfg.k) * args.steps}
        if mid is not None:
            mcfg, mc, mst, mplan = mid
            m_gbs = mc["bytes"] / (mid_ms * 1e-3) / 1e9
            line["mid"] = {
                "workload": workload_desc(mcfg), "us": mid_ms * 1e3, "steps": args.steps,
                "tflops": mc["flops"] / (mid_ms * 1e-3) / 1e12, "gbs": m_gbs,
                "hbm_frac": m_gbs / hbm, "alg_bytes": mc["bytes"],
                "experts_touched": mc["touched"], "plan": mplan,
                "stages_us": stage_dict(mst, mplan["fused"]),
                "note": "timed region without events; stages from a second pass",
                "peak_source": f"{src} copy bandwidth",
                "gpu_launches": kernels_per_layer(mcfg.T, mcfg.k, mplan["fused"]) * args.steps}
        if world == 1 and not args.no_cpu_baseline:
            import oracle
            oracle.build()
            threads = oracle.num_threads()
            n = max(1, min(T, threads))
            f, t, _, _ = oracle_sample_rate(inp, cfg, n)
            target = 10.0
            n2 = int(max(1, min(T, n * max(1.0, target / max(t[0], 1e-3)))))
            if n2 > n:
                f, t, threads, n = oracle_sample_rate(inp, cfg, n2)
            line["cpu_baseline"] = {"value": f / t[0] / 1e12, "unit": "TFLOP/s", "cores": threads,
                                    "kind": "oracle",
                                    "sample": f"{n} of {T} tokens, per-token oracle form, "
                                              f"{t[0]:.1f} s"}
        print(json.dumps(line), flush=True)
    if pg:
        pg.barrier()
        pg.destroy_process_group()
    return 0


def run_swiglu(args):
    """Standalone SwiGLU + MXFP8 quantisation at the three (M, K) sizes;
    each iteration timed alone with an L2 flush (256 MB write) in between."""
    import fp8_block_scaled_route_b200 as moe
    torch.cuda.set_device(0)
    hbm, _, _, src = load_peaks()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    res = []
    shapes = synth.SWIGLU_SHAPES
    if args.swiglu_shape:
        M, K = (int(v) for v in args.swiglu_shape.lower().split("x"))
        shapes = ((M, K),)
    for (M, K) in shapes:
        for variant in ("normal", "block_scaled"):
            x = synth.make_swiglu_input(M, K, variant, seed=0, device="cuda")
            out = torch.empty(M, K, dtype=torch.uint8, device="cuda")
            sc = torch.empty(M, K // 32, dtype=torch.uint8, device="cuda")
            for _ in range(args.warmup):
                moe.swiglu_mxfp8_quant(x, out, sc)
            times = []
            for _ in range(args.steps):
                flush.fill_(1)
                a = torch.cuda.Event(enable_timing=True)
                b = torch.cuda.Event(enable_timing=True)
                a.record()
                moe.swiglu_mxfp8_quant(x, out, sc)
                b.record()
                torch.cuda.synchronize()
                times.append(a.elapsed_time(b))
            ms = statistics.median(times)
            # back to back: many calls captured in one CUDA graph and replayed
            # between two events (no flush, L2-warm inputs): the device-side
            # cost per call without the host's launch overhead
            reps = 1000 if M * K < (1 << 24) else 50
            g = torch.cuda.CUDAGraph()
            cap = torch.cuda.Stream()
            cap.wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(cap):
                with torch.cuda.graph(g, stream=cap):
                    for _ in range(reps):
                        moe.swiglu_mxfp8_quant(x, out, sc, stream=cap)
            torch.cuda.current_stream().wait_stream(cap)
            g.replay()
            torch.cuda.synchronize()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record()
            g.replay()
            b.record()
            torch.cuda.synchronize()
            ms_b2b = a.elapsed_time(b) / reps
            del g
            nbytes = 4 * M * K + M * K + M * K // 32
            res.append({"M": M, "K": K, "input": variant, "us": ms * 1e3,
                        "gbs": nbytes / (ms * 1e-3) / 1e9, "hbm_frac": nbytes / (ms * 1e-3) / 1e9 / hbm,
                        "us_back_to_back": ms_b2b * 1e3, "back_to_back_launches": reps})
    line = {"metric": "SwiGLU+MXFP8 quantisation µs and GB/s as % of HBM", "unit": "us",
            "higher_is_better": False, "steps": args.steps, "warmup": args.warmup,
            "peak_hbm_gbs": hbm, "peak_source": src, "data": "synthetic",
            "config": {"workload": "bf16 [M,2K] (gate|up) -> FP8 [M,K] + E8M0 per 32",
                       "l2": "us: flushed before every timed launch (median of single launches); "
                             "us_back_to_back: mean over back-to-back calls replayed from one CUDA graph, no flush"},
            "results": res}
    print(json.dumps(line), flush=True)
    return 0


def run_router(args, cfg):
    """The router (moe_router_topk) and the router with the grouping in one
    call (moe_router_route) on a workload's routing shape: logits fp32 [T, E]
    ~ N(0,1) (plus the Zipf bias for the prefill workload), top-k."""
    import fp8_block_scaled_route_b200 as moe
    torch.cuda.set_device(0)
    T, E, k = cfg.T, cfg.E, cfg.k
    g = torch.Generator().manual_seed(0)
    logits = torch.randn(T, E, generator=g)
    if cfg.routing == "zipf":
        ranks = torch.randperm(E, generator=g).float() + 1.0
        logits = logits - synth.ZIPF_S * torch.log(ranks)[None, :]
    logits = logits.cuda()
    ids = torch.empty(T, k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, k, dtype=torch.float32, device="cuda")
    m = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(T * k, dtype=torch.int32, device="cuda")
    inv = torch.empty(T * k, dtype=torch.int32, device="cuda")
    ws = torch.empty(moe.moe_route_workspace_size(T, k, E), dtype=torch.uint8, device="cuda")

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(args.steps):
            fn()
        b.record()
        torch.cuda.synchronize()
        return a.elapsed_time(b) / args.steps * 1e3

    us_topk = timed(lambda: moe.moe_router_topk(logits, ids, w))
    us_route = timed(lambda: moe.moe_route_permute(ids, E, m, perm, inv, ws))
    us_both = timed(lambda: moe.moe_router_route(logits, k, ids, w, m, perm, inv, ws))
    line = {"metric": "router and routing latency", "unit": "us", "higher_is_better": False,
            "steps": args.steps, "warmup": args.warmup, "n_gpus": 1, "data": "synthetic",
            "config": {"workload": f"{cfg.name} routing: T={T} E={E} top-{k}, logits fp32"},
            "router_topk_us": us_topk, "route_permute_us": us_route,
            "router_route_one_call_us": us_both,
            "logits_read_gbs": T * E * 4 / (us_topk * 1e-6) / 1e9}
    print(json.dumps(line), flush=True)
    return 0


def run_mx_gemm(args, cfg):
    """MXFP8 grouped GEMM (block-scaled tensor core path) on the gate/up GEMM
    of a workload: A = the workload's routed rows [T*k, H], B = gated weights
    [E, 2I, H], group sizes from its routing; activations and weights drawn
    as N(0,1) / N(0,1/H) with per-32 magnitudes 2^U{-4..4}, quantised to
    MXFP8.  The same shape through the fp32-block-scaled grouped GEMM
    (fp8_groupwise_moe_gemm) is timed beside it.  Inputs exceed L2."""
    import fp8_block_scaled_route_b200 as moe
    torch.cuda.set_device(0)
    hbm, bf16, _, src = load_peaks()
    fp8_peak = bf16 * FP8_OVER_BF16
    ids = synth.make_moe_inputs(cfg, seed=0, device="cuda", weights=False)["topk_ids"]
    sizes = torch.bincount(ids.flatten().long(), minlength=cfg.E).cpu().tolist()
    R, N, K, E = sum(sizes), 2 * cfg.I, cfg.H, cfg.E
    inp = synth.make_mx_gemm_inputs(R, N, K, E, seed=1, device="cuda", group_sizes=sizes)
    a_sf = inp["a_sf"].view(R, K // 128, 4).permute(1, 0, 2).contiguous()
    b_sf = torch.empty(E * N, K // 32, dtype=torch.uint8, device="cuda")
    moe.mxfp8_tile_scales(inp["b_sf"].view(E * N, K // 32), b_sf)
    out = torch.empty(R, N // 2, dtype=torch.bfloat16, device="cuda")

    def mx():
        moe.mxfp8_moe_gemm(inp["a"], inp["b"], a_sf, b_sf, inp["m_indptr"], out, True, "MN")

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(args.steps):
            fn()
        b.record()
        torch.cuda.synchronize()
        return a.elapsed_time(b) / args.steps

    ms_mx = timed(mx)
    del a_sf
    fp = synth.make_grouped_gemm_inputs(R, N, K, E, seed=1, device="cuda", group_sizes=sizes)
    a_mn = fp["a_scale"].t().contiguous()

    def fp32_scaled():
        moe.fp8_groupwise_moe_gemm(fp["a"], fp["b"], a_mn, fp["b_scale"], fp["m_indptr"], out,
                                   "MN", (1, 128, 128), True, -1, -1)

    ms_fp = timed(fp32_scaled)
    flops = 2.0 * R * N * K
    touched = sum(1 for x in sizes if x > 0)
    nbytes = touched * N * K * (1 + 1 / 32) + R * K * (1 + 1 / 32) + R * (N // 2) * 2
    tf = flops / (ms_mx * 1e-3) / 1e12
    line = {"metric": "MXFP8 grouped GEMM (gate/up + SwiGLU) TFLOP/s", "value": tf,
            "unit": "TFLOP/s", "higher_is_better": True, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_mx, "n_gpus": 1, "data": "synthetic",
            "dtype": "mxfp8 e4m3 + e8m0 per 32 (fp32 accumulate)",
            "config": {"workload": f"{cfg.name} gate/up GEMM: R={R} N={N} K={K} E={E}, "
                                   f"group sizes from its routing",
                       "l2": "inputs larger than L2 (no flush)"},
            "roofline": {"bound": "tensor", "achieved": tf, "peak": fp8_peak, "unit": "TFLOP/s",
                         "frac": tf / fp8_peak, "traffic": None,
                         "peak_source": f"{src} (FP8 = bf16 burst x {FP8_OVER_BF16:g})",
                         "alg_bytes": nbytes, "gbs": nbytes / (ms_mx * 1e-3) / 1e9},
            "fp32_block_scaled_same_shape": {"ms": ms_fp,
                                             "tflops": flops / (ms_fp * 1e-3) / 1e12},
            "gpu_launches": args.steps}
    print(json.dumps(line), flush=True)
    return 0


def run_nvfp4_gemm(args, cfg):
    """NVFP4 grouped GEMM (packed E2M1 operands, E4M3 scales per 16 K
    elements, per-expert alpha) on the gate/up GEMM of a workload: A = the
    workload's routed rows [T*k, H], B = gated weights [E, 2I, H], group sizes
    from its routing; activations N(0,1) and weights N(0,1/H) with per-16
    magnitudes 2^U{-3..3}, quantised to NVFP4 with global scales
    448*6/amax.  Inputs exceed L2."""
    import fp8_block_scaled_route_b200 as moe
    torch.cuda.set_device(0)
    _, bf16, _, src = load_peaks()
    fp4_peak = bf16 * FP4_OVER_BF16
    ids = synth.make_moe_inputs(cfg, seed=0, device="cuda", weights=False)["topk_ids"]
    sizes = torch.bincount(ids.flatten().long(), minlength=cfg.E).cpu().tolist()
    R, N, K, E = sum(sizes), 2 * cfg.I, cfg.H, cfg.E
    inp = synth.make_nvfp4_gemm_inputs(R, N, K, E, seed=1, device="cuda", group_sizes=sizes)
    a, b = inp["a_packed"], inp["b_packed"]
    del inp["a"], inp["b"]
    a_sf = inp["a_sf"].view(torch.uint8).view(R, K // 64, 4).permute(1, 0, 2).contiguous()
    b_sf = torch.empty(E * N, K // 16, dtype=torch.uint8, device="cuda")
    moe.nvfp4_tile_scales(inp["b_sf"].view(torch.uint8).view(E * N, K // 16), b_sf)
    alpha = (1.0 / (inp["ga"] * inp["gb"].double())).float()
    out = torch.empty(R, N // 2, dtype=torch.bfloat16, device="cuda")

    def step():
        moe.nvfp4_moe_gemm(a, b, a_sf, b_sf, alpha, inp["m_indptr"], out, True, "MN")

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    ev0.record()
    for _ in range(args.steps):
        step()
    ev1.record()
    torch.cuda.synchronize()
    st = moe.moe_get_device_status(None)
    if st != moe.MOE_OK:
        raise RuntimeError(f"device status: {moe.moe_status_string(st)}")
    ms = ev0.elapsed_time(ev1) / args.steps
    flops = 2.0 * R * N * K
    touched = sum(1 for x in sizes if x > 0)
    nbytes = touched * N * K * (0.5 + 1 / 16) + R * K * (0.5 + 1 / 16) + R * (N // 2) * 2
    tf = flops / (ms * 1e-3) / 1e12
    line = {"metric": "NVFP4 grouped GEMM (gate/up + SwiGLU) TFLOP/s", "value": tf,
            "unit": "TFLOP/s", "higher_is_better": True, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "n_gpus": 1, "data": "synthetic",
            "dtype": "nvfp4 e2m1 + e4m3 per 16 + fp32 global (fp32 accumulate)",
            "config": {"workload": f"{cfg.name} gate/up GEMM: R={R} N={N} K={K} E={E}, "
                                   f"group sizes from its routing",
                       "l2": "inputs larger than L2 (no flush)"},
            "roofline": {"bound": "tensor", "achieved": tf, "peak": fp4_peak, "unit": "TFLOP/s",
                         "frac": tf / fp4_peak, "traffic": None,
                         "peak_source": f"{src} (FP4 = bf16 burst x {FP4_OVER_BF16:g})",
                         "alg_bytes": nbytes, "gbs": nbytes / (ms * 1e-3) / 1e9},
            "gpu_launches": args.steps}
    print(json.dumps(line), flush=True)
    return 0


def timed_layer(step, args, ws, stream, dev):
    """Warm-up, then args.steps timed calls of one fused layer back to back,
    then as many again with its five stage events: (ms per step of the
    first, mean stage times [route, quant, gemm1, gemm2, finish] in ms of the
    second).  Raises on a device status other than MOE_OK."""
    import fp8_block_scaled_route_b200 as moe
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(args.steps)]
    for evs in ev:
        for e in evs:
            e.record(stream)
    torch.cuda.synchronize(dev)
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for i in range(args.steps):
        step()
    b.record(stream)
    torch.cuda.synchronize(dev)
    for i in range(args.steps):
        moe.moe_set_stage_events(ev[i])
        step()
    torch.cuda.synchronize(dev)
    moe.moe_set_stage_events(None)
    st = moe.moe_get_device_status(ws, stream=stream)
    if st != moe.MOE_OK:
        raise RuntimeError(f"device status: {moe.moe_status_string(st)}")
    stages = np.array([[e[j].elapsed_time(e[j + 1]) for j in range(5)] for e in ev]).mean(axis=0)
    return a.elapsed_time(b) / args.steps, stages


def run_nv_moe(args, cfg):
    """The fused layer in the NVFP4 variant (moe_nvfp4_fused) on a workload:
    same routing and x as the FP8 layer, NVFP4 weights (per-expert global
    scales) and the calibrated activation global scales."""
    import fp8_block_scaled_route_b200 as moe
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    _, bf16, _, src = load_peaks()
    fp4_peak = bf16 * FP4_OVER_BF16
    inp = synth.make_nvfp4_moe_inputs(cfg, seed=0, device=dev, keep_codes=False)
    T, H, I, E, k = cfg.T, cfg.H, cfg.I, cfg.E, cfg.k
    w13_sf = torch.empty(E * 2 * I, H // 16, dtype=torch.uint8, device=dev)
    w2_sf = torch.empty(E * H, I // 16, dtype=torch.uint8, device=dev)
    moe.nvfp4_tile_scales(inp["w13_sf"].view(E * 2 * I, H // 16), w13_sf)
    moe.nvfp4_tile_scales(inp["w2_sf"].view(E * H, I // 16), w2_sf)
    del inp["w13_sf"], inp["w2_sf"]
    a13 = (1.0 / (inp["a1_g"] * inp["w13_g"].double())).float()
    a2 = (1.0 / (inp["a2_g"] * inp["w2_g"].double())).float()
    ws = torch.empty(moe.moe_workspace_size(T, H, I, E, k), dtype=torch.uint8, device=dev)
    out = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)
    counts = work_counts(cfg, inp["topk_ids"])
    ms, st = timed_layer(lambda: moe.moe_nvfp4_fused(
        inp["x"], inp["topk_ids"], inp["topk_w"], inp["w13_packed"], w13_sf, a13,
        inp["w2_packed"], w2_sf, a2, inp["a1_g"], inp["a2_g"], out, ws, stream=stream),
        args, ws, stream, dev)
    g1_tf = counts["g1_flops"] / (st[2] * 1e-3) / 1e12
    line = {"metric": "fused MoE layer, NVFP4 variant: TFLOP/s", "unit": "TFLOP/s",
            "value": counts["flops"] / (ms * 1e-3) / 1e12, "ms_per_step": ms,
            "higher_is_better": True, "steps": args.steps, "warmup": args.warmup, "n_gpus": 1,
            "dtype": "nvfp4 e2m1 + e4m3 per 16 + fp32 global (fp32 accumulate)",
            "data": "synthetic",
            "config": {"workload": workload_desc(cfg) + "; NVFP4 weights and activations",
                       "l2": "inputs larger than L2 (no flush)"},
            "stages_us": {n: float(v) * 1e3 for n, v in
                          zip(["route", "quant", "gemm1", "gemm2", "finish"], st)},
            "roofline": {"bound": "tensor", "achieved": g1_tf, "peak": fp4_peak,
                         "unit": "TFLOP/s", "frac": g1_tf / fp4_peak, "traffic": None,
                         "kernel": "NVFP4 GEMM1 (gate/up + SwiGLU + NVFP4 requant)",
                         "peak_source": f"{src} (FP4 = bf16 burst x {FP4_OVER_BF16:g})"},
            # + the K-block-major transpose of x's scales (taken when I >= H / 16)
            "gpu_launches": (kernels_per_layer(T, k) + (1 if 16 * I >= H else 0)) * args.steps}
    print(json.dumps(line), flush=True)
    return 0


def run_mx_moe(args, cfg):
    """The fused layer in the MXFP8 variant (moe_mxfp8_fused) on a workload:
    same routing and x as the FP8 layer, MXFP8 weights; the FP8 layer with
    fp32 block scales is timed on the same routing beside it."""
    import fp8_block_scaled_route_b200 as moe
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    _, bf16, _, src = load_peaks()
    fp8_peak = bf16 * FP8_OVER_BF16
    inp = synth.make_mx_moe_inputs(cfg, seed=0, device=dev)
    T, H, I, E, k = cfg.T, cfg.H, cfg.I, cfg.E, cfg.k
    w13_sf = torch.empty(E * 2 * I, H // 32, dtype=torch.uint8, device=dev)
    w2_sf = torch.empty(E * H, I // 32, dtype=torch.uint8, device=dev)
    moe.mxfp8_tile_scales(inp["w13_sf"].view(E * 2 * I, H // 32), w13_sf)
    moe.mxfp8_tile_scales(inp["w2_sf"].view(E * H, I // 32), w2_sf)
    ws = torch.empty(moe.moe_workspace_size(T, H, I, E, k), dtype=torch.uint8, device=dev)
    out = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)
    counts = work_counts(cfg, inp["topk_ids"])

    def timed(step):
        return timed_layer(step, args, ws, stream, dev)

    ms_mx, st_mx = timed(lambda: moe.moe_mxfp8_fused(
        inp["x"], inp["topk_ids"], inp["topk_w"], inp["w13"], w13_sf, inp["w2"], w2_sf, out, ws,
        stream=stream))
    del w13_sf, w2_sf
    fp = synth.make_moe_inputs(cfg, seed=0, device=dev)
    ms_fp, st_fp = timed(lambda: moe.moe_fp8_fused(
        fp["x"], fp["topk_ids"], fp["topk_w"], fp["w13"], fp["w13_scale"], fp["w2"],
        fp["w2_scale"], out, ws, stream=stream))
    g1_tf = counts["g1_flops"] / (st_mx[2] * 1e-3) / 1e12
    line = {"metric": "fused MoE layer, MXFP8 variant: TFLOP/s", "unit": "TFLOP/s",
            "value": counts["flops"] / (ms_mx * 1e-3) / 1e12, "ms_per_step": ms_mx,
            "higher_is_better": True, "steps": args.steps, "warmup": args.warmup, "n_gpus": 1,
            "dtype": "mxfp8 e4m3 + e8m0 per 32 (fp32 accumulate)", "data": "synthetic",
            "config": {"workload": workload_desc(cfg) + "; MXFP8 weights and activations",
                       "l2": "inputs larger than L2 (no flush)"},
            "stages_us": {n: float(v) * 1e3 for n, v in
                          zip(["route", "quant", "gemm1", "gemm2", "finish"], st_mx)},
            "roofline": {"bound": "tensor", "achieved": g1_tf, "peak": fp8_peak,
                         "unit": "TFLOP/s", "frac": g1_tf / fp8_peak, "traffic": None,
                         "kernel": "MXFP8 GEMM1 (gate/up + SwiGLU + MXFP8 requant)",
                         "peak_source": f"{src} (FP8 = bf16 burst x {FP8_OVER_BF16:g})"},
            "fp8_fp32_scaled_layer_same_routing": {
                "ms_per_step": ms_fp,
                "stages_us": {n: float(v) * 1e3 for n, v in
                              zip(["route", "quant", "gemm1", "gemm2", "finish"], st_fp)}},
            "gpu_launches": kernels_per_layer(T, k) * args.steps}
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="prefill",
                    choices=sorted(synth.CONFIGS) + sorted(PROFILE_SLICES))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-decode", action="store_true",
                    help="with the prefill workload: skip the decode and mid workloads' timing")
    ap.add_argument("--op", default="moe", choices=["moe", "swiglu_mxfp8", "mxfp8_gemm", "mxfp8_moe",
                                                     "nvfp4_gemm", "nvfp4_moe", "router"],
                    help="any other than moe: time that op instead")
    ap.add_argument("--fusion", default="auto", choices=sorted(FUSION_MODES),
                    help="FP8 layer: fused-expert launch automatic, forced on (where it fits) "
                         "or off")
    ap.add_argument("--swiglu-shape", default="",
                    help="with --op swiglu_mxfp8: only this MxK shape (e.g. 8192x7168)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.op == "swiglu_mxfp8":
        return run_swiglu(args)
    cfg = synth.CONFIGS.get(args.workload) or PROFILE_SLICES[args.workload]
    if args.op == "router":
        return run_router(args, cfg)
    if args.op == "mxfp8_gemm":
        return run_mx_gemm(args, cfg)
    if args.op == "nvfp4_gemm":
        return run_nvfp4_gemm(args, cfg)
    if args.op == "mxfp8_moe":
        return run_mx_moe(args, cfg)
    if args.op == "nvfp4_moe":
        return run_nv_moe(args, cfg)
    if args.impl == "reference":
        return run_reference(args, cfg)
    return run_ours(args, cfg)


if __name__ == "__main__":
    sys.exit(main())
