"""Benchmark: one Gated DeltaNet layer forward under NVFP4 W4A4 (prefill).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Workload (one "step"): gdn_layer_forward over B=1, T=32768 tokens (the
long-context layer prefill, the largest single-GPU configuration) of a layer
with hidden 5120, 16 key / 32 value heads, head dims 128 (fused in_proj
N_in = 12352, out_proj 5120 x 4096), synthetic seeded inputs (outlier-heavy
bf16 activations, N(0, 0.02) weights quantised once to NVFP4, untimed).  The
step covers every stage of the path: activation quantisation, fused in_proj
GEMM, gates + q/k normalisation, chunked delta-rule scan, o quantisation,
out_proj GEMM.  The T=4096 layer prefill is measured the same way and
reported under its own key.  L2 (126 MB) is flushed by a 256 MB write before
every timed step; each step is timed with CUDA events on the launching
stream.

Prints one JSON line (rank 0).  Under torchrun each rank runs an independent
replica of the workload (the layer does not shard at this size; weak scaling)
and the reported time is the max over ranks.
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "GDN-layer W4A4 prefill tokens/s; FP4 GEMM TFLOPS and % NVFP4/HBM roofline"
UNIT = "tokens/s"
WORKLOAD = "gdn_layer_prefill_B1_T32768_h5120_hk16_hv32_k128_v128"
HEADLINE_T = 32768
NVFP4_OVER_BF16 = 4.0   # nominal dense FP4 : BF16 tensor throughput on B200 (9 : 2.25 PFLOP/s)

# launches of this library's kernels per gdn_layer_forward (T > 1), as the ncu launch list
# shows them: zero the quantiser words, quantise x (one cooperative launch), in_proj GEMM,
# gates (g, beta), scan (prep, sequential), quantise o (from the scan's amax), out_proj GEMM
LAUNCHES_PER_STEP = 8


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ------------------------------------------------------------------- clocks --
class ClockSampler:
    """nvidia-smi samples of this GPU's SM clock and throttle reasons."""
    FIELDS = ["uuid", "clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]

    def __init__(self, uuid: str | None):
        self.uuid = uuid
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "--query-gpu=" + ",".join(self.FIELDS), "--format=csv,noheader",
                                          "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) != len(self.FIELDS):
                continue
            if self.uuid and f[0] != self.uuid:
                continue
            try:
                sm.append(float(f[1].split()[0]))
                smax.append(float(f[2].split()[0]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        loaded = [s for s in sm if smax and s > 0.5 * max(smax)] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------- workload -----
def make_layer(dev, seed):
    import gdn_synth
    import nvfp4_w4a4_gated_b200 as nv
    sh = gdn_synth.FULL
    f32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(dev)
    W_in = gdn_synth.weights(seed + 100, sh.n_in, sh.H)
    W_out = gdn_synth.weights(seed + 101, sh.H, sh.Hv * sh.V)
    A_log, dt_bias = gdn_synth.gate_params(seed + 102, sh.Hv, 0.0, math.log(16.0))
    dims = nv.GdnDims(sh.Hk, sh.Hv, sh.K, sh.V)
    w = nv.LayerWeights(nv.nvfp4_quantize(f32(W_in)), nv.nvfp4_quantize(f32(W_out)), f32(A_log), f32(dt_bias),
                        dims, sh.H)
    return w, sh


def stage_work(sh, B, T):
    """Algorithmic work per stage of one step (bytes for HBM-bound stages,
    flops for the GEMMs): the per-unit figures times the units one launch
    processes."""
    BT = B * T
    HvV, HkK = sh.Hv * sh.V, sh.Hk * sh.K
    return {
        "quant_x": ("hbm", BT * sh.H * (2 + 0.5 + 1 / 16)),
        "gemm_in": ("tensor", 2.0 * BT * sh.n_in * sh.H),
        "gates": ("hbm", BT * (2 * sh.Hv * 4 + 2 * sh.Hv * 4)),   # a, b columns in; g, beta out
        "scan": ("hbm", BT * (2 * HkK * 4 + HvV * 4 + 2 * sh.Hv * 4 + HvV * 4) + 2 * B * sh.Hv * sh.K * sh.V * 4),
        "quant_o": ("hbm", BT * HvV * (4 + 0.5 + 1 / 16)),
        "gemm_out": ("tensor", 2.0 * BT * sh.H * HvV),
    }


# the layer's own launches per stage (gdn_layer_forward_timed records an event
# before each stage): the scan normalises q and k while staging a chunk, the
# gates kernel forms g and beta only, and o is quantised from the amax word the
# scan filled
STAGE_KERNELS = {"quant_x": "zero_words_kernel + quant_kernel<bf16> (amax pass, grid barrier, quantise pass)",
                 "gemm_in": "w4a4_gemm_kernel", "gates": "gate_kernel (g, beta)",
                 "scan": "chunk_prep_kernel + chunk_seq_kernel", "quant_o": "quant_kernel<f32> (from the scan's amax)",
                 "gemm_out": "w4a4_gemm_kernel"}


def traffic_for(stage: str, T: int):
    """DRAM bytes per launch of the stage's kernels at T tokens from the committed
    ncu summary (profiles/dram_traffic.txt), or None when absent or when the
    kernel source changed since the counters were taken.  A figure captured at
    another T is scaled by the tokens processed (the stage's traffic grows in
    proportion to T: per-chunk records, per-token rows)."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(p):
        return None
    src_of = {"gemm_in": "gemm.cu", "gemm_out": "gemm.cu", "scan": "scan.cu", "quant_x": "quantize.cu",
              "quant_o": "quantize.cu", "gates": "gates.cu"}
    src = os.path.join(ROOT, "nvfp4_w4a4_gated_b200", "csrc", src_of[stage])
    sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    for ln in open(p):
        f = ln.split()
        if len(f) >= 4 and not ln.startswith("#") and f[0] == stage:
            return float(f[1]) * T / float(f[3]) if f[2] == sha else None
    return None


def cpu_baseline(sample_tokens: int, seed: int):
    """The oracle, as it stands, on a prefix of the same workload's sequence."""
    import gdn_synth
    import oracle
    sh = gdn_synth.FULL
    W_in = gdn_synth.weights(seed + 100, sh.n_in, sh.H)
    W_out = gdn_synth.weights(seed + 101, sh.H, sh.Hv * sh.V)
    A_log, dt_bias = gdn_synth.gate_params(seed + 102, sh.Hv, 0.0, math.log(16.0))
    Wid = oracle.dequantize(*oracle.quantize(W_in))
    Wod = oracle.dequantize(*oracle.quantize(W_out))
    _, x = gdn_synth.activations(seed, HEADLINE_T, sh.H, hot="percent")
    xs = np.ascontiguousarray(x[:sample_tokens])
    del x
    t0 = time.perf_counter()
    oracle.layer_forward(xs, None, None, A_log, dt_bias, 1, sample_tokens, sh.Hk, sh.Hv, sh.K, sh.V, W_in_deq=Wid,
                         W_out_deq=Wod)
    dt = time.perf_counter() - t0
    return {"value": sample_tokens / dt, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"first {sample_tokens} of the {HEADLINE_T} tokens (B=1), full layer width, float64 oracle; "
                      f"weights dequantised before timing", "seconds": dt}


# ------------------------------------------------------------- our arm -----
def max_over_ranks(values, dev, distributed: bool):
    """Each timing as the maximum over the ranks (the slowest rank sets the
    job's time); unchanged on one rank."""
    t = torch.tensor(values, dtype=torch.float64, device=dev)
    if distributed:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return [float(v) for v in t]


def job_throughput(world: int, tokens_per_rank_step: int, steps: int, total_ms: float):
    """Whole-job tokens and tokens/s: every rank's tokens over the slowest
    rank's time (weak scaling: each rank runs the same workload)."""
    tokens = world * tokens_per_rank_step * steps
    return tokens, tokens / (total_ms / 1e3)


def spread(ms):
    return {"min": round(min(ms), 4), "median": round(statistics.median(ms), 4), "max": round(max(ms), 4)}


def time_prefill(nv, w, sh, dev, B, T, steps, warmup, flush, stream, seed):
    """gdn_layer_forward over B x T tokens: `steps` timed steps (L2 flushed before
    each, CUDA events on the launching stream), then `steps` more through
    gdn_layer_forward_timed, which records an event before each of the layer's
    six stages and after the last (per-stage times of the same launches)."""
    import gdn_synth
    bits, _ = gdn_synth.activations(seed, B * T, sh.H, hot="percent")
    x = torch.from_numpy(bits.view(np.int16)).to(dev).view(torch.bfloat16)
    y = torch.empty((B * T, sh.H), dtype=torch.float32, device=dev)
    lay = nv.layer_workspace_layout(w, B, T)
    ws = torch.empty(lay["total"], dtype=torch.uint8, device=dev)

    def step():
        nv.gdn_layer_forward(w, x, B, T, y=y, workspace=ws, stream=stream)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    nv.check_device_error()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    torch.cuda.synchronize()
    for i in range(steps):
        flush.zero_()
        starts[i].record(stream)
        step()
        ends[i].record(stream)
    torch.cuda.synchronize()
    step_ms = [a.elapsed_time(b) for a, b in zip(starts, ends)]
    nstage = 6
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nstage + 1)] for _ in range(steps)]
    for i in range(steps):
        flush.zero_()
        nv.gdn_layer_forward(w, x, B, T, y=y, workspace=ws, stream=stream, events=evs[i])
    torch.cuda.synchronize()
    nv.check_device_error()
    names = ["quant_x", "gemm_in", "gates", "scan", "quant_o", "gemm_out"]
    stage_ms = {n: statistics.median(evs[i][j].elapsed_time(evs[i][j + 1]) for i in range(steps))
                for j, n in enumerate(names)}
    return dict(x=x, y=y, ws=ws, lay=lay, step_ms=step_ms, stage_ms=stage_ms, names=names)


def roofline_of(sh, B, T, stage_ms, pk):
    """The dominant stage's roofline and every stage's achieved fraction."""
    work = stage_work(sh, B, T)
    dom = max(stage_ms, key=stage_ms.get)
    bound, units = work[dom]
    if bound == "tensor":
        peak = pk["bf16_tflops"] * NVFP4_OVER_BF16
        achieved = units / (stage_ms[dom] / 1e3) / 1e12
        unit, peak_note = "TFLOP/s", f"{pk['source']} bf16 burst x {NVFP4_OVER_BF16:g} (nominal FP4:BF16)"
    else:
        peak = pk["hbm_gbs"]
        achieved = units / (stage_ms[dom] / 1e3) / 1e9
        unit, peak_note = "GB/s", f"{pk['source']} HBM copy"
    stages = {}
    for n, ms in stage_ms.items():
        b, u = work[n]
        if b == "tensor":
            stages[n] = {"ms": round(ms, 4), "TFLOP/s": round(u / (ms / 1e3) / 1e12, 1),
                         "frac": round(u / (ms / 1e3) / 1e12 / (pk["bf16_tflops"] * NVFP4_OVER_BF16), 3)}
        else:
            stages[n] = {"ms": round(ms, 4), "GB/s": round(u / (ms / 1e3) / 1e9, 1),
                         "frac": round(u / (ms / 1e3) / 1e9 / pk["hbm_gbs"], 3)}
    roof = {"bound": bound, "kernel": f"{dom}: {STAGE_KERNELS[dom]}", "achieved": round(achieved, 1),
            "peak": round(peak, 1), "unit": unit, "frac": round(achieved / peak, 4),
            "traffic": traffic_for(dom, T), "peak_source": peak_note}
    return roof, stages


def run_ours(args, rank, world, local_rank):
    import nvfp4_w4a4_gated_b200 as nv
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    dist = world > 1
    seed = 2 + rank
    B, T = 1, HEADLINE_T
    w, sh = make_layer(dev, seed)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    pk = peaks()

    # ---- timed region: K steps of gdn_layer_forward at T = 32768, L2 flushed before each
    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    clocks = ClockSampler(uuid)
    clocks.start()
    time.sleep(0.3)
    if dist:
        torch.distributed.barrier()
    run = time_prefill(nv, w, sh, dev, B, T, args.steps, args.warmup, flush, stream, seed)
    if dist:
        torch.distributed.barrier()
    clk = clocks.stop()
    total_ms = sum(run["step_ms"])
    stage_ms = run["stage_ms"]
    x, y, ws = run["x"], run["y"], run["ws"]

    # ---- the T = 4096 layer prefill, the same measurement (its own key)
    run4k = time_prefill(nv, w, sh, dev, 1, 4096, args.steps, args.warmup, flush, stream, seed)
    roof4k, stages4k = roofline_of(sh, 1, 4096, run4k["stage_ms"], pk)
    prefill_4k = {"workload": "gdn_layer_prefill_B1_T4096_h5120_hk16_hv32_k128_v128",
                  "value": round(4096 / (statistics.mean(run4k["step_ms"]) / 1e3), 1), "unit": UNIT,
                  "ms_per_step": round(statistics.mean(run4k["step_ms"]), 4), "ms_spread": spread(run4k["step_ms"]),
                  "roofline": roof4k, "stages": stages4k}
    x4k = run4k["x"]
    del run4k

    # ---- standalone GEMM workload (M=8192, N=12288, K=5120), TFLOPS
    gemm = bench_gemm(nv, dev, args.steps, flush, stream)
    # ---- batch-64 decode step (HBM-bound)
    decode = bench_decode(nv, dev, w, sh, args.steps, stream)
    # ---- the T = 4096 prefill step with the optional output gate
    gated = bench_gated(nv, dev, w, sh, x4k, 1, 4096, args.steps, flush, stream)
    # ---- the 32K-token scan split into eight spans (one sequence-parallel rank's work)
    seqpar = bench_seqpar(nv, dev, args.steps, flush, stream, clk.get("sm_max_mhz"))

    # ---- end to end through the public call with host buffers, pipelined over steps:
    # the upload of step i+1 (pinned x -> device) and the download of step i's y
    # (device -> pinned) run on their own streams while step i / i+1 computes; inputs
    # and outputs are double-buffered, events order every reuse.  The L2 flush stays
    # in front of every forward, on the compute stream.  Time = one window from the
    # first upload to the last download.
    x_host = torch.empty(x.shape, dtype=torch.bfloat16, pin_memory=True)
    x_host.copy_(x.cpu())
    y_host = [torch.empty(y.shape, dtype=torch.float32, pin_memory=True) for _ in range(2)]
    x_dev = [torch.empty_like(x) for _ in range(2)]
    y_dev = [torch.empty_like(y) for _ in range(2)]
    s_up, s_down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()
    up_done = [ev() for _ in range(args.steps)]
    comp_done = [ev() for _ in range(args.steps)]
    down_done = [ev() for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    t_start.record(stream)
    s_up.wait_event(t_start)
    s_down.wait_event(t_start)
    for i in range(args.steps):
        j = i % 2
        with torch.cuda.stream(s_up):
            if i >= 2:
                s_up.wait_event(comp_done[i - 2])       # x_dev[j] read by step i-2
            x_dev[j].copy_(x_host, non_blocking=True)
            up_done[i].record(s_up)
        stream.wait_event(up_done[i])
        if i >= 2:
            stream.wait_event(down_done[i - 2])          # y_dev[j] read back by step i-2
        flush.zero_()
        nv.gdn_layer_forward(w, x_dev[j], B, T, y=y_dev[j], workspace=ws, stream=stream)
        comp_done[i].record(stream)
        with torch.cuda.stream(s_down):
            s_down.wait_event(comp_done[i])
            y_host[j].copy_(y_dev[j], non_blocking=True)
            down_done[i].record(s_down)
    stream.wait_event(down_done[args.steps - 1])
    t_end.record(stream)
    torch.cuda.synchronize()
    e2e_ms = t_start.elapsed_time(t_end)

    # ---- aggregate over ranks: max time
    total_ms, e2e_ms = max_over_ranks([total_ms, e2e_ms], dev, dist)
    tokens, value = job_throughput(world, B * T, args.steps, total_ms)
    roof, stages = roofline_of(sh, B, T, stage_ms, pk)
    out = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(total_ms / args.steps, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "nvfp4(e2m1,e4m3)+f32", "data": "synthetic",
        "config": {"workload": WORKLOAD, "B": B, "T": T, "hidden": sh.H, "Hk": sh.Hk, "Hv": sh.Hv, "K": sh.K,
                   "V": sh.V, "n_in": sh.n_in, "form": "pages", "scan": "chunked C=64",
                   "l2": "flushed (256 MB write) before every timed step", "replicas": world},
        "ms_spread": spread(run["step_ms"]),
        "roofline": roof,
        "stages": stages,
        "prefill_T4096": prefill_4k,
        "gemm_standalone": gemm,
        "decode": decode,
        "output_gate": gated,
        "sequence_parallel_scan": seqpar,
        "e2e": {"value": round(tokens / (e2e_ms / 1e3), 1), "unit": UNIT,
                "h2d_bytes_per_step": int(x.numel() * 2), "d2h_bytes_per_step": int(y.numel() * 4)},
        "gpu_launches": LAUNCHES_PER_STEP * args.steps,
        "clocks": clk,
    }
    return out


def bench_gated(nv, dev, w, sh, x, B, T, steps, flush, stream):
    """The same prefill step with the optional output gate (out_proj reads
    RMSNorm(o) * w * SiLU(z)), and the gate kernel alone.  Algorithmic bytes of
    the gate: o and z read, the gated output written, 12 B per element."""
    import dataclasses
    import gdn_synth
    w_norm = torch.from_numpy(gdn_synth.gaussian(9, (sh.V,), std=1.0)).to(dev)
    wg = dataclasses.replace(w, out_norm=w_norm)
    lay = nv.layer_workspace_layout(wg, B, T)
    ws = torch.empty(lay["total"], dtype=torch.uint8, device=dev)
    y = torch.empty((B * T, sh.H), dtype=torch.float32, device=dev)
    for _ in range(3):
        nv.gdn_layer_forward(wg, x, B, T, y=y, workspace=ws, stream=stream)
    torch.cuda.synchronize()
    ts = []
    for _ in range(steps):
        flush.zero_()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record(stream)
        nv.gdn_layer_forward(wg, x, B, T, y=y, workspace=ws, stream=stream)
        e.record(stream)
        ts.append((s, e))
    # the gate kernel alone, on the step's own o and z
    BT, HvV = B * T, sh.Hv * sh.V
    ldp = (sh.n_in + 3) // 4 * 4
    o = ws[lay["o"]:lay["o"] + BT * HvV * 4].view(torch.float32).view(BT, sh.Hv, sh.V)
    P = ws[lay["proj"]:lay["proj"] + BT * ldp * 4].view(torch.float32).view(BT, ldp)
    z = P[:, 2 * sh.Hk * sh.K + HvV:]
    G = ws[lay["o_gated"]:lay["o_gated"] + BT * HvV * 4].view(torch.float32).view(BT, sh.Hv, sh.V)
    gt = []
    for _ in range(steps):
        flush.zero_()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record(stream)
        nv.gdn_output_gate(o, z, w_norm, out=G, stream=stream)
        e.record(stream)
        gt.append((s, e))
    torch.cuda.synchronize()
    nv.check_device_error()
    ms = statistics.mean(s.elapsed_time(e) for s, e in ts)
    gms = statistics.mean(s.elapsed_time(e) for s, e in gt)
    gbs = BT * HvV * 12 / (gms / 1e3) / 1e9
    # the whole block: short convolution on q|k|v (width 4) and the output gate
    C = 2 * sh.Hk * sh.K + HvV
    conv_w = torch.from_numpy(gdn_synth.gaussian(10, (C, 4), std=0.5)).to(dev)
    wf = dataclasses.replace(wg, conv_weight=conv_w, conv_width=4)
    layf = nv.layer_workspace_layout(wf, B, T)
    wsf = torch.empty(layf["total"], dtype=torch.uint8, device=dev)
    for _ in range(3):
        nv.gdn_layer_forward(wf, x, B, T, y=y, workspace=wsf, stream=stream)
    torch.cuda.synchronize()
    tf, ct = [], []
    for _ in range(steps):
        flush.zero_()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record(stream)
        nv.gdn_layer_forward(wf, x, B, T, y=y, workspace=wsf, stream=stream)
        e.record(stream)
        tf.append((s, e))
    # the convolution kernel alone on the step's projection (4 B read + 4 B written per element)
    Pf = wsf[layf["proj"]:layf["proj"] + BT * ldp * 4].view(torch.float32).view(BT, ldp)
    qkv = wsf[layf["qkv_conv"]:layf["qkv_conv"] + BT * C * 4].view(torch.float32).view(BT, C)
    for _ in range(steps):
        flush.zero_()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record(stream)
        nv.gdn_short_conv(Pf, conv_w, B, T, out=qkv, stream=stream)
        e.record(stream)
        ct.append((s, e))
    torch.cuda.synchronize()
    nv.check_device_error()
    fms = statistics.mean(s.elapsed_time(e) for s, e in tf)
    cms = statistics.mean(s.elapsed_time(e) for s, e in ct)
    cgbs = BT * C * 8 / (cms / 1e3) / 1e9
    return {"workload": WORKLOAD + "_output_gate", "ms_per_step": round(ms, 4),
            "tokens_per_s": round(B * T / (ms / 1e3), 1),
            "output_gate_kernel": {"ms": round(gms, 4), "GB/s": round(gbs, 1),
                                   "frac_of_hbm": round(gbs / peaks()["hbm_gbs"], 4)},
            "with_short_conv": {"workload": WORKLOAD + "_short_conv4_output_gate", "ms_per_step": round(fms, 4),
                                "tokens_per_s": round(B * T / (fms / 1e3), 1),
                                "short_conv_kernel": {"ms": round(cms, 4), "GB/s": round(cgbs, 1),
                                                      "frac_of_hbm": round(cgbs / peaks()["hbm_gbs"], 4)}}}


def bench_seqpar(nv, dev, steps, flush, stream, sm_max_mhz):
    """The 32K-token scan (B = 1, 16 key / 32 value heads of 128) split into
    eight spans of 4096 tokens, as eight ranks of a sequence-parallel scan run
    it, timed on one GPU: the last rank's steps (its span's zero-start scan and
    maps in one gdn_scan_span call, the seven earlier maps composed in one
    gdn_state_combine launch, the output correction) against the unsplit scan.
    The all-gather of (P, S_loc), 4 MiB per rank, is not measured on one GPU.
    The correction kernel (tcgen05, TF32) does 2 T Hv K V FLOP and moves
    (T Hv (K + 2 V) + Hv K V) x 4 bytes: HBM-bound."""
    B, T, Hk, Hv, K, V, n = 1, 32768, 16, 32, 128, 128, 8
    Ts = T // n
    dims = nv.GdnDims(Hk, Hv, K, V)
    g_ = torch.Generator(device=dev)
    g_.manual_seed(11)
    q = torch.nn.functional.normalize(torch.randn((T, Hk, K), generator=g_, device=dev), dim=-1)
    k = torch.nn.functional.normalize(torch.randn((T, Hk, K), generator=g_, device=dev), dim=-1)
    v = torch.randn((T, Hv * V), generator=g_, device=dev)
    g = torch.log(torch.rand((T, Hv), generator=g_, device=dev) * (0.9999 - 0.99) + 0.99)
    beta = torch.rand((T, Hv), generator=g_, device=dev)
    o = torch.empty((T, Hv, V), device=dev)
    S = torch.empty((B, Hv, K, V), device=dev)
    ws = torch.empty(nv.lib().gdn_scan_workspace_size(B, T, ctypes.byref(dims.c()), nv.SCAN_AUTO),
                     dtype=torch.uint8, device=dev)
    a = T - Ts                                   # the last rank's span
    span = (q[a:], k[a:], v[a:], g[a:], beta[a:])
    ws_s = torch.empty(nv.lib().gdn_scan_span_workspace_size(B, Ts, ctypes.byref(dims.c()), nv.SCAN_AUTO),
                       dtype=torch.uint8, device=dev)
    Ps = torch.randn((n - 1, B, Hv, K, K), generator=g_, device=dev) * (K ** -0.5)
    Sl = torch.randn((n - 1, B, Hv, K, V), generator=g_, device=dev)
    S_in = torch.empty((B, Hv, K, V), device=dev)

    def whole():
        nv.gdn_scan(q, k, v, g, beta, B, T, dims, o=o, state_out=S, workspace=ws, stream=stream)

    def rank_steps(ev):
        ev[0].record(stream)
        o_s, S_loc, P, qmap = nv.gdn_scan_span(*span, B, Ts, dims, workspace=ws_s, stream=stream)
        ev[1].record(stream)
        nv.gdn_state_combine(Ps, Sl, None, out=S_in, stream=stream)
        ev[2].record(stream)
        nv.gdn_scan_correct(qmap, S_in, o_s, B, Ts, stream=stream)
        ev[3].record(stream)
        nv.gdn_state_combine(P, S_loc, S_in, out=S_loc, stream=stream)   # the state after the span
        ev[4].record(stream)

    mk = lambda m: [torch.cuda.Event(enable_timing=True) for _ in range(m)]
    for _ in range(3):
        whole()
        rank_steps(mk(5))
    torch.cuda.synchronize()
    tw, tr = [], []
    for _ in range(steps):
        flush.zero_()
        ev = mk(2)
        ev[0].record(stream)
        whole()
        ev[1].record(stream)
        tw.append(ev)
        flush.zero_()
        ev = mk(5)
        rank_steps(ev)
        tr.append(ev)
    torch.cuda.synchronize()
    nv.check_device_error()
    mean = lambda evs, i, j: statistics.mean(e[i].elapsed_time(e[j]) for e in evs)
    whole_ms, rank_ms = mean(tw, 0, 1), mean(tr, 0, 4)
    corr_ms = mean(tr, 2, 3)
    # the correction alone, tensor-core kernel and the CUDA-core one (same launch, same inputs)
    o_c = torch.randn((Ts, Hv, V), generator=g_, device=dev)
    m_c = torch.randn((Ts, Hv, K), generator=g_, device=dev) * 0.1
    alone = {}
    for variant in ("tcgen05", "cuda_core"):
        if variant == "cuda_core":
            os.environ["NVFP4_CORRECT_VARIANT"] = "cuda_core"
        ts = []
        for _ in range(steps):
            flush.zero_()
            ev = mk(2)
            ev[0].record(stream)
            nv.gdn_scan_correct(m_c, S_in, o_c, B, Ts, stream=stream)
            ev[1].record(stream)
            ts.append(ev)
        torch.cuda.synchronize()
        os.environ.pop("NVFP4_CORRECT_VARIANT", None)
        alone[variant] = mean(ts, 0, 1)
    nv.check_device_error()
    flop = 2.0 * Ts * Hv * K * V
    byt = (Ts * Hv * (K + 2 * V) + Hv * K * V) * 4
    return {"workload": "gdn_scan_B1_T32768_hk16_hv32_k128_v128_in_8_spans_of_4096",
            "whole_scan_ms": round(whole_ms, 4), "per_rank_ms": round(rank_ms, 4),
            "per_rank_speedup_without_exchange": round(whole_ms / rank_ms, 2),
            "rank_steps_ms": {"span_scan_and_maps": round(mean(tr, 0, 1), 4),
                              "combine_7_maps": round(mean(tr, 1, 2), 4), "correct": round(corr_ms, 4),
                              "end_state": round(mean(tr, 3, 4), 4)},
            "exchange": "all-gather of P and S_loc (4 MiB per rank): not measured on one GPU",
            "correct_kernel": {"bound": "hbm", "GB/s": round(byt / (corr_ms / 1e3) / 1e9, 1),
                               "frac": round(byt / (corr_ms / 1e3) / 1e9 / peaks()["hbm_gbs"], 4),
                               "peak_source": "measured HBM copy",
                               "TFLOP/s": round(flop / (corr_ms / 1e3) / 1e12, 2),
                               "note": "tcgen05 kind::tf32; 2 T Hv K V FLOP, (T Hv (K + 2 V) + Hv K V) x 4 bytes",
                               "alone_ms": {k_: round(v_, 4) for k_, v_ in alone.items()}}}


def bench_decode(nv, dev, w, sh, steps, stream):
    """Batch-64 decode: gdn_layer_forward with T = 1 and the 64 x 32 fp32 states
    carried in place.  The states (268 MB) are larger than L2, so no flush is
    needed between steps.  Algorithmic bytes per step: the states read and
    written, both NVFP4 weights (codes + scales), x and y."""
    import gdn_synth
    B = 64
    S = torch.from_numpy(gdn_synth.gaussian(9, (B, sh.Hv, sh.K, sh.V), std=0.3)).to(dev)
    xs = [torch.from_numpy(gdn_synth.activations(2000 + i, B, sh.H, hot="none")[0].view(np.int16)).to(dev)
          .view(torch.bfloat16) for i in range(4)]
    y = torch.empty((B, sh.H), dtype=torch.float32, device=dev)
    lay = nv.layer_workspace_layout(w, B, 1)
    ws = torch.empty(lay["total"], dtype=torch.uint8, device=dev)

    def step(i):
        nv.gdn_layer_forward(w, xs[i % 4], B, 1, y=y, state_in=S, state_out=S, workspace=ws, stream=stream)

    for i in range(5):
        step(i)
    n = max(steps, 32)
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    s.record(stream)
    for i in range(n):
        step(i)
    e.record(stream)
    torch.cuda.synchronize()
    nv.check_device_error()
    ms = s.elapsed_time(e) / n
    pk = peaks()
    state = 2 * B * sh.Hv * sh.K * sh.V * 4
    weights = sh.n_in * sh.H // 2 + sh.n_in * sh.H // 16 + sh.H * sh.Hv * sh.V // 2 + sh.H * sh.Hv * sh.V // 16
    io = B * sh.H * 2 + B * sh.H * 4
    nbytes = state + weights + io
    gbs = nbytes / (ms / 1e3) / 1e9
    return {"workload": "gdn_decode_B64_h5120_hk16_hv32_k128_v128", "ms_per_step": round(ms, 4),
            "tokens_per_s": round(B / (ms / 1e3), 1), "bytes_per_step": nbytes, "GB/s": round(gbs, 1),
            "frac_of_hbm": round(gbs / pk["hbm_gbs"], 4), "steps": n,
            "l2": "states (268 MB) larger than L2; no flush"}


def bench_gemm(nv, dev, steps, flush, stream):
    """Standalone block-scaled GEMM, M=8192, N=12288 (q|k|v|z slices with 4x
    module amax spread, one harmonised scale), K=5120, fp32 C."""
    import gdn_synth
    M, N, K = 8192, 12288, 5120
    bits, _ = gdn_synth.activations(1, M, K, hot="percent")
    Wt = gdn_synth.weights(2, N, K, slice_rows=gdn_synth.GEMM_SLICES, slice_gain=gdn_synth.GEMM_SLICE_GAIN)
    xa = torch.from_numpy(bits.view(np.int16)).to(dev).view(torch.bfloat16)
    A = nv.nvfp4_quantize(xa)
    Bm = nv.nvfp4_quantize(torch.from_numpy(Wt).to(dev))
    C = torch.empty((M, N), dtype=torch.float32, device=dev)
    for _ in range(3):
        nv.w4a4_gemm(A, Bm, C, stream=stream)
    qa = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
    ts = []
    for i in range(steps):
        flush.zero_()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record(stream)
        nv.w4a4_gemm(A, Bm, C, stream=stream)
        e.record(stream)
        ts.append((s, e))
    # quantiser on the same activation (HBM-bound)
    qt = []
    for i in range(steps):
        flush.zero_()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record(stream)
        nv.nvfp4_quantize(xa, out=A, stream=stream)
        e.record(stream)
        qt.append((s, e))
    torch.cuda.synchronize()
    ms = statistics.mean(s.elapsed_time(e) for s, e in ts)
    qms = statistics.mean(s.elapsed_time(e) for s, e in qt)
    pk = peaks()
    tflops = 2.0 * M * N * K / (ms / 1e3) / 1e12
    qgbs = M * K * 2.5625 / (qms / 1e3) / 1e9
    del qa
    return {"workload": "gemm_M8192_N12288_K5120_fp32out", "ms": round(ms, 4), "TFLOP/s": round(tflops, 1),
            "frac_of_nvfp4_peak": round(tflops / (pk["bf16_tflops"] * NVFP4_OVER_BF16), 4),
            "quantize_8192x5120_bf16": {"ms": round(qms, 4), "GB/s": round(qgbs, 1),
                                         "frac_of_hbm": round(qgbs / pk["hbm_gbs"], 4)}}


# ------------------------------------------------------ reference arm -----
def run_reference(args):
    """The oracle as the reference implementation, timed on the host cores:
    each step is the layer forward over a bounded prefix of the workload."""
    import gdn_synth
    import oracle
    sh = gdn_synth.FULL
    seed = 2
    sample = args.ref_tokens
    W_in = gdn_synth.weights(seed + 100, sh.n_in, sh.H)
    W_out = gdn_synth.weights(seed + 101, sh.H, sh.Hv * sh.V)
    A_log, dt_bias = gdn_synth.gate_params(seed + 102, sh.Hv, 0.0, math.log(16.0))
    Wid = oracle.dequantize(*oracle.quantize(W_in))
    Wod = oracle.dequantize(*oracle.quantize(W_out))
    # the workload's activations (the hot channels depend on the row count), then a prefix
    _, x = gdn_synth.activations(seed, HEADLINE_T, sh.H, hot="percent")
    xs = np.ascontiguousarray(x[:sample])
    del x

    def step():
        oracle.layer_forward(xs, None, None, A_log, dt_bias, 1, sample, sh.Hk, sh.Hv, sh.K, sh.V, W_in_deq=Wid,
                             W_out_deq=Wod)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    value = sample * args.steps / dt
    return {"impl": "reference", "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 2),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64 (quantiser exact f32)",
            "data": "synthetic",
            "config": {"workload": WORKLOAD, "B": 1, "T": HEADLINE_T, "hidden": sh.H, "Hk": sh.Hk, "Hv": sh.Hv,
                       "K": sh.K, "V": sh.V, "sample_tokens_per_step": sample},
            "cpu_baseline": {"value": round(value, 2), "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
                             "sample": f"first {sample} tokens of the T={HEADLINE_T} workload per step"},
            "e2e": {"value": round(value, 2), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def run_studies(args):
    """The pages' mechanism studies (review page, paper sec.5.2 Table 3, sec.5.3
    Fig. 1 and Table 6) through the library's kernels on the layer-prefill
    shapes: the sensitivity replay over the T = 4096 workload, the lockstep
    trajectories, the impulse and the gate-noise table over the T = 32768
    workload.  Synthetic inputs and random weights: context, not the pages'
    numbers (theirs come from a trained model)."""
    import gdn_synth
    import nvfp4_w4a4_gated_b200 as nv
    from nvfp4_w4a4_gated_b200 import studies
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    be = studies.CudaBackend(dev, device_noise=True)
    sh = gdn_synth.FULL
    seed = 2
    W_in = gdn_synth.weights(seed + 100, sh.n_in, sh.H)
    W_out = gdn_synth.weights(seed + 101, sh.H, sh.Hv * sh.V)
    dims = nv.GdnDims(sh.Hk, sh.Hv, sh.K, sh.V)
    _, x4 = gdn_synth.activations(seed, 4096, sh.H, hot="percent")
    _, x32 = gdn_synth.activations(seed, HEADLINE_T, sh.H, hot="percent")
    xs4, xs = be.upload(x4), be.upload(x32)
    del x4, x32
    # two gate regimes: the layer's own (A_log ~ U(log 1, log 16): decays of a few tokens on
    # these random weights) and long memory, alpha within ~1e-4 of 1 (horizons of 10^4-10^5
    # tokens, the regime the pages' trained layers sit in)
    regimes = {"layer_gates": gdn_synth.gate_params(seed + 102, sh.Hv, 0.0, math.log(16.0)),
               "long_memory": gdn_synth.gate_params(seed + 103, sh.Hv, math.log(1e-5), math.log(1e-4))}
    out = {}
    for name, (A_log, dt_bias) in regimes.items():
        L = studies.StudyLayer.make(be, W_in, W_out, A_log, dt_bias, dims, sh.H)
        t1 = studies.sensitivity(be, L, xs4, 1, 4096)
        t2 = studies.lockstep(be, L, xs, HEADLINE_T, [256, 512, 1024, 2048, 4096, 8192, 16384, 32768],
                              n_perturbed=11)
        imp = studies.impulse(be, L, xs, HEADLINE_T, t_imp=1024)
        t3 = studies.gate_noise(be, L, xs, HEADLINE_T)
        out[name] = (t1, t2, imp, t3)
    nv.check_device_error()

    def summary(vals):
        got = sorted(v for v in vals if v is not None)
        return {"min": got[0] if got else None, "median": got[len(got) // 2] if got else None,
                "max": got[-1] if got else None, "not_reached": sum(v is None for v in vals)}
    res = {"study": "mechanism studies (sensitivity replay, lockstep trajectories, impulse, gate noise)",
           "data": "synthetic inputs, random weights (N(0, 0.02)); context, not the pages' trained-model numbers",
           "workloads": {"sensitivity": "gdn_layer_prefill_B1_T4096_h5120_hk16_hv32_k128_v128",
                         "lockstep_impulse_gate_noise": WORKLOAD}}
    for name, (t1, t2, imp, t3) in out.items():
        res[name] = {"sensitivity": t1, "lockstep": t2,
                     "impulse": {"t_inject": 1024, "size": 0.01, "resolution": imp["resolution"],
                                 "steps_to_1_over_e": summary(imp["steps_to_1_over_e"]),
                                 "steps_to_1_over_10": summary(imp["steps_to_1_over_10"]),
                                 "horizon_1_over_1_minus_alpha": summary(imp["horizon_1_over_1_minus_alpha"])},
                     "gate_noise": t3}
    return res


def kernel_case(args):
    """One kernel on a fixed-size case, a few launches, for profiler captures
    (ncu -k <kernel> -c <n>); prints the mean launch time."""
    import nvfp4_w4a4_gated_b200 as nv
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    g = torch.Generator(device=dev)
    g.manual_seed(0)
    stream = torch.cuda.current_stream(dev)
    if args.kernel_case == "gemm":
        M, N, K = args.M, args.N, args.K
        A = nv.nvfp4_quantize(torch.randn((M, K), generator=g, device=dev).to(torch.bfloat16))
        Bm = nv.nvfp4_quantize(torch.randn((N, K), generator=g, device=dev) * 0.02)
        C = torch.empty((M, N), dtype=torch.float32, device=dev)
        fn = lambda: nv.w4a4_gemm(A, Bm, C)
    elif args.kernel_case == "quant":
        x = torch.randn((args.M, args.K), generator=g, device=dev).to(torch.bfloat16)
        out = nv.NVFP4Matrix.empty(args.M, args.K, dev)
        fn = lambda: nv.nvfp4_quantize(x, out=out)
    elif args.kernel_case == "scan":
        B, T, Hk, Hv, Kd = 1, args.T, 16, 32, 128
        dims = nv.GdnDims(Hk, Hv, Kd, Kd)
        qh = torch.nn.functional.normalize(torch.randn((B * T, Hk, Kd), generator=g, device=dev), dim=-1)
        kh = torch.nn.functional.normalize(torch.randn((B * T, Hk, Kd), generator=g, device=dev), dim=-1)
        v = torch.randn((B * T, Hv * Kd), generator=g, device=dev)
        gg = torch.log(torch.rand((B * T, Hv), generator=g, device=dev) * 0.5 + 0.5)
        bt = torch.rand((B * T, Hv), generator=g, device=dev)
        o = torch.empty((B * T, Hv, Kd), device=dev)
        ws = torch.empty(nv.lib().gdn_scan_workspace_size(B, T, __import__("ctypes").byref(dims.c()), 0),
                         dtype=torch.uint8, device=dev)
        fn = lambda: nv.gdn_scan(qh, kh, v, gg, bt, B, T, dims, o=o, workspace=ws)
    elif args.kernel_case in ("gate", "conv"):
        # the optional output gate / short convolution on the layer-sized operands
        B, T, Hk, Hv, Kd = 1, args.T, 16, 32, 128
        C = 2 * Hk * Kd + Hv * Kd
        ldp = 2 * C                              # projection-like row stride
        P = torch.randn((B * T, ldp), generator=g, device=dev)
        if args.kernel_case == "gate":
            o = torch.randn((B * T, Hv, Kd), generator=g, device=dev)
            wn = torch.randn((Kd,), generator=g, device=dev)
            G = torch.empty_like(o)
            fn = lambda: nv.gdn_output_gate(o, P[:, C:], wn, out=G)
        else:
            wc = torch.randn((C, 4), generator=g, device=dev) * 0.5
            out = torch.empty((B * T, C), device=dev)
            fn = lambda: nv.gdn_short_conv(P, wc, B, T, out=out)
    elif args.kernel_case == "correct":
        # the sequence-parallel scan's output correction over one span of T tokens
        B, T, Hv, Kd = 1, args.T, 32, 128
        qm = torch.randn((B * T, Hv, Kd), generator=g, device=dev) * 0.1
        S_in = torch.randn((B, Hv, Kd, Kd), generator=g, device=dev)
        o = torch.randn((B * T, Hv, Kd), generator=g, device=dev)
        fn = lambda: nv.gdn_scan_correct(qm, S_in, o, B, T)
    elif args.kernel_case == "layer":
        # one layer prefill of T tokens (B = 1), the headline step's launches
        import gdn_synth
        w, sh = make_layer(dev, 2)
        bits, _ = gdn_synth.activations(2000, args.T, sh.H, hot="percent")
        x = torch.from_numpy(bits.view(np.int16)).to(dev).view(torch.bfloat16)
        y = torch.empty((args.T, sh.H), dtype=torch.float32, device=dev)
        lay = nv.layer_workspace_layout(w, 1, args.T)
        wsl = torch.empty(lay["total"], dtype=torch.uint8, device=dev)
        S = torch.zeros((1, sh.Hv, sh.K, sh.V), dtype=torch.float32, device=dev)
        fn = lambda: nv.gdn_layer_forward(w, x, 1, args.T, y=y, state_in=S, state_out=S, workspace=wsl, stream=stream)
    elif args.kernel_case == "decode":
        # one batch-64 decode step of the layer (T = 1, states carried in place)
        import gdn_synth
        w, sh = make_layer(dev, 2)
        Bd = 64
        S = torch.from_numpy(gdn_synth.gaussian(9, (Bd, sh.Hv, sh.K, sh.V), std=0.3)).to(dev)
        x = torch.from_numpy(gdn_synth.activations(2000, Bd, sh.H, hot="none")[0].view(np.int16)).to(dev)
        x = x.view(torch.bfloat16)
        y = torch.empty((Bd, sh.H), dtype=torch.float32, device=dev)
        lay = nv.layer_workspace_layout(w, Bd, 1)
        wsd = torch.empty(lay["total"], dtype=torch.uint8, device=dev)
        fn = lambda: nv.gdn_layer_forward(w, x, Bd, 1, y=y, state_in=S, state_out=S, workspace=wsd, stream=stream)
    elif args.kernel_case == "statepass":
        # one rank's joining steps over a span of T tokens: seven maps composed, then the correction
        B, T, Hv, Kd = 1, args.T, 32, 128
        Ps = torch.randn((7, B, Hv, Kd, Kd), generator=g, device=dev) * (Kd ** -0.5)
        Sl = torch.randn((7, B, Hv, Kd, Kd), generator=g, device=dev)
        S_in = torch.empty((B, Hv, Kd, Kd), device=dev)
        qm = torch.randn((B * T, Hv, Kd), generator=g, device=dev) * 0.1
        o = torch.randn((B * T, Hv, Kd), generator=g, device=dev)

        def fn():
            nv.gdn_state_combine(Ps, Sl, None, out=S_in)
            nv.gdn_scan_correct(qm, S_in, o, B, T)
    else:
        raise SystemExit("unknown kernel case")
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    if args.flush:
        # L2 written over before each launch; each launch timed on its own
        flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        for s, e in ev:
            flush.fill_(1)
            s.record(stream)
            fn()
            e.record(stream)
        torch.cuda.synchronize()
        ms = sum(s.elapsed_time(e) for s, e in ev) / args.steps
    else:
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record(stream)
        for _ in range(args.steps):
            fn()
        e.record(stream)
        torch.cuda.synchronize()
        ms = s.elapsed_time(e) / args.steps
    nv.check_device_error()
    print(json.dumps({"kernel_case": args.kernel_case, "ms_per_launch": ms, "l2_flushed": bool(args.flush),
                      "M": args.M, "N": args.N, "K": args.K, "T": args.T}))


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-sample-tokens", type=int, default=512)
    ap.add_argument("--ref-tokens", type=int, default=64)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--study", action="store_true",
                    help="print the mechanism-study tables (sensitivity replay, lockstep, impulse, gate noise)")
    ap.add_argument("--kernel-case", choices=["gemm", "quant", "scan", "gate", "conv", "correct", "statepass",
                                              "decode", "layer"],
                    default=None,
                    help="profile helper: run one kernel on a fixed case and exit")
    ap.add_argument("--M", type=int, default=8192)
    ap.add_argument("--N", type=int, default=12288)
    ap.add_argument("--K", type=int, default=5120)
    ap.add_argument("--T", type=int, default=4096)
    ap.add_argument("--flush", action="store_true", help="kernel case: write over L2 before each launch")
    args = ap.parse_args(argv)
    if args.kernel_case:
        kernel_case(args)
        return 0
    if args.study:
        print(json.dumps(run_studies(args)), flush=True)
        return 0
    args.warmup = max(args.warmup, 3)
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank != 0:
            return 0
        print(json.dumps(run_reference(args)), flush=True)
        return 0

    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    try:
        out = run_ours(args, rank, world, local_rank)
        if rank == 0:
            if world == 1 and not args.no_cpu_baseline:
                out["cpu_baseline"] = cpu_baseline(args.cpu_sample_tokens, 2)
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
