#!/usr/bin/env python3
"""Benchmark of the NVFP4 W4A4 linear layer on B200.

One step = the whole hot path on one batch: NVFP4-quantize the activation
(nvfp4_quantize) and run the block-scaled W4A4 GEMM against the pre-quantized
weight (nvfp4_gemm) -- exactly the two launches w4a4_gemm makes -- on the
prefill MLP gate/up workload (X bf16 [32768, 5120], W [34816, 5120], BF16
out).  Weights are quantized offline (untimed); the activation global scale is
a static calibrated scale (untimed), as in the pages' checkpoints.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]

Prints one JSON line.  Under torchrun each rank runs an independent replica
(the layer is data-parallel over tokens and needs no collective); the time is
the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import re
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from nvfp4_w4a4_quantized_06_b200 import workloads as W  # noqa: E402

HEADLINE = "prefill_mlp_gate_up"
METRIC = "W4A4 GEMM TFLOPS (incl. act quantize) & % dense FP4 peak; quantize GB/s"
FP4_OVER_BF16 = 4.0          # nominal dense FP4 / BF16 tensor throughput ratio on B200
FP4_SPEC_TFLOPS = 9000.0     # NVIDIA's dense FP4 figure, for context
L2_BYTES = 126e6             # B200 L2


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "src": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "src": "fallback"}


# --------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples during the timed region (clocks and throttle reasons)."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = os.path.join(ROOT, "_build", f"nvfp4_clocks_{os.getpid()}.csv")

    def start(self):
        os.makedirs(os.path.dirname(self.path), exist_ok=True)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (FileNotFoundError, OSError):
            self.proc = None
            if os.path.exists(self.path):
                os.unlink(self.path)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = max(float(r[2]) for r in rows if r[2].replace(".", "").isdigit())
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower().startswith("active")})
        loaded = [s for s in sm if s > 0.5 * smax] or sm
        cap = sum(1 for r in rows if r[8].lower().startswith("active")) / len(rows)
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": smax, "reasons": reasons,
                "samples": len(rows), "power_cap_share": round(cap, 3),
                "power_w_max": max(float(r[3]) for r in rows if r[3].replace(".", "").isdigit())}


def fp4_peak_for(pk, clocks):
    """The dense FP4 denominator for a kernel timed in this run: 4 x the
    measured BF16 GEMM rate (the nominal FP4/BF16 ratio), taken at the burst
    figure unless the power cap held the clocks for most of the timed region,
    in which case the sustained (power-capped) figure applies."""
    share = clocks.get("power_cap_share") or 0.0
    if "sw_power_cap" in clocks.get("reasons", []) and share > 0.5:
        return pk["bf16_tflops_sustained"] * FP4_OVER_BF16, "sustained"
    return pk["bf16_tflops"] * FP4_OVER_BF16, "burst"


# ---------------------------------------------------------------- helpers
def max_over_ranks(values, world: int, device):
    """Elementwise maximum of per-rank timings (the slowest replica sets the
    job's time); a no-op on one rank."""
    if world <= 1:
        return list(values)
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return t.tolist()


def job_throughput(work_per_rank: float, world: int, ms: float) -> float:
    """Whole-job rate: every replica processes work_per_rank units in the
    (max-over-ranks) time ms; returns units per second / 1e12."""
    return work_per_rank * world / (ms * 1e-3) / 1e12


def quantized_weight(wl, dev):
    """Offline weight preparation: per-module quantize into the fused buffer,
    then the fused-group global-scale harmonization (untimed)."""
    from nvfp4_w4a4_quantized_06_b200 import native
    K, N = wl.K, wl.N
    offs = np.concatenate([[0], np.cumsum(wl.modules)]).astype(np.int64)
    codes = torch.empty((N, K // 2), dtype=torch.uint8, device=dev)
    sf = torch.empty(native.sf_bytes(N, K), dtype=torch.uint8, device=dev)
    gs = []
    for m in range(len(wl.modules)):
        wd = W.make_w(wl, m).to(dev)
        g = native.amax_gscale(wd)
        native.quantize(wd, g, codes=codes[offs[m]:offs[m + 1]], sf=sf, sf_row0=int(offs[m]), sf_rows_total=N)
        gs.append(g)
        del wd
    gw = native.harmonize(sf, N, K, offs, torch.cat(gs)) if len(gs) > 1 else gs[0]
    return codes, sf, gw


GEMM_SOURCES = ("gemm.cuh", "gemm_pair.cuh", "ptx.cuh")
QUANT_SOURCES = ("quantize.cuh", "ptx.cuh")


def kernel_src_hash(files=GEMM_SOURCES):
    """Digest of the sources a kernel is compiled from (its launch shape lives
    in nvfp4w4a4.cu's plan; a change there that touches the kernel's launch
    must refresh profiles/dram_traffic.json by hand)."""
    h = hashlib.sha256()
    for f in files:
        text = open(os.path.join(ROOT, "nvfp4_w4a4_quantized_06_b200", "csrc", f), encoding="utf-8").read()
        # comments do not change the kernel: hash the code only
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        code = (line.split("//", 1)[0].rstrip() for line in text.splitlines())
        text = "\n".join(line for line in code if line)
        h.update(text.encode())
    return h.hexdigest()[:16]


def recorded_traffic(name: str, files=GEMM_SOURCES):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(path):
        return None
    d = json.load(open(path)).get(name)
    if not d or d.get("src_hash") != kernel_src_hash(files):
        return None
    return d.get("bytes_per_launch")


def quant_bytes(M, K):
    return M * K * 2 + M * K // 2 + ((M + 127) // 128 * 128) * (K // 16)


# ------------------------------------------------------------ native arm
def run_native(args, rank, world, dev):
    from nvfp4_w4a4_quantized_06_b200 import native
    wl = W.WORKLOADS[args.workload]
    M, N, K = wl.M, wl.N, wl.K
    x_cpu = W.make_x(wl)
    x = x_cpu.to(dev)
    w_codes, w_sf, gw = quantized_weight(wl, dev)
    gx = native.amax_gscale(x)                       # static calibrated activation scale
    y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    a_codes = torch.empty((M, K // 2), dtype=torch.uint8, device=dev)
    a_sf = torch.empty(native.sf_bytes(M, K), dtype=torch.uint8, device=dev)
    ws_bytes = native.lib().nvfp4_gemm_workspace_bytes(M, N, K)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)

    def step():
        native.quantize(x, gx, codes=a_codes, sf=a_sf)
        native.gemm(a_codes, a_sf, gx, w_codes, w_sf, gw, out=y, workspace=ws)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert native.last_device_status() == 0

    stream = torch.cuda.current_stream()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    sampler = ClockSampler(dev.index if dev.index is not None else 0)
    sampler.start()
    time.sleep(0.3)
    launches0 = native.launch_count()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for s in range(args.steps):
        ev[s][0].record(stream)
        native.quantize(x, gx, codes=a_codes, sf=a_sf)
        ev[s][1].record(stream)
        native.gemm(a_codes, a_sf, gx, w_codes, w_sf, gw, out=y, workspace=ws)
        ev[s][2].record(stream)
    t_end.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    launches = native.launch_count() - launches0
    clocks = sampler.stop()
    flags = native.last_device_status()
    assert flags == 0, f"device error flags {flags}"

    total_ms = t_start.elapsed_time(t_end)
    tq = [ev[s][0].elapsed_time(ev[s][1]) for s in range(args.steps)]
    tg = [ev[s][1].elapsed_time(ev[s][2]) for s in range(args.steps)]
    total_ms, sq, sg = max_over_ranks([total_ms, sum(tq), sum(tg)], world, dev)
    ms_per_step = total_ms / args.steps
    flops = 2.0 * M * N * K
    value = job_throughput(flops, world, ms_per_step)
    pk = peaks()
    tq_ms, tg_ms = sq / args.steps, sg / args.steps
    fp4_peak, peak_kind = fp4_peak_for(pk, clocks)
    fp4_peak_burst = pk["bf16_tflops"] * FP4_OVER_BF16
    fp4_peak_sust = pk["bf16_tflops_sustained"] * FP4_OVER_BF16
    gemm_tflops = flops / (tg_ms * 1e-3) / 1e12
    q_gbs = quant_bytes(M, K) / (tq_ms * 1e-3) / 1e9

    # ---- end to end through the public one-call API, host buffers
    e2e = None if args.no_e2e else measure_e2e(native, x_cpu, gx, w_codes, w_sf, gw, M, N, K, dev, world,
                                               steps=min(args.steps, 50))

    also = {}
    if world == 1 and not args.headline_only:
        also = measure_secondary(native, dev)
        torch.cuda.empty_cache()

    xb, yb = M * K * x.element_size(), M * N * 2
    l2_note = (f"inputs larger than L2 (X {xb / 1e6:.0f} MB, Y {yb / 1e6:.0f} MB per step; no flush)"
               if xb + yb > L2_BYTES else f"X {xb / 1e6:.1f} MB and Y {yb / 1e6:.1f} MB fit in L2 (warm, no flush)")
    out = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "nvfp4 (e2m1 x e4m3/16 x fp32 scale) -> fp32 accumulate -> bf16",
        "data": "synthetic (seeded PCG64 Gaussians with block outliers; random-init weights)",
        "config": {"workload": f"{wl.name} {M}x{N}x{K}", "M": M, "N": N, "K": K, "x_dtype": "bf16",
                   "y_dtype": "bf16", "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2": l2_note},
        "breakdown_ms": {"quantize": round(tq_ms, 4), "gemm": round(tg_ms, 4)},
        "quantize_gbs": round(q_gbs, 1),
        "quantize_frac_hbm": round(q_gbs / pk["hbm_gbs"], 3),
        "gemm_tflops": round(gemm_tflops, 1),
        "frac_fp4_spec": round(value / world / FP4_SPEC_TFLOPS, 3),
        "frac_fp4_incl_quantize": round(value / world / fp4_peak, 3),
        "roofline": {"bound": "tensor", "kernel": "nvfp4_gemm_pair_kernel<bf16>",
                     "achieved": round(gemm_tflops, 1), "peak": round(fp4_peak, 1), "unit": "TFLOP/s",
                     "frac": round(gemm_tflops / fp4_peak, 3),
                     "peak_src": f"{pk['src']} bf16 {peak_kind} x {FP4_OVER_BF16:g} (nominal fp4/bf16), "
                                 f"chosen from the sampled clocks (sustained only when sw_power_cap held "
                                 f"most samples); burst {fp4_peak_burst:.1f} -> frac "
                                 f"{gemm_tflops / fp4_peak_burst:.3f}, sustained {fp4_peak_sust:.1f} -> frac "
                                 f"{gemm_tflops / fp4_peak_sust:.3f}, NVIDIA dense spec {FP4_SPEC_TFLOPS:.0f} -> "
                                 f"frac {gemm_tflops / FP4_SPEC_TFLOPS:.3f}",
                     "traffic": recorded_traffic("gemm_prefill_mlp_gate_up")},
        "roofline_quant": {"bound": "hbm", "kernel": "quantize_tma_kernel<bf16>",
                           "achieved": round(q_gbs, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
                           "frac": round(q_gbs / pk["hbm_gbs"], 3),
                           "per_unit": "2 B read + 0.5 B codes + 1/16 B scale per element",
                           "traffic": recorded_traffic("quantize_prefill_mlp_gate_up", QUANT_SOURCES)},
        "e2e": e2e,
        "gpu_launches": int(launches),
        "clocks": clocks,
    }
    if also:
        out["also"] = also
    return out


def measure_e2e(native, x_cpu, gx, w_codes, w_sf, gw, M, N, K, dev, world, steps=20):
    """Same metric through w4a4_gemm with host buffers: every step copies its X
    from pinned host memory, runs the layer and reads its Y back into pinned
    host memory, all inside the timed region.  Steps alternate between two
    streams with their own device and host buffers, the way a serving loop
    pipelines them: one step's Y read-back (the PCIe-bound part) overlaps the
    next step's X copy and layer."""
    x_host = x_cpu.pin_memory()
    lanes = []
    for _ in range(2):
        lanes.append({"stream": torch.cuda.Stream(device=dev),
                      "y_host": torch.empty((M, N), dtype=torch.bfloat16).pin_memory(),
                      "x_dev": torch.empty_like(x_host, device=dev),
                      "y_dev": torch.empty((M, N), dtype=torch.bfloat16, device=dev),
                      "ws": torch.empty(native.linear_workspace_bytes(M, N, K), dtype=torch.uint8, device=dev)})

    def one(ln):
        with torch.cuda.stream(ln["stream"]):
            ln["x_dev"].copy_(x_host, non_blocking=True)
            native.linear(ln["x_dev"], gx, w_codes, w_sf, gw, out=ln["y_dev"], workspace=ln["ws"])
            ln["y_host"].copy_(ln["y_dev"], non_blocking=True)

    main = torch.cuda.current_stream()
    for ln in lanes:                               # warm-up, one step per lane
        ln["stream"].wait_stream(main)
        one(ln)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(main)
    for ln in lanes:
        ln["stream"].wait_event(e0)
    for i in range(steps):
        one(lanes[i % 2])
    for ln in lanes:
        main.wait_stream(ln["stream"])
    e1.record(main)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    ms = max_over_ranks([ms], world, dev)[0]
    del lanes
    return {"value": round(job_throughput(2.0 * M * N * K, world, ms), 2), "unit": "TFLOP/s",
            "ms_per_step": round(ms, 3), "steps": steps, "h2d_bytes_per_step": x_host.numel() * 2,
            "d2h_bytes_per_step": M * N * 2, "streams": 2}


SECONDARY = ("gdn_qkv_z", "gdn_gates_ab", "decode_out_proj", "decode_down_proj", "gdn_gates_fused_activations",
             "fake_quant_bf16", "fp8_kv_quantize", "rmsnorm_quantize", "harmonize_requant_qkv_z")


def measure_secondary(native, dev, only=None):
    """The other workloads of the layer and the rows built beyond it, one line
    each (median of CUDA events): GDN fused groups (TFLOP/s), decode shapes
    (HBM GB/s over weights+X+Y, rotating over >= 4x L2 of weight copies inside
    a CUDA graph), then the gate epilogue, fake-quant, FP8 KV quantize, the
    RMSNorm-fused quantize and the re-quantizing harmonize.  `only`: a set of
    line names to run (all when None)."""
    res = {}
    pk = peaks()
    want = (lambda name: True) if only is None else (lambda name: name in only)
    flush = torch.empty(512 * 2 ** 20, dtype=torch.uint8, device=dev)

    def timed(fn, reps=12):
        times = []
        for i in range(reps):
            flush.zero_()
            # keep the GPU busy while the host enqueues the start event and
            # the call, so that host-side call overhead is not timed as GPU time
            torch.cuda._sleep(100000)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            if i >= 2:
                times.append(e0.elapsed_time(e1))
        return statistics.median(times)

    def hbm(byts, ms):
        return {"gbs_algorithmic": round(byts / (ms * 1e-3) / 1e9, 1),
                "frac_hbm": round(byts / (ms * 1e-3) / 1e9 / pk["hbm_gbs"], 3)}

    for name in ("gdn_qkv_z", "gdn_gates_ab"):
        if not want(name):
            continue
        wl = W.WORKLOADS[name]
        x = W.make_x(wl).to(dev)
        wc, wsf, gw = quantized_weight(wl, dev)
        gx = native.amax_gscale(x)
        y = torch.empty((wl.M, wl.N), dtype=torch.bfloat16, device=dev)
        ws = torch.empty(native.linear_workspace_bytes(wl.M, wl.N, wl.K), dtype=torch.uint8, device=dev)
        ms = timed(lambda: native.linear(x, gx, wc, wsf, gw, out=y, workspace=ws))
        byts = wl.M * wl.K * 2 + wl.N * wl.K // 2 + wl.N * wl.K // 16 + wl.M * wl.N * 2
        res[name] = {"shape": f"{wl.M}x{wl.N}x{wl.K}", "ms": round(ms, 4),
                     "tflops": round(wl.flops / (ms * 1e-3) / 1e12, 1), **hbm(byts, ms),
                     "l2": "512 MB flush between reps"}
        if name == "gdn_gates_ab":
            # the W4A4 product against the unquantized one (float64, untimed):
            # the pages put 4-bit GEMM error on real gate inputs at 8.5-11%
            w64 = torch.cat([W.make_w(wl, m) for m in range(len(wl.modules))]).to(dev).double()
            y32 = native.linear(x, gx, wc, wsf, gw, out_dtype=torch.float32, workspace=ws).double()
            y64 = x.double() @ w64.T
            res[name]["gemm_rel_error"] = round(float((y32 - y64).norm() / y64.norm()), 5)
            del w64, y32, y64
        del x, wc, wsf, y, ws
    for name in ("decode_out_proj", "decode_down_proj"):
        if not want(name):
            continue
        wl = W.WORKLOADS[name]
        x = W.make_x(wl).to(dev)
        wc, wsf, gw = quantized_weight(wl, dev)
        gx = native.amax_gscale(x)
        wbytes = wc.numel() + wsf.numel()
        copies = max(4, int(np.ceil(4 * 126e6 / wbytes)))
        wcs = [wc.clone() for _ in range(copies)]
        wsfs = [wsf.clone() for _ in range(copies)]
        y = torch.empty((wl.M, wl.N), dtype=torch.bfloat16, device=dev)
        ws = torch.empty(native.linear_workspace_bytes(wl.M, wl.N, wl.K), dtype=torch.uint8, device=dev)
        for i in range(copies):                   # warm-up outside capture
            native.linear(x, gx, wcs[i], wsfs[i], gw, out=y, workspace=ws)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = 5
        per_call = {}
        for label, fn in (("layer", native.linear), ("fused", None)):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                for i in range(copies):
                    if fn is None:
                        native.linear_fused(x, gx, wcs[i], wsfs[i], gw, out=y)
                    else:
                        fn(x, gx, wcs[i], wsfs[i], gw, out=y, workspace=ws)
            g.replay()
            torch.cuda.synchronize()
            e0.record()
            for _ in range(reps):
                g.replay()
            e1.record()
            torch.cuda.synchronize()
            per_call[label] = e0.elapsed_time(e1) / (reps * copies)
            del g
        ms = per_call["layer"]
        byts = wbytes + wl.M * wl.K * 2 + wl.M * wl.N * 2
        res[name] = {"shape": f"{wl.M}x{wl.N}x{wl.K}", "us": round(ms * 1e3, 2), **hbm(byts, ms),
                     "l2": f"CUDA graph over {copies} weight copies ({copies * wbytes / 1e6:.0f} MB)",
                     # the same calls through the one-kernel variant (activation quantized in the GEMM)
                     "fused_prologue_us": round(per_call["fused"] * 1e3, 2)}
        del wcs, wsfs, x, y, ws
    if want("gdn_gates_fused_activations"):
        wl = W.WORKLOADS["gdn_gates_ab"]
        x = W.make_x(wl).to(dev)
        wc, wsf, gw = quantized_weight(wl, dev)
        gx = native.amax_gscale(x)
        out = torch.empty((wl.M, wl.N), dtype=torch.float32, device=dev)
        ws = torch.empty(native.linear_workspace_bytes(wl.M, wl.N, wl.K), dtype=torch.uint8, device=dev)
        ms = timed(lambda: native.gdn_gates(x, gx, wc, wsf, gw, n_a=wl.modules[0], out=out, workspace=ws))
        byts = wl.M * wl.K * 2 + wl.N * wl.K // 2 + wl.N * wl.K // 16 + wl.M * wl.N * 4
        res["gdn_gates_fused_activations"] = {"shape": f"{wl.M}x{wl.N}x{wl.K}", "ms": round(ms, 4), **hbm(byts, ms),
                                              "l2": "512 MB flush between reps"}
        del x, wc, wsf, out, ws
    wl = W.WORKLOADS["prefill_mlp_gate_up"]
    x = W.make_x(wl).to(dev) if (want("fake_quant_bf16") or want("rmsnorm_quantize")) else None
    if want("fake_quant_bf16"):
        g = native.amax_gscale(x)
        fq = torch.empty_like(x)
        st = torch.empty(2, dtype=torch.float64, device=dev)
        ms = timed(lambda: native.lib().nvfp4_fake_quant(x.data_ptr(), 0, wl.M, wl.K, wl.K, g.data_ptr(), fq.data_ptr(),
                                                         0, wl.K, st.data_ptr(),
                                                         torch.cuda.current_stream().cuda_stream))
        res["fake_quant_bf16"] = {"shape": f"{wl.M}x{wl.K}", "ms": round(ms, 4), **hbm(wl.M * wl.K * 4, ms),
                                  "rel_error": round(float(np.sqrt(st[0].item() / st[1].item())), 5)}
        del fq
    if want("fp8_kv_quantize"):
        # 32 seqs x 4096 tokens, K and V: seeded N(0, 1) values and the static
        # scale amax / 448.  How often x / s lands exactly on an E4M3 midpoint
        # depends on s: none for this input's scale, about 1% for scales with
        # few significant bits, where the kernel settles those ties.
        gen = torch.Generator(device=dev)
        gen.manual_seed(0)
        kv = torch.randn(32 * 4096 * 4 * 256 * 2, dtype=torch.float32, device=dev, generator=gen).to(torch.bfloat16)
        sc = (kv.abs().max().float() / 448.0).reshape(1)
        q8 = torch.empty(kv.numel(), dtype=torch.uint8, device=dev)
        ms = timed(lambda: native.fp8_quantize(kv, sc, out=q8))
        res["fp8_kv_quantize"] = {"shape": "32x4096 tokens x 4 kv heads x 256 x (K,V) bf16", "ms": round(ms, 4),
                                  **hbm(kv.numel() * 3, ms), "scale": float(sc.item())}
        del kv, q8
    if want("rmsnorm_quantize"):
        # quantize fused into the RMSNorm that produces this activation
        wn = W.norm_weight(wl.K, seed=11).to(dev)
        gy = native.amax_gscale(torch.nn.functional.rms_norm(x, (wl.K,), weight=wn, eps=1e-6))
        yc = torch.empty((wl.M, wl.K // 2), dtype=torch.uint8, device=dev)
        ysf = torch.empty(native.sf_bytes(wl.M, wl.K), dtype=torch.uint8, device=dev)
        yinv = torch.empty(wl.M, dtype=torch.float32, device=dev)
        ms = timed(lambda: native.rmsnorm_quantize(x, wn, 1e-6, gy, codes=yc, sf=ysf, inv=yinv))

        def unfused():
            y = torch.nn.functional.rms_norm(x, (wl.K,), weight=wn, eps=1e-6)
            native.quantize(y, gy, codes=yc, sf=ysf)

        ms_unfused = timed(unfused)
        byts = wl.M * wl.K * 2 + wl.M * wl.K // 2 + wl.M * wl.K // 16 + wl.K * 2 + wl.M * 4
        res["rmsnorm_quantize"] = {"shape": f"{wl.M}x{wl.K} bf16 residual", "ms": round(ms, 4), **hbm(byts, ms),
                                   "unfused_torch_rms_norm_then_quantize_ms": round(ms_unfused, 4),
                                   "l2": "512 MB flush between reps"}
        del yc, ysf, yinv
    del x
    if want("harmonize_requant_qkv_z"):
        # re-quantizing harmonize of the fused qkv+z weight (offline; in place, so
        # every rep re-encodes the previous rep's output)
        wl = W.WORKLOADS["gdn_qkv_z"]
        wc, wsf, gw = quantized_weight(wl, dev)
        offs = [0, wl.modules[0], wl.N]
        gsm = torch.cat([gw, gw * 0.8])
        ms = timed(lambda: native.harmonize_requant(wc, wsf, wl.K, offs, gsm))
        byts = 2 * (wl.N * wl.K // 2 + wl.N * wl.K // 16)
        res["harmonize_requant_qkv_z"] = {"shape": f"{wl.N}x{wl.K}", "ms": round(ms, 4), **hbm(byts, ms),
                                          "l2": "512 MB flush between reps"}
        del wc, wsf
    del flush
    assert native.last_device_status() == 0
    return res


# ------------------------------------------------------------ CPU oracle
def oracle_sample(wl, rows: int, cols: int, seed: int = 7):
    import oracle
    x = W.make_x(wl)
    r = W.sample_rows(wl.M, rows, seed=seed)
    xs = x[torch.from_numpy(r)].float().numpy()
    w = W.make_w(wl, 0)
    c = W.sample_rows(wl.modules[0], cols, seed=seed + 1)
    wsub = w[torch.from_numpy(c)].float().numpy()
    gx = oracle.global_scale(x.float().numpy())
    gw = oracle.global_scale(w.float().numpy())
    wc, wsf = oracle.quantize(wsub, gw)                  # offline weight prep, untimed
    return xs, gx, wc, wsf, gw


def time_oracle(wl, seconds: float = 10.0, rows: int = 128, cols: int = 2048):
    """The oracle (quantize activation rows, float64 dequantize + GEMM) on a
    bounded sample of the workload, repeated for about `seconds`."""
    import oracle
    xs, gx, wc, wsf, gw = oracle_sample(wl, rows, cols)
    oracle.linear_reference(xs, gx, wc, wsf, gw)          # warm
    reps, t0 = 0, time.perf_counter()
    while True:
        oracle.linear_reference(xs, gx, wc, wsf, gw)
        reps += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    flops = 2.0 * xs.shape[0] * wc.shape[0] * wl.K * reps
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    return {"value": round(flops / el / 1e12, 6), "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "sample": f"{xs.shape[0]} activation rows x {wc.shape[0]} weight rows x K={wl.K} "
                      f"(quantize + float64 dequantize/GEMM), {reps} reps in {el:.1f} s; "
                      f"OpenMP threads {oracle.num_threads()}, numpy BLAS threads as configured"}


def oracle_table():
    """The oracle, as it stands, on every configuration on the host cores:
    the global scale and quantize of each full activation tensor, and the
    whole linear (activation quantize, float64 dequantize and GEMM) in full
    for the configurations with at most 4096 activation rows x 128 weight
    rows of work per K, else on 256 seeded activation rows, extrapolated
    linearly in M.  Weight preparation is untimed.  No GPU is used."""
    import oracle
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    table = []
    for name, wl in W.WORKLOADS.items():
        x = W.make_x(wl).float().numpy()
        t0 = time.perf_counter()
        gx = oracle.global_scale(x)
        oracle.quantize(x, gx)
        tq = time.perf_counter() - t0
        K, N = wl.K, wl.N
        offs = np.concatenate([[0], np.cumsum(wl.modules)]).astype(np.int64)
        wsf = np.zeros(oracle.sf_bytes(N, K), np.uint8)
        wcs, gws = [], []
        for m in range(len(wl.modules)):
            w = W.make_w(wl, m).float().numpy()
            g = oracle.global_scale(w)
            wcs.append(oracle.quantize(w, g, sf=wsf, sf_row0=int(offs[m]))[0])
            gws.append(g)
        gw = oracle.harmonize(wsf, K, offs, gws) if len(gws) > 1 else gws[0]
        wc = np.concatenate(wcs)
        full = wl.M * N <= 4096 * 128
        rows = np.arange(wl.M) if full else W.sample_rows(wl.M, 256)
        t0 = time.perf_counter()
        oracle.linear_reference(x[rows], gx, wc, wsf, gw)
        tg = (time.perf_counter() - t0) * (wl.M / len(rows))
        table.append({"workload": f"{name} {wl.M}x{N}x{K}", "quantize_s": round(tq, 3),
                      "quantize_gbs": round(wl.M * K * (2.0 if wl.x_dtype == torch.bfloat16 else 4.0) / tq / 1e9, 3),
                      "linear_s": round(tg, 3), "linear_gflops": round(wl.flops / tg / 1e9, 2),
                      "linear_rows": "all" if full else f"{len(rows)} of {wl.M}, extrapolated"})
        del x, wcs, wc, wsf
    return {"oracle_table": table, "cores": cores, "openmp_threads": oracle.num_threads()}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return None
    wl = W.WORKLOADS[args.workload]
    import oracle
    xs, gx, wc, wsf, gw = oracle_sample(wl, 64, 1024)
    for _ in range(args.warmup):
        oracle.linear_reference(xs, gx, wc, wsf, gw)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.linear_reference(xs, gx, wc, wsf, gw)
    el = time.perf_counter() - t0
    flops = 2.0 * xs.shape[0] * wc.shape[0] * wl.K * args.steps
    value = flops / el / 1e12
    cores = len(os.sched_getaffinity(0))
    sample = f"{xs.shape[0]} activation rows x {wc.shape[0]} weight rows x K={wl.K} per step"
    return {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s",
            "n_gpus": int(os.environ.get("WORLD_SIZE", "1")), "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(el / args.steps * 1e3, 3), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32 quantize, f64 GEMM", "data": "synthetic",
            "config": {"workload": f"{wl.name} {wl.M}x{wl.N}x{wl.K}", "M": wl.M, "N": wl.N, "K": wl.K},
            "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--workload", default=HEADLINE, choices=sorted(W.WORKLOADS))
    ap.add_argument("--headline-only", action="store_true", help="skip the secondary workloads")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end leg")
    ap.add_argument("--oracle-table", action="store_true",
                    help="time the CPU oracle on every configuration (host cores only) and exit")
    ap.add_argument("--only", default=None,
                    help="comma-separated secondary lines to measure instead of the headline "
                         f"(one GPU; any of {', '.join(SECONDARY)}); prints them as one JSON line")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    if args.oracle_table:
        print(json.dumps(oracle_table()), flush=True)
        return

    if args.impl == "reference":
        out = run_reference(args)
        if out is not None:
            print(json.dumps(out), flush=True)
        return

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if args.only is not None:
        names = {n.strip() for n in args.only.split(",") if n.strip()}
        unknown = names - set(SECONDARY)
        if unknown:
            raise SystemExit(f"--only: unknown line(s) {sorted(unknown)}; choose from {list(SECONDARY)}")
        from nvfp4_w4a4_quantized_06_b200 import native
        print(json.dumps({"only": measure_secondary(native, dev, only=names)}), flush=True)
        return
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=dev)
    out = run_native(args, rank, world, dev)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = time_oracle(W.WORKLOADS[args.workload])
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
