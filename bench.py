#!/usr/bin/env python
"""Benchmark of the MX hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--no-breakdown]

One step = one pass of the weight-quantisation workload over a 4096 x 4096 bf16 matrix
(N(0, 0.02) with 0.1% N(0, 1) outliers): MXFP4 (E2M1, block 32, E8M0, floor scale) and
NVFP4 (E2M1, block 16, UE4M3 + fp32 tensor scale), each emitting both the row-major and
the tcgen05 scale layouts.  value = algorithmic bytes of the step / step time (GB/s).
The input (32 MiB) is smaller than L2, so consecutive steps rotate over 8 copies of the
weight (256 MiB): each step reads its input from HBM.  K steps are timed back to back in
one CUDA-event pair.  Every other row of the hot path (row-wise
MXFP8 quantise + dequantise, dual-orientation quantisation, dequantisation, the two
block-scaled matmuls) is measured in "breakdown", each against its own roofline.

Multi-GPU (torchrun): every rank quantises its own weight matrix (independent units, no
data-path collective); value = all ranks' bytes / the slowest rank's time.
"""
from __future__ import annotations

import argparse
import json
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

METRIC = "MX quantize GB/s (frac of HBM peak); block-scaled GEMM TFLOPS (frac of MX peak)"
HBM_NOMINAL_GBS = 8000.0
MX_NOMINAL_TFLOPS = 4500.0
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# algorithmic bytes (read input once + write codes and scales once)
R2 = C2 = 4096
BYTES_MXFP4 = R2 * C2 * 2 + R2 * C2 // 2 + 2 * (R2 * C2 // 32)            # 42,991,616
BYTES_NVFP4 = R2 * C2 * 2 + R2 * C2 // 2 + 2 * (R2 * C2 // 16) + 4         # 44,040,196
NCU_TRAFFIC_NVFP4 = 67149056      # dram read + write bytes of one NVFP4 call (both kernels, ncu, L2 flushed per kernel)
NCU_TRAFFIC_MXFP4 = 33568768      # same for mx_rows_kernel<E2M1, floor, both layouts>
STEP_BYTES = BYTES_MXFP4 + BYTES_NVFP4
NROT = 8                 # rotating copies of the weight (8 x 32 MiB > 2 x L2)


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return dict(FALLBACK, source="fallback")


# ----------------------------------------------------------------------------- utilities
class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.2)
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
        for ln in getattr(self, "lines", []):
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        out = {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax, "reasons": sorted(reasons),
               "samples": len(sm)}
        pw = []
        for ln in getattr(self, "lines", []):
            try:
                pw.append(float(ln.split(",")[3]))
            except (ValueError, IndexError):
                pass
        if pw:
            out["power_w_max"] = max(pw)
        return out


def max_over_ranks(ms, world, dev):
    """The job's time: the slowest rank's device time (identity on one rank)."""
    if world <= 1:
        return ms
    t = torch.tensor([ms], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_throughput_gbs(bytes_per_step, steps, world, total_ms):
    """Whole-job GB/s: every rank processes its own units (weak scaling)."""
    return bytes_per_step * world * steps / (total_ms * 1e-3) / 1e9


def to_dev(bits, dev):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)


def event_pair():
    return torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)


# ----------------------------------------------------------------------------- our step
class WeightQuantStep:
    """MXFP4 (floor) + NVFP4 quantisation of one 4096 x 4096 bf16 weight, both layouts."""

    def __init__(self, mx, x_dev):
        from microscaling_precision_number_b200 import _lib as L
        self.mx, self.L = mx, L
        self.x = x_dev
        dev = x_dev.device
        R, C = x_dev.shape
        self.R, self.C = R, C
        self.e4 = torch.empty(R * C // 2, dtype=torch.uint8, device=dev)
        self.s4 = torch.empty(R * C // 32, dtype=torch.uint8, device=dev)
        self.s4t = torch.empty(mx.scale_bytes(R, C // 32, "tcgen05"), dtype=torch.uint8, device=dev)
        self.en = torch.empty(R * C // 2, dtype=torch.uint8, device=dev)
        self.sn = torch.empty(R * C // 16, dtype=torch.uint8, device=dev)
        self.snt = torch.empty(mx.scale_bytes(R, C // 16, "tcgen05"), dtype=torch.uint8, device=dev)
        self.g = torch.empty(1, dtype=torch.float32, device=dev)
        self.launches_per_step = 3      # MXFP4 quantiser; NVFP4 maximum + quantiser (no padding at 4096)

    def mxfp4(self, stream):
        L = self.L
        L.check(L.lib.mx_quantize(self.x.data_ptr(), self.R, self.C, L.MX_FMT_E2M1, L.MX_AXIS_ROW,
                                  L.MX_SCALE_FLOOR_OCP, self.e4.data_ptr(), self.s4.data_ptr(), 3,
                                  self.s4t.data_ptr(), None, stream), "mx_quantize(mxfp4)")

    def nvfp4(self, stream):
        L = self.L
        L.check(L.lib.mx_quantize(self.x.data_ptr(), self.R, self.C, L.MX_FMT_NVFP4, L.MX_AXIS_ROW,
                                  L.MX_SCALE_CEIL_RECIPE, self.en.data_ptr(), self.sn.data_ptr(), 3,
                                  self.snt.data_ptr(), self.g.data_ptr(), stream), "mx_quantize(nvfp4)")

    def outputs(self):
        return [self.e4, self.s4, self.s4t, self.en, self.sn, self.snt, self.g]


def run_ours(args, rank, world, dev):
    import microscaling_precision_number_b200 as mx

    pk = peaks()
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    sptr = stream.cuda_stream
    x_bits = synth.weight_fp4(seed=rank)
    x0 = to_dev(x_bits, dev)
    # NROT copies of the weight (8 x 32 MiB, over twice L2): step k works on copy k % NROT,
    # so every timed step reads its input from HBM without an L2 flush in between.
    steps = [WeightQuantStep(mx, x0.clone()) for _ in range(NROT)]

    def run_steps(n, which="both"):
        for k in range(n):
            s = steps[k % NROT]
            if which in ("both", "mxfp4"):
                s.mxfp4(sptr)
            if which in ("both", "nvfp4"):
                s.nvfp4(sptr)

    run_steps(max(args.warmup, NROT))
    torch.cuda.synchronize()

    with ClockSampler(torch.cuda.current_device()) as clk:
        # soak: keep the GPU busy with the same steps for ~0.4 s so that the clock samples
        # below see it under load, then the timed region proper
        t0 = time.perf_counter()
        while time.perf_counter() - t0 < 0.4:
            run_steps(200)
            torch.cuda.synchronize()
        e0, e1 = event_pair()
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        e0.record(stream)
        run_steps(args.steps)
        e1.record(stream)
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
    total_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    ms_per_step = total_ms / args.steps
    value = job_throughput_gbs(STEP_BYTES, args.steps, world, total_ms)

    # per-call durations for the roofline: many launches of one call per event pair
    ncall = max(args.steps, 50)
    per = {}
    for which in ("mxfp4", "nvfp4"):
        run_steps(NROT, which)
        a, b = event_pair()
        a.record(stream)
        run_steps(ncall, which)
        b.record(stream)
        torch.cuda.synchronize()
        per[which] = a.elapsed_time(b) / ncall
    mean_mx, mean_nv = per["mxfp4"], per["nvfp4"]
    # DRAM bytes per call (read + write) from one ncu capture of the same kernels on this
    # workload (profiles/nvfp4_and_rows_weight4096.md); ncu replays each launch with a
    # flushed L2, so a kernel's outputs are still in L2 at its end and count as 0 written
    # bytes
    if mean_nv >= mean_mx:
        dom = {"kernel": "mx_quantize(NVFP4) call: nvfp4_amax_bulk_kernel + nvfp4_quant_bulk_kernel<both layouts>",
               "ms": mean_nv,
               "bytes": BYTES_NVFP4, "traffic": NCU_TRAFFIC_NVFP4}
    else:
        dom = {"kernel": "mx_quantize(MXFP4): mx_rows_kernel<E2M1,floor,both layouts>", "ms": mean_mx,
               "bytes": BYTES_MXFP4, "traffic": NCU_TRAFFIC_MXFP4}
    achieved = dom["bytes"] / (dom["ms"] * 1e-3) / 1e9
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": round(achieved / pk["hbm_gbs"], 4), "traffic": dom["traffic"],
                "peak_source": pk["source"] + " copy bandwidth (MEASURED_PEAKS hbm_gbs), burst",
                "kernel": dom["kernel"], "algorithmic_bytes_per_launch": dom["bytes"],
                "ms_per_launch": round(dom["ms"], 5),
                "calls": {"mxfp4_ms": round(mean_mx, 5), "mxfp4_GBps": round(BYTES_MXFP4 / mean_mx / 1e6, 1),
                          "nvfp4_ms": round(mean_nv, 5), "nvfp4_GBps": round(BYTES_NVFP4 / mean_nv / 1e6, 1),
                          "launches_timed": ncall},
                "frac_of_nominal_8TBps": round(achieved / HBM_NOMINAL_GBS, 4)}

    # end to end through the public API with host buffers (pinned), copies inside the timing.
    # Pipelined as a user would run a stream of weights: step k's upload, step k-1's
    # quantisation and step k-2's download overlap on three streams (two buffer sets,
    # ordered by events); the serial form (upload, quantise, download on one stream) is
    # reported beside it.
    sets = steps[:2]
    x_host = torch.from_numpy(x_bits.view(np.int16)).view(torch.bfloat16).pin_memory()
    outs_host = [[torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for o in st.outputs()] for st in sets]
    h2d = x_host.numel() * 2
    d2h = sum(o.numel() * o.element_size() for o in outs_host[0])
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    ev_up, ev_comp, ev_down = ([torch.cuda.Event() for _ in sets] for _ in range(3))

    def pipelined(n):
        for k in range(n):
            b = k % 2
            st = sets[b]
            up.wait_event(ev_comp[b])                  # the buffer's previous step has read it
            with torch.cuda.stream(up):
                st.x.copy_(x_host, non_blocking=True)
            ev_up[b].record(up)
            stream.wait_event(ev_up[b])
            stream.wait_event(ev_down[b])              # its previous outputs have been copied out
            st.mxfp4(sptr)
            st.nvfp4(sptr)
            ev_comp[b].record(stream)
            down.wait_event(ev_comp[b])
            with torch.cuda.stream(down):
                for h, d in zip(outs_host[b], st.outputs()):
                    h.copy_(d, non_blocking=True)
            ev_down[b].record(down)

    def serial(n):
        st = sets[0]
        for _ in range(n):
            st.x.copy_(x_host, non_blocking=True)
            st.mxfp4(sptr)
            st.nvfp4(sptr)
            for h, d in zip(outs_host[0], st.outputs()):
                h.copy_(d, non_blocking=True)

    def timed_e2e(run):
        run(2)
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        e0, e1 = event_pair()
        e0.record(stream)
        up.wait_event(e0)
        down.wait_event(e0)
        run(args.steps)
        for ev in ev_down:
            stream.wait_event(ev)
        e1.record(stream)
        torch.cuda.synchronize()
        return max_over_ranks(e0.elapsed_time(e1), world, dev)

    e2e_ms = timed_e2e(pipelined)
    ser_ms = timed_e2e(serial)
    e2e = {"value": round(job_throughput_gbs(STEP_BYTES, args.steps, world, e2e_ms), 2), "unit": "GB/s",
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
           "ms_per_step": round(e2e_ms / args.steps, 4),
           "form": "pipelined: upload / quantise / download of consecutive steps overlap on three streams",
           "serial": {"value": round(job_throughput_gbs(STEP_BYTES, args.steps, world, ser_ms), 2),
                      "ms_per_step": round(ser_ms / args.steps, 4)}}

    breakdown = None
    if not args.no_breakdown and rank == 0:
        breakdown = run_breakdown(mx, dev, pk)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(x_bits, target_s=args.cpu_seconds)

    if rank == 0:
        line = {"metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
                "data": "synthetic (numpy default_rng, seed = rank)",
                "config": {"workload": "weight_4096x4096_mxfp4_floor_and_nvfp4_both_scale_layouts",
                           "shape": [R2, C2], "formats": ["MXFP4 E2M1/E8M0 floor block 32",
                                                          "NVFP4 E2M1/UE4M3+fp32 block 16"],
                           "step_bytes": STEP_BYTES,
                           "l2": f"inputs larger than L2: steps rotate over {NROT} copies of the weight "
                                 f"({NROT * R2 * C2 * 2 >> 20} MiB)",
                           "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
                "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
                "gpu_launches": steps[0].launches_per_step * args.steps, "clocks": clk.summary()}
        if breakdown is not None:
            line["breakdown"] = breakdown
        print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- breakdown
def timed(fns, iters, stream):
    """Mean device time of one call, over `iters` calls cycling through `fns` (one closure
    per rotating buffer set), in a single event pair."""
    for f in fns:
        f()
    torch.cuda.synchronize()
    a, b = event_pair()
    a.record(stream)
    for i in range(iters):
        fns[i % len(fns)]()
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b) / iters


def best_of(fn, n, stream):
    """Shortest device time of n single calls, each between its own event pair (the way the
    bf16 matmul peak in MEASURED_PEAKS is taken: best of 10)."""
    best = float("inf")
    for _ in range(n):
        a, b = event_pair()
        a.record(stream)
        fn()
        b.record(stream)
        torch.cuda.synchronize()
        best = min(best, a.elapsed_time(b))
    return best


def soak_clocks(fn, seconds=1.5):
    """SM clock and throttle reasons while fn runs back to back for about `seconds` (the
    sampler's short idle lead-in and tail are a minority of the samples)."""
    with ClockSampler(torch.cuda.current_device()) as clk:
        t0 = time.perf_counter()
        while time.perf_counter() - t0 < seconds:
            for _ in range(16):
                fn()
            torch.cuda.synchronize()
    return clk.summary()


def run_breakdown(mx, dev, pk):
    stream = torch.cuda.current_stream()
    out = {}
    hbm = pk["hbm_gbs"]
    mx_peak = 2.0 * pk["bf16_tflops"]          # FP8 / mxf8f6f4 rate = 2 x the bf16 rate

    # C1: MXFP8 E4M3 row-wise quantise + dequantise, 1024 x 1024, 64 rotating copies (> L2)
    x1 = to_dev(synth.mx8_rowwise(), dev)
    xs = [x1.clone() for _ in range(64)]
    qs = [mx.quantize(x, "e4m3", "row", "ceil", layout="rowmajor") for x in xs]
    ys = [torch.empty_like(x) for x in xs]
    tq = timed([lambda x=x, q=q: mx.quantize(x, "e4m3", "row", "ceil", layout="rowmajor", out=q)
                for x, q in zip(xs, qs)], 256, stream)
    td = timed([lambda q=q, y=y: mx.dequantize(q, "rowmajor", out=y) for q, y in zip(qs, ys)], 256, stream)
    b1 = 1024 * 1024 * 2 + 1024 * 1024 + 1024 * 32
    out["mxfp8_rowwise_1024x1024"] = {"quantize_us": round(tq * 1e3, 2), "dequantize_us": round(td * 1e3, 2),
                                    "quantize_GBps": round(b1 / tq / 1e6, 1),
                                    "dequantize_GBps": round(b1 / td / 1e6, 1),
                                    "frac_hbm": round(b1 / tq / 1e6 / hbm, 4),
                                    "note": "3.2 MB per call, back-to-back calls from Python: host-launch bound"}
    # the same 64 calls captured once in a CUDA graph and replayed: device time per call
    try:
        graphs = []
        for fn in ("q", "d"):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):                        # captured on torch's side stream
                for x, q, y in zip(xs, qs, ys):
                    if fn == "q":
                        mx.quantize(x, "e4m3", "row", "ceil", layout="rowmajor", out=q)
                    else:
                        mx.dequantize(q, "rowmajor", out=y)
            graphs.append(g)
        gq, gd = (timed([g.replay], 4, stream) / len(xs) for g in graphs)
        out["mxfp8_rowwise_1024x1024"].update({"graph_quantize_us": round(gq * 1e3, 2),
                                             "graph_dequantize_us": round(gd * 1e3, 2),
                                             "graph_quantize_GBps": round(b1 / gq / 1e6, 1),
                                             "graph_dequantize_GBps": round(b1 / gd / 1e6, 1),
                                             "graph_frac_hbm": round(b1 / gq / 1e6 / hbm, 4),
                                             "graph_note": "64 calls on 64 rotating copies in one CUDA graph"})
        del graphs
    except RuntimeError as e:                              # capture refused: report, keep going
        out["mxfp8_rowwise_1024x1024"]["graph_error"] = str(e)[:200]
    del x1, xs, qs

    # dequantise the 4096 x 4096 weight (MXFP4 and NVFP4), tcgen05 scales, 8 rotating copies
    xw = to_dev(synth.weight_fp4(), dev)
    q4 = [mx.quantize(xw, "e2m1", "row", "floor", layout="tcgen05") for _ in range(NROT)]
    qn = [mx.quantize(xw, "nvfp4", "row", "ceil", layout="tcgen05") for _ in range(NROT)]
    ys = [torch.empty_like(xw) for _ in range(NROT)]
    t4 = timed([lambda q=q, y=y: mx.dequantize(q, "tcgen05", out=y) for q, y in zip(q4, ys)], 64, stream)
    tn = timed([lambda q=q, y=y: mx.dequantize(q, "tcgen05", out=y) for q, y in zip(qn, ys)], 64, stream)
    bd4 = R2 * C2 // 2 + R2 * C2 // 32 + R2 * C2 * 2
    bdn = R2 * C2 // 2 + R2 * C2 // 16 + 4 + R2 * C2 * 2
    out["dequantize_4096x4096"] = {"mxfp4_GBps": round(bd4 / t4 / 1e6, 1), "mxfp4_frac_hbm": round(bd4 / t4 / 1e6 / hbm, 4),
                                 "nvfp4_GBps": round(bdn / tn / 1e6, 1), "nvfp4_frac_hbm": round(bdn / tn / 1e6 / hbm, 4)}
    del xw, q4, qn, ys

    # C3: dual-orientation MXFP8, activations (E4M3) and gradients (E5M2), tcgen05 scales
    for name, gen, fmt in (("act_16384x4096_e4m3", synth.activations, "e4m3"),
                           ("grad_16384x14336_e5m2", synth.gradients, "e5m2")):
        xb = gen()
        R, C = xb.shape
        x3 = to_dev(xb, dev)
        del xb
        o3 = mx.quantize_dual(x3, fmt, "ceil", "tcgen05")
        t = timed([lambda: mx.quantize_dual(x3, fmt, "ceil", "tcgen05", out=o3)], 20, stream)
        nbytes = R * C * 2 + 2 * (R * C + R * C // 32)
        out[f"dual_{name}"] = {"ms": round(t, 4), "GBps": round(nbytes / t / 1e6, 1),
                                  "frac_hbm": round(nbytes / t / 1e6 / hbm, 4), "algorithmic_bytes": nbytes,
                                  "l2": "input larger than L2"}
        del x3, o3
        torch.cuda.empty_cache()

    # C4 / C5: block-scaled matmuls (operands quantised outside the timing)
    # (plus the MXFP6 x MXFP6 matmul, which runs on the same kind at the same rate)
    for name, (M, N, K), afmt, bfmt, bsig in (
            ("gemm_e4m3_8192", (8192, 8192, 8192), "e4m3", "e4m3", 1.0),
            ("gemm_e4m3_x_e2m1_8192x14336x4096", (8192, 14336, 4096), "e4m3", "e2m1", 0.02),
            ("gemm_mxfp6_e2m3_8192", (8192, 8192, 8192), "e2m3", "e2m3", 1.0)):
        a = mx.quantize(to_dev(synth.normal(M, K, seed=40), dev), afmt, "row", "ceil", layout="tcgen05")
        b = mx.quantize(to_dev(synth.normal(N, K, sigma=bsig, seed=41), dev), bfmt, "row",
                        "floor" if bfmt == "e2m1" else "ceil", layout="tcgen05")
        c = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        t = timed([lambda: mx.gemm(a, b, c)], 10, stream)
        tb = best_of(lambda: mx.gemm(a, b, c), 10, stream)
        tf, tfb = (2.0 * M * N * K / (x * 1e-3) / 1e12 for x in (t, tb))
        out[name] = {"ms": round(t, 4), "TFLOPS": round(tf, 1), "frac_mx_peak_measured": round(tf / mx_peak, 4),
                     "clocks_back_to_back": soak_clocks(lambda: mx.gemm(a, b, c)),
                     "best_of_10_ms": round(tb, 4), "best_of_10_TFLOPS": round(tfb, 1),
                     "frac_best_of_10_mx_peak_measured": round(tfb / mx_peak, 4),
                     "mx_peak_measured_TFLOPS": mx_peak, "frac_mx_nominal_4500": round(tf / MX_NOMINAL_TFLOPS, 4),
                     "peak_note": "bf16 burst (MEASURED_PEAKS, best of 10) x 2, the FP8/f8f6f4 to bf16 nominal "
                                  "ratio; ms / TFLOPS: mean of 10 back-to-back calls"}
        del a, b, c
        torch.cuda.empty_cache()

    # library comparator (not this library's path): cuBLASLt's MXFP8 block-scaled matmul via
    # torch._scaled_mm on the same 8192^3 E4M3 operands -- the E8M0 scales in the tcgen05
    # tiling are the layout it takes
    try:
        M = N = K = 8192
        a = mx.quantize(to_dev(synth.normal(M, K, seed=40), dev), "e4m3", "row", "ceil", layout="tcgen05")
        b = mx.quantize(to_dev(synth.normal(N, K, seed=41), dev), "e4m3", "row", "ceil", layout="tcgen05")
        af = a.elems.view(torch.float8_e4m3fn).view(M, K)
        bf = b.elems.view(torch.float8_e4m3fn).view(N, K)
        sa = a.scales.view(torch.float8_e8m0fnu)
        sb = b.scales.view(torch.float8_e8m0fnu)

        def lib():
            return torch._scaled_mm(af, bf.t(), scale_a=sa, scale_b=sb, out_dtype=torch.bfloat16)
        ref = lib()
        ours = mx.gemm(a, b)
        rel = ((ref.float() - ours.float()).abs().max() / ours.float().abs().max()).item()
        t = timed([lib], 10, stream)
        tb = best_of(lib, 10, stream)
        tf, tfb = (2.0 * M * N * K / (x * 1e-3) / 1e12 for x in (t, tb))
        out["cublaslt_mxfp8_8192_comparator"] = {
            "ms": round(t, 4), "TFLOPS": round(tf, 1), "best_of_10_TFLOPS": round(tfb, 1),
            "frac_mx_peak_measured": round(tf / mx_peak, 4), "max_abs_diff_vs_ours_rel_to_max": rel,
            "clocks_back_to_back": soak_clocks(lib),
            "note": "torch._scaled_mm (cuBLASLt) on the same operands: a comparator, not this library's path"}
        del a, b, af, bf, sa, sb, ref, ours
    except Exception as e:                                   # comparator unavailable: say why
        out["cublaslt_mxfp8_8192_comparator"] = {"unavailable": str(e)[:200]}
    torch.cuda.empty_cache()

    # FP4 x FP4 block-scaled matmuls (kind::mxf4 and kind::mxf4nvf4), 8192^3,
    # against the dense FP4 rate (2 x the FP8 rate; 9 PFLOP/s nominal)
    fp4_peak = 2.0 * mx_peak
    for name, fmt in (("gemm_mxfp4_x_mxfp4_8192", "e2m1"), ("gemm_nvfp4_x_nvfp4_8192", "nvfp4")):
        M = N = K = 8192
        a = mx.quantize(to_dev(synth.normal(M, K, seed=60), dev), fmt, "row", "floor", layout="tcgen05")
        b = mx.quantize(to_dev(synth.normal(N, K, sigma=0.02, seed=61), dev), fmt, "row", "floor", layout="tcgen05")
        c = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        t = timed([lambda: mx.gemm(a, b, c)], 10, stream)
        tb = best_of(lambda: mx.gemm(a, b, c), 10, stream)
        tf, tfb = (2.0 * M * N * K / (x * 1e-3) / 1e12 for x in (t, tb))
        out[name] = {"ms": round(t, 4), "TFLOPS": round(tf, 1), "frac_fp4_peak_measured": round(tf / fp4_peak, 4),
                     "clocks_back_to_back": soak_clocks(lambda: mx.gemm(a, b, c)),
                     "best_of_10_ms": round(tb, 4), "best_of_10_TFLOPS": round(tfb, 1),
                     "frac_best_of_10_fp4_peak_measured": round(tfb / fp4_peak, 4),
                     "fp4_peak_measured_TFLOPS": fp4_peak, "frac_fp4_nominal_9000": round(tf / (2 * MX_NOMINAL_TFLOPS), 4),
                     "peak_note": "bf16 burst (MEASURED_PEAKS, best of 10) x 4, the FP4 to bf16 nominal ratio; "
                                  "ms / TFLOPS: mean of 10 back-to-back calls"}
        del a, b, c
        torch.cuda.empty_cache()

    # MXFP6 / MXINT8 row-wise quantisation of the 16384 x 4096 activations
    # (16384 x 4096 bf16; FP6 codes packed 6 bits each, INT8 one byte), against the HBM roofline
    x3 = to_dev(synth.activations(), dev)
    R, C = x3.shape
    for name, fmt in (("quant_mxfp6_e2m3_16384x4096", "e2m3"), ("quant_mxint8_16384x4096", "int8")):
        q = mx.quantize(x3, fmt, "row", "ceil", layout="tcgen05")
        t = timed([lambda q=q: mx.quantize(x3, fmt, "row", "ceil", layout="tcgen05", out=q)], 20, stream)
        nb = R * C * 2 + mx.elem_bytes(R, C, fmt) + R * C // 32
        out[name] = {"ms": round(t, 4), "GBps": round(nb / t / 1e6, 1), "frac_hbm": round(nb / t / 1e6 / hbm, 4),
                     "algorithmic_bytes": nb}
        del q
    del x3

    # nested blocks -- the 14336 x 4096 MXFP4 weight re-expressed as
    # FP8 E4M3 with 128 x 128 block scales
    from microscaling_precision_number_b200 import _lib as L
    xw = to_dev(synth.normal(14336, 4096, sigma=0.02, seed=51), dev)
    qw = mx.quantize(xw, "e2m1", "row", "floor", layout="rowmajor")
    R, C = xw.shape
    del xw
    # four rotating (codes, output) sets, 4 x 88 MiB > L2
    sets = [(qw.elems if i == 0 else qw.elems.clone(), qw.scales if i == 0 else qw.scales.clone(),
             torch.empty(R * C, dtype=torch.uint8, device=dev)) for i in range(4)]
    bsc = torch.empty((R // 128) * (C // 128), dtype=torch.float32, device=dev)
    bok = torch.empty((R // 128) * (C // 128), dtype=torch.uint8, device=dev)

    def nested(e, sc, o8):
        L.check(L.lib.mx_mxfp4_to_fp8_blocks(e.data_ptr(), sc.data_ptr(), R, C, o8.data_ptr(),
                                             bsc.data_ptr(), bok.data_ptr(), stream.cuda_stream),
                "mx_mxfp4_to_fp8_blocks")
    t = timed([lambda st=st: nested(*st) for st in sets], 20, stream)
    nb = R * C // 2 + R * C // 32 + R * C + 5 * (R // 128) * (C // 128)
    out["nested_mxfp4_to_fp8_14336x4096"] = {"ms": round(t, 4), "GBps": round(nb / t / 1e6, 1),
                                                   "frac_hbm": round(nb / t / 1e6 / hbm, 4), "algorithmic_bytes": nb,
                                                   "blocks_exact": int(bok.sum().item()), "blocks": int(bok.numel()),
                                                   "l2": "four rotating sets, 352 MiB > L2"}
    del qw, sets, bsc, bok
    torch.cuda.empty_cache()

    # training-side quantiser on the 16384 x 14336 gradient shape (bf16):
    # 16 x 16 random Hadamard transform + stochastic rounding (one random byte per element),
    # NVFP4 (two passes; the maximum pass's re-read is not counted) and MXFP4; tcgen05 scales
    R, C = 16384, 14336
    xg = to_dev(synth.normal(R, C, sigma=1e-3, seed=70), dev)
    rnd = torch.from_numpy(np.random.default_rng(71).integers(0, 256, R * C, dtype=np.uint8)).to(dev)
    for name, f, B in (("train_nvfp4_rht_sr_16384x14336", L.MX_FMT_NVFP4, 16),
                       ("train_mxfp4_rht_sr_16384x14336", L.MX_FMT_E2M1, 32)):
        el = torch.empty(R * C // 2, dtype=torch.uint8, device=dev)
        sc = torch.empty(mx.scale_bytes(R, C // B, "tcgen05"), dtype=torch.uint8, device=dev)
        gs = torch.empty(1, dtype=torch.float32, device=dev) if f == L.MX_FMT_NVFP4 else None

        def train(f=f, el=el, sc=sc, gs=gs):
            L.check(L.lib.mx_quantize_train(xg.data_ptr(), R, C, f, 0, 1, 0xB5C3, rnd.data_ptr(), el.data_ptr(),
                                            sc.data_ptr(), L.MX_LAYOUT_TCGEN05, None,
                                            gs.data_ptr() if gs is not None else None, stream.cuda_stream),
                    "mx_quantize_train")
        t = timed([train], 10, stream)
        nb = R * C * 2 + R * C + R * C // 2 + sc.numel() + (4 if gs is not None else 0)
        out[name] = {"ms": round(t, 4), "GBps": round(nb / t / 1e6, 1), "frac_hbm": round(nb / t / 1e6 / hbm, 4),
                     "algorithmic_bytes": nb, "note": "input, random bytes, codes, scales; input larger than L2"}
        del el, sc, gs
    del xg, rnd
    torch.cuda.empty_cache()

    # NVFP4 with 16 x 16 weight blocks on the 4096 x 4096 weight
    R = C = 4096
    xw = to_dev(synth.weight_fp4(), dev)
    el = torch.empty(R * C // 2, dtype=torch.uint8, device=dev)
    sc = torch.empty(mx.scale_bytes(R, C // 16, "tcgen05"), dtype=torch.uint8, device=dev)
    gs = torch.empty(1, dtype=torch.float32, device=dev)

    xs = [xw] + [xw.clone() for _ in range(5)]           # six rotating inputs (192 MiB > L2)

    def nvfp4_2d(x):
        L.check(L.lib.mx_quantize_nvfp4_2d(x.data_ptr(), R, C, el.data_ptr(), sc.data_ptr(), L.MX_LAYOUT_TCGEN05,
                                           None, gs.data_ptr(), stream.cuda_stream), "mx_quantize_nvfp4_2d")
    t = timed([lambda x=x: nvfp4_2d(x) for x in xs], 24, stream)
    nb = R * C * 2 + R * C // 2 + sc.numel() + 4
    out["quant_nvfp4_2d_4096x4096"] = {"ms": round(t, 4), "GBps": round(nb / t / 1e6, 1),
                                              "frac_hbm": round(nb / t / 1e6 / hbm, 4), "algorithmic_bytes": nb,
                                              "l2": "six rotating inputs, 192 MiB > L2"}
    del xw, xs, el, sc, gs
    torch.cuda.empty_cache()
    return out


# ----------------------------------------------------------------------------- CPU oracle
def cpu_baseline(x_bits, target_s=12.0):
    """The oracle as it stands, single-threaded, on a bounded row sample of the workload."""
    import oracle
    oracle.lib()
    rows = 64
    t0 = time.perf_counter()
    done_rows = 0
    while True:
        xs = np.ascontiguousarray(x_bits[done_rows % R2: done_rows % R2 + rows])
        e4, s4 = oracle.quantize_mx(xs, oracle.E2M1, oracle.ROW, oracle.FLOOR)
        oracle.to_tcgen05_layout(s4)
        en, sn, g = oracle.quantize_nvfp4(xs)
        oracle.to_tcgen05_layout(sn)
        done_rows += rows
        if time.perf_counter() - t0 > target_s or done_rows >= R2:
            break
    dt = time.perf_counter() - t0
    bytes_done = STEP_BYTES * done_rows / R2
    return {"value": round(bytes_done / dt / 1e9, 5), "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"{done_rows} of {R2} rows of the 4096x4096 weight (MXFP4 + NVFP4, both layouts), "
                      f"{dt:.1f} s single-threaded", "seconds": round(dt, 2)}


def run_reference(args, rank, world):
    """The oracle as the reference arm: rank 0 only, bounded sample per step."""
    if rank != 0:
        return
    x_bits = synth.weight_fp4(seed=0)
    per_step = max(1.0, args.cpu_seconds / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        cpu_baseline(x_bits, target_s=per_step)
    vals, secs = [], []
    for _ in range(args.steps):
        r = cpu_baseline(x_bits, target_s=per_step)
        vals.append(r["value"])
        secs.append(r["seconds"])
        sample = r["sample"]
    v = statistics.mean(vals)
    line = {"impl": "reference", "metric": METRIC, "value": round(v, 5), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * statistics.mean(secs), 1),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic (numpy default_rng, seed 0)",
            "config": {"workload": "weight_4096x4096_mxfp4_floor_and_nvfp4_both_scale_layouts", "shape": [R2, C2]},
            "cpu_baseline": {"kind": "oracle", "cores": 1, "sample": sample, "value": round(v, 5)},
            "e2e": {"value": round(v, 5), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- one case
def run_case(name, iters, dev):
    """Run one workload's hot call `iters` times and nothing else (for profiler captures:
    the launch list then holds only this case's kernels).  Prints the mean device time per
    call, which under a profiler is not a benchmark number."""
    import microscaling_precision_number_b200 as mx
    stream = torch.cuda.current_stream()
    if name == "weight4096":
        st = WeightQuantStep(mx, to_dev(synth.weight_fp4(), dev))
        fns = [lambda: (st.mxfp4(stream.cuda_stream), st.nvfp4(stream.cuda_stream))]
    elif name == "mx8_1024":
        x = to_dev(synth.mx8_rowwise(), dev)
        q = mx.quantize(x, "e4m3", "row", "ceil", layout="rowmajor")
        y = torch.empty_like(x)
        fns = [lambda: (mx.quantize(x, "e4m3", "row", "ceil", layout="rowmajor", out=q),
                        mx.dequantize(q, "rowmajor", out=y))]
    elif name in ("dual_act", "dual_grad"):
        gen, fmt = (synth.activations, "e4m3") if name == "dual_act" else (synth.gradients, "e5m2")
        x = to_dev(gen(), dev)
        o = mx.quantize_dual(x, fmt, "ceil", "tcgen05")
        fns = [lambda: mx.quantize_dual(x, fmt, "ceil", "tcgen05", out=o)]
    elif name == "dequant4096":
        xw = to_dev(synth.weight_fp4(), dev)
        q4 = mx.quantize(xw, "e2m1", "row", "floor", layout="tcgen05")
        qn = mx.quantize(xw, "nvfp4", "row", "ceil", layout="tcgen05")
        y = torch.empty_like(xw)
        fns = [lambda: (mx.dequantize(q4, "tcgen05", out=y), mx.dequantize(qn, "tcgen05", out=y))]
    elif name in ("gemm_mxfp4_8192", "gemm_nvfp4_8192"):
        fmt = "e2m1" if name == "gemm_mxfp4_8192" else "nvfp4"
        a = mx.quantize(to_dev(synth.normal(8192, 8192, seed=60), dev), fmt, "row", "floor", layout="tcgen05")
        b = mx.quantize(to_dev(synth.normal(8192, 8192, sigma=0.02, seed=61), dev), fmt, "row", "floor",
                        layout="tcgen05")
        c = torch.empty((8192, 8192), dtype=torch.bfloat16, device=dev)
        fns = [lambda: mx.gemm(a, b, c)]
    elif name in ("gemm8192", "gemm_w4a8"):
        (M, N, K), bfmt, bsig = (((8192, 8192, 8192), "e4m3", 1.0) if name == "gemm8192"
                                 else ((8192, 14336, 4096), "e2m1", 0.02))
        a = mx.quantize(to_dev(synth.normal(M, K, seed=40), dev), "e4m3", "row", "ceil", layout="tcgen05")
        b = mx.quantize(to_dev(synth.normal(N, K, sigma=bsig, seed=41), dev), bfmt, "row",
                        "floor" if bfmt == "e2m1" else "ceil", layout="tcgen05")
        c = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        fns = [lambda: mx.gemm(a, b, c)]
    elif name == "gemm_cmp":
        # the 8192^3 E4M3 operands through this library's matmul and through cuBLASLt's MXFP8
        # matmul (torch._scaled_mm), one call each per round, for side-by-side counters
        M = N = K = 8192
        a = mx.quantize(to_dev(synth.normal(M, K, seed=40), dev), "e4m3", "row", "ceil", layout="tcgen05")
        b = mx.quantize(to_dev(synth.normal(N, K, seed=41), dev), "e4m3", "row", "ceil", layout="tcgen05")
        c = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        af, bf = a.elems.view(torch.float8_e4m3fn).view(M, K), b.elems.view(torch.float8_e4m3fn).view(N, K)
        sa, sb = a.scales.view(torch.float8_e8m0fnu), b.scales.view(torch.float8_e8m0fnu)
        fns = [lambda: (mx.gemm(a, b, c),
                        torch._scaled_mm(af, bf.t(), scale_a=sa, scale_b=sb, out_dtype=torch.bfloat16))]
    elif name == "extended":
        # one call of each extended kernel: training quantiser (NVFP4 and MXFP4, RHT + SR) on an
        # 8192 x 14336 gradient, nested conversion, MXFP6 matmul, 2-D NVFP4 weight blocks
        from microscaling_precision_number_b200 import _lib as L
        xg = to_dev(synth.normal(8192, 14336, sigma=1e-3, seed=70), dev)
        rnd = torch.from_numpy(np.random.default_rng(71).integers(0, 256, xg.numel(), dtype=np.uint8)).to(dev)
        xw = to_dev(synth.normal(14336, 4096, sigma=0.02, seed=51), dev)
        qw = mx.quantize(xw, "e2m1", "row", "floor", layout="rowmajor")
        o8 = torch.empty(xw.numel(), dtype=torch.uint8, device=dev)
        bsc = torch.empty(xw.numel() // 16384, dtype=torch.float32, device=dev)
        bok = torch.empty(xw.numel() // 16384, dtype=torch.uint8, device=dev)
        a6 = mx.quantize(to_dev(synth.normal(8192, 8192, seed=40), dev), "e2m3", "row", "ceil", layout="tcgen05")
        b6 = mx.quantize(to_dev(synth.normal(8192, 8192, seed=41), dev), "e2m3", "row", "ceil", layout="tcgen05")
        c6 = torch.empty((8192, 8192), dtype=torch.bfloat16, device=dev)
        x2 = to_dev(synth.weight_fp4(), dev)
        s = stream.cuda_stream

        def all_rows():
            mx.quantize_train(xg, "nvfp4", "ceil", rht_signs=0xB5C3, sr_random=rnd, layout="tcgen05", stream=stream)
            mx.quantize_train(xg, "e2m1", "floor", rht_signs=0xB5C3, sr_random=rnd, layout="tcgen05", stream=stream)
            L.check(L.lib.mx_mxfp4_to_fp8_blocks(qw.elems.data_ptr(), qw.scales.data_ptr(), 14336, 4096,
                                                 o8.data_ptr(), bsc.data_ptr(), bok.data_ptr(), s), "nested")
            mx.gemm(a6, b6, c6, stream=stream)
            mx.quantize_nvfp4_2d(x2, layout="tcgen05", stream=stream)
        fns = [all_rows]
    else:
        raise SystemExit(f"unknown case {name}")
    t = timed(fns, iters, stream)
    assert mx.watchdog_status() == 0
    print(f"{name}: {iters} calls, {t * 1e3:.1f} us per call", flush=True)


CASES = ["weight4096", "mx8_1024", "dual_act", "dual_grad", "dequant4096", "gemm8192", "gemm_w4a8",
         "gemm_mxfp4_8192", "gemm_nvfp4_8192", "gemm_cmp", "extended"]


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-breakdown", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--case", choices=CASES, help="run one workload's hot call only (profiling)")
    ap.add_argument("--iters", type=int, default=3, help="calls for --case (one warm-up call before)")
    args = ap.parse_args()
    if args.case:
        dev = torch.device("cuda", 0)
        torch.cuda.set_device(dev)
        run_case(args.case, args.iters, dev)
        return
    if args.warmup < 3:
        args.warmup = 3
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=dev)
    try:
        run_ours(args, rank, world, dev)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
