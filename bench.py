#!/usr/bin/env python
"""Benchmark of the MX hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--no-breakdown]

One step = dual-orientation MXFP8 quantisation (row-wise and column-wise from one read,
E8M0 scales in the tcgen05 tiling, no-clip scale rule) of the training workload's two
tensors: the 16384 x 4096 bf16 activations (N(0,1) times a per-channel 2^v, v ~ U[-4, 4])
in E4M3, and the 16384 x 14336 bf16 gradients (N(0, 1e-3), 5% exact zeros) in E5M2.
value = algorithmic bytes of the step (read the input once, write both codes and scales
once: 1,226,833,920 B) / step time (GB/s).  The inputs (604 MB) exceed L2, so consecutive
steps read HBM without a flush.  K steps are timed back to back in one CUDA-event pair.
Every other row of the hot path (the 1024^2 MXFP8 quantise + dequantise, the 4096^2 MXFP4
+ NVFP4 weight quantisation, dequantisation, the block-scaled matmuls and the extension
rows) is measured in "breakdown", each against its own roofline.

Multi-GPU (torchrun): every rank quantises its own tensors (independent units, no
data-path collective); value = all ranks' bytes / the slowest rank's time.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import hashlib
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

# the training workload: dual-orientation MXFP8 of activations (E4M3) and gradients (E5M2)
ACT = (16384, 4096)
GRAD = (16384, 14336)


def dual_bytes(R, C):
    """Read the bf16 input once; write row-wise and column-wise FP8 codes and E8M0 scales."""
    return R * C * 2 + 2 * (R * C + R * C // 32)


BYTES_ACT = dual_bytes(*ACT)           # 272,629,760
BYTES_GRAD = dual_bytes(*GRAD)         # 954,204,160
STEP_BYTES = BYTES_ACT + BYTES_GRAD    # 1,226,833,920
WORKLOAD = "dual_mxfp8_act_16384x4096_e4m3_and_grad_16384x14336_e5m2_tcgen05_scales"

# DRAM bytes (read + write) of one quant_dual_kernel launch on the gradients, from an ncu
# capture of the benchmark's own back-to-back sequence (no cache control, no clock
# control), and the SHA-256 of the kernel source that capture ran: when dual.cu has
# changed since, the traffic is reported as null.
NCU_TRAFFIC_GRAD = 955400107      # mean of 3 launches: read ~469.88 MB + write ~485.52 MB
NCU_TRAFFIC_SRC_SHA = "d3e0aad265bfe978daae80f6618d0c20056e6cd34940c0736dbd8f49b43c169a"
DUAL_SRC = os.path.join(ROOT, "microscaling_precision_number_b200", "csrc", "dual.cu")

# the 4096 x 4096 weight: MXFP4 (floor) + NVFP4, both scale layouts (a breakdown row)
R2 = C2 = 4096
BYTES_MXFP4 = R2 * C2 * 2 + R2 * C2 // 2 + 2 * (R2 * C2 // 32)            # 42,991,616
BYTES_NVFP4 = R2 * C2 * 2 + R2 * C2 // 2 + 2 * (R2 * C2 // 16) + 4         # 44,040,196
NROT = 8                 # rotating copies of the 32 MiB weight (8 x 32 MiB > 2 x L2)


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


def file_sha(path):
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()


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
class DualStep:
    """Dual-orientation MXFP8 quantisation of the activations (E4M3) and the gradients
    (E5M2) through the C ABI, tcgen05-tiled scales, no-clip rule."""

    def __init__(self, mx, x_act, x_grad):
        from microscaling_precision_number_b200 import _lib as L
        self.L = L
        self.parts = []
        for x, fmt in ((x_act, L.MX_FMT_E4M3), (x_grad, L.MX_FMT_E5M2)):
            R, C = x.shape
            dev = x.device
            o = dict(x=x, R=R, C=C, fmt=fmt,
                     re=torch.empty(R * C, dtype=torch.uint8, device=dev),
                     rs=torch.empty(mx.scale_bytes(R, C // 32, "tcgen05"), dtype=torch.uint8, device=dev),
                     ce=torch.empty(R * C, dtype=torch.uint8, device=dev),
                     cs=torch.empty(mx.scale_bytes(C, R // 32, "tcgen05"), dtype=torch.uint8, device=dev))
            self.parts.append(o)
        self.launches_per_step = 2

    def run_part(self, i, stream):
        L, o = self.L, self.parts[i]
        L.check(L.lib.mx_quantize_dual(o["x"].data_ptr(), o["R"], o["C"], o["fmt"], L.MX_SCALE_CEIL_RECIPE,
                                       o["re"].data_ptr(), o["rs"].data_ptr(), o["ce"].data_ptr(),
                                       o["cs"].data_ptr(), L.MX_LAYOUT_TCGEN05, None, None, stream),
                "mx_quantize_dual")

    def run(self, stream):
        self.run_part(0, stream)
        self.run_part(1, stream)

    def inputs(self):
        return [o["x"] for o in self.parts]

    def outputs(self):
        return [o[k] for o in self.parts for k in ("re", "rs", "ce", "cs")]


def run_ours(args, rank, world, dev):
    import microscaling_precision_number_b200 as mx

    pk = peaks()
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    sptr = stream.cuda_stream
    a_bits = synth.activations(seed=rank)
    g_bits = synth.gradients(seed=rank + 1)
    step = DualStep(mx, to_dev(a_bits, dev), to_dev(g_bits, dev))

    def run_steps(n):
        for _ in range(n):
            step.run(sptr)

    run_steps(args.warmup)
    torch.cuda.synchronize()

    with ClockSampler(torch.cuda.current_device()) as clk:
        # soak: keep the GPU busy with the same steps for ~0.5 s so that the clock samples
        # below see it under load, then the timed region proper
        t0 = time.perf_counter()
        while time.perf_counter() - t0 < 0.5:
            run_steps(10)
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

    # the dominant kernel's launch duration: the gradient dual call, back to back on the
    # launching stream (inputs larger than L2)
    ncall = max(args.steps, 20)
    per = {}
    for i, name in ((0, "act"), (1, "grad")):
        step.run_part(i, sptr)
        a, b = event_pair()
        a.record(stream)
        for _ in range(ncall):
            step.run_part(i, sptr)
        b.record(stream)
        torch.cuda.synchronize()
        per[name] = a.elapsed_time(b) / ncall
    achieved = BYTES_GRAD / (per["grad"] * 1e-3) / 1e9
    traffic = NCU_TRAFFIC_GRAD if (NCU_TRAFFIC_SRC_SHA is not None and file_sha(DUAL_SRC) == NCU_TRAFFIC_SRC_SHA) \
        else None
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": round(achieved / pk["hbm_gbs"], 4), "traffic": traffic,
                "peak_source": pk["source"] + " copy bandwidth (MEASURED_PEAKS hbm_gbs), burst",
                "kernel": "quant_dual_kernel<E5M2, no-clip, tcgen05 scales> (mx_quantize_dual on the gradients)",
                "algorithmic_bytes_per_launch": BYTES_GRAD, "ms_per_launch": round(per["grad"], 5),
                "launches_timed": ncall,
                "calls": {"act_ms": round(per["act"], 5), "act_GBps": round(BYTES_ACT / per["act"] / 1e6, 1),
                          "act_frac": round(BYTES_ACT / per["act"] / 1e6 / pk["hbm_gbs"], 4),
                          "grad_ms": round(per["grad"], 5), "grad_GBps": round(BYTES_GRAD / per["grad"] / 1e6, 1)},
                "frac_of_nominal_8TBps": round(achieved / HBM_NOMINAL_GBS, 4)}

    e2e = run_e2e(args, step, world, dev, stream, sptr, a_bits, g_bits)

    breakdown = None
    if not args.no_breakdown and rank == 0:
        del step
        torch.cuda.empty_cache()
        breakdown = run_breakdown(mx, dev, pk, cpu=(world == 1 and not args.no_cpu_baseline))

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(a_bits, g_bits, target_s=args.cpu_seconds)

    if rank == 0:
        line = {"metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
                "data": "synthetic (numpy default_rng; activations seed = rank, gradients seed = rank + 1)",
                "config": step_config(world),
                "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
                "gpu_launches": step_launches(args.steps), "clocks": clk.summary()}
        if breakdown is not None:
            line["breakdown"] = breakdown
        print(json.dumps(line), flush=True)


def step_launches(steps):
    return 2 * steps                   # one quant_dual_kernel launch per tensor


def run_e2e(args, step, world, dev, stream, sptr, a_bits, g_bits):
    """The same step through the C ABI with host buffers: every step uploads both bf16
    inputs from pinned host memory and downloads all codes and scales.  Pipelined as a
    stream of training steps would run: the upload of step k, the quantisation of step k-1
    and the download of step k-2 overlap on three streams, with two device buffer sets
    ordered by events; the serial form (upload, quantise, download on one stream) is
    reported beside it."""
    import microscaling_precision_number_b200 as mx
    sets = [step, DualStep(mx, torch.empty_like(step.parts[0]["x"]), torch.empty_like(step.parts[1]["x"]))]
    x_host = [torch.from_numpy(b.view(np.int16)).view(torch.bfloat16).pin_memory() for b in (a_bits, g_bits)]
    outs_host = [[torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for o in st.outputs()] for st in sets]
    h2d = sum(x.numel() * 2 for x in x_host)
    d2h = sum(o.numel() * o.element_size() for o in outs_host[0])
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    ev_up, ev_comp, ev_down = ([torch.cuda.Event() for _ in sets] for _ in range(3))

    def pipelined(n):
        for k in range(n):
            b = k % 2
            st = sets[b]
            up.wait_event(ev_comp[b])                  # the buffer's previous step has read it
            with torch.cuda.stream(up):
                for d, h in zip(st.inputs(), x_host):
                    d.copy_(h, non_blocking=True)
            ev_up[b].record(up)
            stream.wait_event(ev_up[b])
            stream.wait_event(ev_down[b])              # its previous outputs have been copied out
            st.run(sptr)
            ev_comp[b].record(stream)
            down.wait_event(ev_comp[b])
            with torch.cuda.stream(down):
                for h, d in zip(outs_host[b], st.outputs()):
                    h.copy_(d, non_blocking=True)
            ev_down[b].record(down)

    def serial(n):
        st = sets[0]
        for _ in range(n):
            for d, h in zip(st.inputs(), x_host):
                d.copy_(h, non_blocking=True)
            st.run(sptr)
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
    out = {"value": round(job_throughput_gbs(STEP_BYTES, args.steps, world, e2e_ms), 2), "unit": "GB/s",
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
           "ms_per_step": round(e2e_ms / args.steps, 4),
           "form": "pipelined: upload / quantise / download of consecutive steps overlap on three streams",
           "serial": {"value": round(job_throughput_gbs(STEP_BYTES, args.steps, world, ser_ms), 2),
                      "ms_per_step": round(ser_ms / args.steps, 4)},
           "note": "host<->device copies over PCIe bound this number"}
    del sets[1], outs_host, x_host
    return out


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

    def both(self, stream):
        """Both encodings in one call (the MX pass supplies the NVFP4 tensor maximum)."""
        L = self.L
        L.check(L.lib.mx_quantize_mx_nvfp4(self.x.data_ptr(), self.R, self.C, L.MX_FMT_E2M1, L.MX_SCALE_FLOOR_OCP,
                                           self.e4.data_ptr(), self.s4.data_ptr(), 3, self.s4t.data_ptr(),
                                           self.en.data_ptr(), self.sn.data_ptr(), 3, self.snt.data_ptr(),
                                           self.g.data_ptr(), stream), "mx_quantize_mx_nvfp4")


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


def run_breakdown(mx, dev, pk, cpu=False):
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

    # dequantise the 4096 x 4096 weight (MXFP4 and NVFP4), tcgen05 scales, 8 rotating copies.
    # A call takes ~9-10 us on the device, about what the Python wrapper's per-call work takes
    # on the host, so the timed loop calls the C ABI directly (as the weight-step rows do);
    # the wrapper's per-call time is reported beside it.
    from microscaling_precision_number_b200 import _lib as L
    xw = to_dev(synth.weight_fp4(), dev)
    q4 = [mx.quantize(xw, "e2m1", "row", "floor", layout="tcgen05") for _ in range(NROT)]
    qn = [mx.quantize(xw, "nvfp4", "row", "ceil", layout="tcgen05") for _ in range(NROT)]
    ys = [torch.empty_like(xw) for _ in range(NROT)]

    def dq(q, y):
        gs = q.global_scale.data_ptr() if q.global_scale is not None else None
        L.check(L.lib.mx_dequantize(q.elems.data_ptr(), q.scales.data_ptr(), gs, q.rows, q.cols, q.fmt,
                                    L.MX_LAYOUT_TCGEN05, y.data_ptr(), stream.cuda_stream), "mx_dequantize")
    t4 = timed([lambda q=q, y=y: dq(q, y) for q, y in zip(q4, ys)], 64, stream)
    tn = timed([lambda q=q, y=y: dq(q, y) for q, y in zip(qn, ys)], 64, stream)
    t4p = timed([lambda q=q, y=y: mx.dequantize(q, "tcgen05", out=y, stream=stream) for q, y in zip(q4, ys)], 64, stream)
    bd4 = R2 * C2 // 2 + R2 * C2 // 32 + R2 * C2 * 2
    bdn = R2 * C2 // 2 + R2 * C2 // 16 + 4 + R2 * C2 * 2
    out["dequantize_4096x4096"] = {"mxfp4_us": round(t4 * 1e3, 2), "mxfp4_GBps": round(bd4 / t4 / 1e6, 1),
                                   "mxfp4_frac_hbm": round(bd4 / t4 / 1e6 / hbm, 4),
                                   "nvfp4_us": round(tn * 1e3, 2), "nvfp4_GBps": round(bdn / tn / 1e6, 1),
                                   "nvfp4_frac_hbm": round(bdn / tn / 1e6 / hbm, 4),
                                   "mxfp4_python_wrapper_us_per_call": round(t4p * 1e3, 2),
                                   "note": "C ABI calls back to back; the Python wrapper adds host time per call"}
    del xw, q4, qn, ys

    # dequantise the 16384 x 4096 activations (MXFP8 E4M3, MXFP4, NVFP4; tcgen05 scales):
    # codes + scales in, 128 MiB of bf16 out, each call larger than L2
    xa = to_dev(synth.activations(), dev)
    ya = torch.empty_like(xa)
    RA, CA = xa.shape
    da = {}
    for fmt, rnd, bpe, blk in (("e4m3", "ceil", 1.0, 32), ("e2m1", "floor", 0.5, 32), ("nvfp4", "ceil", 0.5, 16)):
        q = mx.quantize(xa, fmt, "row", rnd, layout="tcgen05")
        t = timed([lambda q=q: mx.dequantize(q, "tcgen05", out=ya)], 20, stream)
        nb = int(RA * CA * bpe) + RA * CA // blk + (4 if fmt == "nvfp4" else 0) + RA * CA * 2
        da[fmt + "_us"] = round(t * 1e3, 2)
        da[fmt + "_GBps"] = round(nb / t / 1e6, 1)
        da[fmt + "_frac_hbm"] = round(nb / t / 1e6 / hbm, 4)
        del q
    out["dequantize_16384x4096"] = da
    del xa, ya

    # the 4096 x 4096 weight: MXFP4 (floor) and NVFP4, both scale layouts, each call on
    # eight rotating copies (256 MiB > L2); one step = both calls
    xw0 = to_dev(synth.weight_fp4(), dev)
    wsteps = [WeightQuantStep(mx, xw0.clone()) for _ in range(NROT)]
    sptr = stream.cuda_stream
    t4 = timed([lambda s=s: s.mxfp4(sptr) for s in wsteps], 64, stream)
    tn = timed([lambda s=s: s.nvfp4(sptr) for s in wsteps], 64, stream)
    tb = timed([lambda s=s: (s.mxfp4(sptr), s.nvfp4(sptr)) for s in wsteps], 64, stream)
    tf = timed([lambda s=s: s.both(sptr) for s in wsteps], 64, stream)
    out["weight_4096x4096_mxfp4_floor_and_nvfp4_both_layouts"] = {
        "step_us": round(tb * 1e3, 2), "step_GBps": round((BYTES_MXFP4 + BYTES_NVFP4) / tb / 1e6, 1),
        "step_frac_hbm": round((BYTES_MXFP4 + BYTES_NVFP4) / tb / 1e6 / hbm, 4),
        "one_call_us": round(tf * 1e3, 2), "one_call_GBps": round((BYTES_MXFP4 + BYTES_NVFP4) / tf / 1e6, 1),
        "one_call_frac_hbm": round((BYTES_MXFP4 + BYTES_NVFP4) / tf / 1e6 / hbm, 4),
        "one_call_note": "mx_quantize_mx_nvfp4: both encodings, the MX pass supplies the NVFP4 tensor maximum",
        "mxfp4_us": round(t4 * 1e3, 2), "mxfp4_GBps": round(BYTES_MXFP4 / t4 / 1e6, 1),
        "mxfp4_frac_hbm": round(BYTES_MXFP4 / t4 / 1e6 / hbm, 4),
        "nvfp4_us": round(tn * 1e3, 2), "nvfp4_GBps": round(BYTES_NVFP4 / tn / 1e6, 1),
        "nvfp4_frac_hbm": round(BYTES_NVFP4 / tn / 1e6 / hbm, 4),
        "algorithmic_bytes": {"mxfp4": BYTES_MXFP4, "nvfp4": BYTES_NVFP4},
        "l2": f"{NROT} rotating copies of the weight ({NROT * R2 * C2 * 2 >> 20} MiB)"}
    del wsteps, xw0
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
        if cpu and name != "gemm_mxfp6_e2m3_8192":
            cpu_gemm = gemm_cpu_baseline((M, N, K), afmt, bfmt, bsig)
        else:
            cpu_gemm = None
        out[name] = {"ms": round(t, 4), "TFLOPS": round(tf, 1), "frac_mx_peak_measured": round(tf / mx_peak, 4),
                     "cpu_baseline": cpu_gemm,
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
    # row-wise MXFP8 (E4M3) and column-wise-only MXFP8 of the same activations (the
    # transposed output alone: mx_quantize with axis = COL), tcgen05 scales
    for name, axis in (("quant_mxfp8_rowwise_16384x4096", "row"), ("quant_mxfp8_colwise_16384x4096", "col")):
        q = mx.quantize(x3, "e4m3", axis, "ceil", layout="tcgen05")
        t = timed([lambda q=q, axis=axis: mx.quantize(x3, "e4m3", axis, "ceil", layout="tcgen05", out=q)], 20, stream)
        nb = R * C * 2 + R * C + R * C // 32
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
def _workers():
    return max(1, min(64, os.cpu_count() or 1))


def cpu_baseline(a_bits, g_bits, target_s=12.0, band=64):
    """The oracle as it stands on a bounded sample of the workload: bands of `band`
    consecutive rows of both tensors, each band quantised row-wise and column-wise by the
    oracle with tcgen05-tiled scales; bands run on all host cores (one oracle call per
    thread).  value = the workload's bytes for the rows done / wall time."""
    import oracle
    oracle.lib()
    R = ACT[0]
    bands = list(range(0, R, band))
    workers = _workers()

    def one(r0):
        for x, fmt in ((a_bits, oracle.E4M3), (g_bits, oracle.E5M2)):
            xs = np.ascontiguousarray(x[r0:r0 + band])
            _, s = oracle.quantize_mx(xs, fmt, oracle.ROW, oracle.CEIL)
            oracle.to_tcgen05_layout(s)
            _, s = oracle.quantize_mx(xs, fmt, oracle.COL, oracle.CEIL)
            oracle.to_tcgen05_layout(s)
        return band

    t0 = time.perf_counter()
    done = 0
    with cf.ThreadPoolExecutor(workers) as ex:
        i = 0
        while i < len(bands) and time.perf_counter() - t0 < target_s:
            chunk = bands[i:i + workers]
            done += sum(ex.map(one, chunk))
            i += len(chunk)
    dt = time.perf_counter() - t0
    return {"value": round(STEP_BYTES * done / R / dt / 1e9, 5), "unit": "GB/s", "cores": workers, "kind": "oracle",
            "sample": f"{done} of {R} rows of both tensors (bands of {band} rows, row- and column-wise, "
                      f"tcgen05 scales), {dt:.1f} s on {workers} threads", "seconds": round(dt, 2)}


def gemm_cpu_baseline(shape, afmt, bfmt, bsig, target_s=6.0):
    """The oracle's fp64 matmul reference (one plain k-loop per entry) on sampled entries of
    the benchmark's operands, on all host cores; TFLOP/s = 2 K x entries / wall time."""
    import oracle
    M, N, K = shape
    fm = {"e4m3": oracle.E4M3, "e2m1": oracle.E2M1, "e2m3": oracle.E2M3}
    rng = np.random.default_rng(5)
    ra = np.sort(rng.choice(M, 32, replace=False))
    rb = np.sort(rng.choice(N, 32, replace=False))
    a = synth.normal(M, K, seed=40)[ra]
    b = synth.normal(N, K, sigma=bsig, seed=41)[rb]
    ae, as_ = oracle.quantize_mx(a, fm[afmt], oracle.ROW, oracle.CEIL)
    be, bs = oracle.quantize_mx(b, fm[bfmt], oracle.ROW, oracle.FLOOR if bfmt == "e2m1" else oracle.CEIL)
    pairs = np.array([(i, j) for i in range(32) for j in range(32)], dtype=np.int64)
    workers = _workers()
    chunks = [pairs[i::workers] for i in range(workers)]

    def one(p):
        oracle.gemm_ref(ae, as_, fm[afmt], be, bs, fm[bfmt], 32, 32, K, p)
        return len(p)

    t0 = time.perf_counter()
    done = 0
    with cf.ThreadPoolExecutor(workers) as ex:
        while time.perf_counter() - t0 < target_s:
            done += sum(ex.map(one, chunks))
    dt = time.perf_counter() - t0
    return {"value": round(2.0 * K * done / dt / 1e12, 8), "unit": "TFLOP/s", "cores": workers, "kind": "oracle",
            "sample": f"{done} entries of C ({len(pairs)} distinct, K = {K}), fp64, {dt:.1f} s on {workers} threads"}


def step_config(world):
    """The headline workload's description, the same in both arms' lines."""
    return {"workload": WORKLOAD,
            "tensors": {"activations": {"shape": list(ACT), "format": "MXFP8 E4M3", "bytes": BYTES_ACT},
                        "gradients": {"shape": list(GRAD), "format": "MXFP8 E5M2", "bytes": BYTES_GRAD}},
            "orientations": "row-wise and column-wise (transposed) from one read",
            "scale_rule": "no-clip (ceil), E8M0, block 32", "scale_layout": "tcgen05",
            "step_bytes": STEP_BYTES,
            "l2": "inputs larger than L2 (604 MB per step), no flush needed",
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU"}


def run_reference(args, rank, world):
    """The oracle as the reference arm: rank 0 only, a bounded sample per step."""
    if rank != 0:
        return
    a_bits = synth.activations(seed=0)
    g_bits = synth.gradients(seed=1)
    per_step = max(1.0, args.cpu_seconds / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        cpu_baseline(a_bits, g_bits, target_s=per_step)
    vals, secs = [], []
    for _ in range(args.steps):
        r = cpu_baseline(a_bits, g_bits, target_s=per_step)
        vals.append(r["value"])
        secs.append(r["seconds"])
        sample, cores = r["sample"], r["cores"]
    v = statistics.mean(vals)
    line = {"impl": "reference", "metric": METRIC, "value": round(v, 5), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * statistics.mean(secs), 1),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic (numpy default_rng; activations seed 0, gradients seed 1)",
            "config": step_config(world),
            "cpu_baseline": {"kind": "oracle", "cores": cores, "sample": sample, "value": round(v, 5)},
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
    elif name == "weight4096_one_call":
        st = WeightQuantStep(mx, to_dev(synth.weight_fp4(), dev))
        fns = [lambda: st.both(stream.cuda_stream)]
    elif name == "step":
        # the headline step itself (both dual calls), for the launch list and DRAM traffic
        st = DualStep(mx, to_dev(synth.activations(), dev), to_dev(synth.gradients(), dev))
        fns = [lambda: st.run(stream.cuda_stream)]
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
    elif name == "quant_act":
        # row-wise and column-wise-only MXFP8 (E4M3, no-clip, tcgen05 scales) of the activations
        xa = to_dev(synth.activations(), dev)
        qr = mx.quantize(xa, "e4m3", "row", "ceil", layout="tcgen05")
        qc = mx.quantize(xa, "e4m3", "col", "ceil", layout="tcgen05")
        fns = [lambda: (mx.quantize(xa, "e4m3", "row", "ceil", layout="tcgen05", out=qr),
                        mx.quantize(xa, "e4m3", "col", "ceil", layout="tcgen05", out=qc))]
    elif name == "dequant_act":
        xa = to_dev(synth.activations(), dev)
        qs = [mx.quantize(xa, f, "row", r, layout="tcgen05") for f, r in (("e4m3", "ceil"), ("e2m1", "floor"),
                                                                           ("nvfp4", "ceil"))]
        y = torch.empty_like(xa)
        fns = [lambda: [mx.dequantize(q, "tcgen05", out=y) for q in qs]]
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


CASES = ["step", "weight4096", "weight4096_one_call", "mx8_1024", "dual_act", "dual_grad", "dequant4096", "dequant_act",
         "quant_act",
         "gemm8192", "gemm_w4a8",
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
