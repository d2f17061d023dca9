#!/usr/bin/env python
"""Benchmark of the DualScale / SegLinear quantized linear layer on B200.

One step = one pass of the whole path over one batch: static calibration on
the workload's calibration rows, weight quantization, and the forward.  With
the default `--path codes` the forward writes the DualScale codes q+/q- once
and runs the GEMM from codes (two int8 tensor-core products per k step, fused
epilogue); `--path fused` quantizes inside the GEMM, `--path combined` goes
through the combined code.  The metric counts the executed int8 work of the
forward, 4*M*N*K ops (two products, one per polarity), per second of step
time.  The same line reports the dominant kernel against its roofline, the
fused, single-scale and (int4 weights) block-Hadamard forwards beside it, the
small-M forwards, the end-to-end rate through the API with host buffers, and
the CPU oracle on the host cores.

Timing: W warm-up steps, then K timed steps (each one CUDA-graph replay) on
the device with CUDA events on the launching stream; before every timed
launch the L2 is flushed (a 256 MiB write, then a 256 MiB read, outside the
events) so that every step starts from a cold L2.  Under torchrun each rank
runs its own batch (independent problems, no collective on the data path), the
per-rank time is the max over ranks, and the value is the whole-job rate.

`--impl reference` times the CPU oracle (the plain C implementation in
oracle/) on the host cores, on a bounded row sample of the same workload.
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "quantized-linear int8 TOPS and % of B200 int8 tensor peak (GB/s at small M)"
FALLBACK_BF16_TFLOPS = 1590.0
FALLBACK_HBM_GBS = 6650.0
INT8_PER_BF16 = 2.0  # nominal dense ratio: 4.5 POPS int8 / 2.25 PFLOP/s bf16

# DRAM bytes (read + write) of one launch of the dominant kernel, from one ncu
# capture of the current kernel build (profiles/*.md); keyed by (workload,
# path).  Absent: no capture of the current build.
NCU_TRAFFIC_BYTES = {
    ("dit_xl2_fc2_cfg", "codes"): 93068032 + 11148288,   # dualscale_gemm_codes_kernel
    ("w4a8", "codes"): 105879296 + 71072768,             # dualscale_gemm_codes_kernel (W4)
}


def gemm_kernel_name(path: str, bits: int, x_dtype: str) -> str:
    """The GEMM kernel a forward of this path launches (default switches)."""
    if path == "codes":          # int8 and int4 weights alike
        return "dualscale_gemm_codes_kernel"
    if bits == 4:
        return "dualscale_gemm_kernel"
    if path == "combined":
        return "dualscale_gemm_combined_kernel"
    return "dualscale_gemm_inplace_kernel" if x_dtype == "bf16" else "dualscale_gemm_kernel"


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="dit_xl2_fc2_cfg")
    ap.add_argument("--path", choices=["fused", "codes", "combined"], default="codes",
                    help="fused: quantize X inside the GEMM; codes: quantize X once into "
                         "q+/q- code tensors, then the GEMM loads the codes; combined: quantize "
                         "X once into c = q+ + q- (one byte per activation), then the GEMM "
                         "loads c and splits it")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--no-small-m", action="store_true",
                    help="skip the small-M (M <= 128, HBM-bound) measurements")
    ap.add_argument("--small-m-only", action="store_true",
                    help="run only the small-M measurements (one GPU) and print them as one "
                         "JSON line; not a bench line")
    return ap.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["bf16_tflops"]) * INT8_PER_BF16, float(p["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_BF16_TFLOPS * INT8_PER_BF16, FALLBACK_HBM_GBS, "fallback"


# ------------------------------------------------------------------ L2 flush
class L2Flush:
    """Evicts the step's inputs from the 126 MB L2 before every timed launch:
    writes a 256 MiB buffer, then reads a second 256 MiB buffer, so the dirty
    lines of the write are written back inside the flush and the L2 is left
    holding clean lines (a write-only flush would leave the next launch to pay
    for writing ~126 MB back to HBM)."""

    def __init__(self, dev):
        import torch
        self.a = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        self.b = torch.ones(256 << 20, dtype=torch.uint8, device=dev)

    def __call__(self, i: int):
        self.a.fill_(i & 0xFF)
        self.b.max()


# ------------------------------------------------------------------ small M
SMALL_M_SHAPES = ((3072, 12288), (4608, 1152))
SMALL_M_ROWS = (16, 64, 128)
SMALL_M_LAYERS = 8     # distinct weight copies of the layer-stream measurement


def small_m_measure(dev, flush, steps: int, hbm_peak: float):
    """HBM-bound small-M forwards (one K segment, int8 weights, bf16 out): the
    split-K GEMM from codes and the one-pass GEMM from codes, each replayed
    from a CUDA graph with the L2 flushed before every launch.  Bytes = weight
    codes + weight scales + q+/q- codes + Y (the algorithmic traffic).

    `one_pass_layers`: the one-pass GEMM over SMALL_M_LAYERS distinct copies
    of the weight, back to back in one graph (a stack of layers, each reading
    its own cold weight: 8 x 37.7 MB exceeds the L2), the L2 flushed before
    every replay; time per layer = replay time / layers.  This spreads the
    replay's fixed launch cost (several microseconds, and the event clock here
    advances in 2.048-microsecond steps) over the layers, as in a model."""
    import torch
    import post_quantized_linear_b200 as pq
    from synth import workloads as W
    out = []
    for (K, N) in SMALL_M_SHAPES:
        for M in SMALL_M_ROWS:
            wl = W.small_case(M, K, N, seed=7, act="silu", bias=False, out="bf16")
            x, w, _ = W.generate(wl)
            xd, wd = x.to(dev), w.to(dev)
            sp, sn = pq.calibrate(xd, wl.kseg)
            qw = pq.quantize_weights(wd, wl.kseg, wl.nseg, bits=8)
            qp, qn = pq.quantize_activations(xd, wl.kseg, sp, sn)
            y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
            ws = pq.splitk_workspace(M, N, K, device=dev)
            res = {"M": M, "K": K, "N": N}
            for name, fn in (("splitk", lambda: pq.linear_from_codes_splitk(qp, qn, qw, sp, sn, ws, out=y)),
                             ("one_pass", lambda: pq.linear_from_codes(qp, qn, qw, sp, sn, out=y))):
                fn()
                torch.cuda.synchronize()
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g):
                    fn()
                ts = []
                for i in range(max(steps, 5)):
                    flush(i)
                    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    e0.record()
                    g.replay()
                    e1.record()
                    torch.cuda.synchronize()
                    ts.append(e0.elapsed_time(e1))
                us = statistics.median(ts) * 1e3
                byts = N * K + 4 * N + 2 * M * K + 2 * M * N
                res[name] = {"us": us, "gbs": byts / (us * 1e-6) / 1e9,
                             "frac_hbm": byts / (us * 1e-6) / 1e9 / hbm_peak}
                del g
            qws = [qw] + [pq.quantize_weights(wd, wl.kseg, wl.nseg, bits=8)
                          for _ in range(SMALL_M_LAYERS - 1)]
            ys = [torch.empty((M, N), dtype=torch.bfloat16, device=dev) for _ in qws]

            def layers():
                for q_l, y_l in zip(qws, ys):
                    pq.linear_from_codes(qp, qn, q_l, sp, sn, out=y_l)
            layers()
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                layers()
            ts = []
            for i in range(max(steps, 5)):
                flush(i)
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                g.replay()
                e1.record()
                torch.cuda.synchronize()
                ts.append(e0.elapsed_time(e1))
            us = statistics.median(ts) * 1e3 / len(qws)
            res["one_pass_layers"] = {"layers": len(qws), "us_per_layer": us,
                                      "gbs": byts / (us * 1e-6) / 1e9,
                                      "frac_hbm": byts / (us * 1e-6) / 1e9 / hbm_peak}
            del g, qws, ys
            out.append(res)
    return out


# ------------------------------------------------------------------ clocks
REASON_BITS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}


class ClockSampler:
    """nvidia-smi sampled every 200 ms while the timed region runs."""

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.rows = []
        self.proc = None
        self.thread = None

    def start(self):
        cmd = ["nvidia-smi", "-i", str(self.gpu),
               "--query-gpu=clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active",
               "--format=csv,noheader,nounits", "-lms", "200"]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 4:
                self.rows.append(parts)

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], None, set()
        for p in self.rows:
            try:
                s = float(p[0]); m = float(p[1]); r = int(p[3], 16)
            except ValueError:
                continue
            mx = m
            if r & 0x1:  # idle sample
                continue
            sm.append(s)
            for bit, name in REASON_BITS.items():
                if r & bit:
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------- CPU oracle
def cpu_oracle_step(wl, xn, wn, bn, rows):
    """One oracle step on a row sample; returns (seconds, seconds scaled to the full batch)."""
    import numpy as np
    import oracle as O
    t0 = time.perf_counter()
    calib = xn if wl.calib_rows is None else xn[: wl.calib_rows]
    sp, sn = O.calibrate(calib, wl.kseg)
    t1 = time.perf_counter()
    if wl.bits == 8:
        wc, ws = O.quantize_weights_w8(wn, wl.kseg)
    else:
        wc, ws = O.quantize_weights_w4(wn)
    t2 = time.perf_counter()
    O.linear_forward(np.ascontiguousarray(xn[:rows]), wl.kseg, sp, sn, wl.bits, wc, ws, bn,
                     out="f32" if wl.out == "f32" else "bf16")
    t3 = time.perf_counter()
    return t3 - t0, (t2 - t0) + (t3 - t2) * (wl.M / rows)


def cpu_baseline(wl, x, w, b, target_s=12.0):
    import numpy as np
    import oracle as O
    from synth import workloads as W
    O.build()
    xn, wn = W.to_numpy_x(x), w.numpy()
    bn = None if b is None else b.numpy()
    probe_rows = 8
    t_probe, _ = cpu_oracle_step(wl, xn, wn, bn, probe_rows)
    per_row = max(t_probe / probe_rows, 1e-6)
    rows = int(max(8, min(wl.M, target_s / per_row)))
    t, t_full = cpu_oracle_step(wl, xn, wn, bn, rows)
    cores = len(os.sched_getaffinity(0))
    threads = int(os.environ.get("OMP_NUM_THREADS", cores))
    return {
        "value": wl.exec_ops / t_full / 1e12, "unit": "TOPS", "cores": threads, "kind": "oracle",
        "sample": (f"calibration on the full calibration rows, weight quantization of the full "
                   f"[{wl.N},{wl.K}] weight, forward of {rows}/{wl.M} rows ({t:.1f} s); "
                   "forward time scaled by M/rows"),
    }


def run_reference(args):
    """The reference arm: the CPU oracle, as it stands, on the host cores."""
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from synth import workloads as W
    import oracle as O
    O.build()
    wl = W.WORKLOADS[args.workload]
    x, w, b = W.generate(wl)
    xn, wn = W.to_numpy_x(x), w.numpy()
    bn = None if b is None else b.numpy()
    steps, warm = args.steps, args.warmup
    budget_s = 150.0
    t_probe, _ = cpu_oracle_step(wl, xn, wn, bn, 8)
    per_row = max(t_probe / 8, 1e-6)
    rows = int(max(8, min(wl.M, budget_s / (steps + warm) / per_row)))
    for _ in range(warm):
        cpu_oracle_step(wl, xn, wn, bn, rows)
    full = []
    raw = []
    for _ in range(steps):
        t, tf = cpu_oracle_step(wl, xn, wn, bn, rows)
        raw.append(t)
        full.append(tf)
    t_step = sum(full) / len(full)
    value = wl.exec_ops / t_step / 1e12
    cores = len(os.sched_getaffinity(0))
    threads = int(os.environ.get("OMP_NUM_THREADS", cores))
    sample = (f"each step: calibration on the calibration rows, full weight quantization, "
              f"forward of {rows}/{wl.M} rows (mean {sum(raw)/len(raw):.2f} s); forward time "
              "scaled by M/rows")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": world,
        "steps": steps, "warmup": warm, "ms_per_step": t_step * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "int8", "data": "synthetic",
        "config": config_of(wl, "host cores, no L2 flush", "oracle"),
        "cpu_baseline": {"value": value, "unit": "TOPS", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def config_of(wl, l2, path="fused"):
    return {"workload": wl.name, "path": path, "M": wl.M, "K": wl.K, "N": wl.N, "bits": wl.bits,
            "x_dtype": wl.x_dtype, "out_dtype": wl.out, "k_segments": list(wl.kseg),
            "n_segments": list(wl.nseg), "calib_rows": wl.calib_rows or wl.M,
            "global_batch": wl.M, "l2": l2}


# ------------------------------------------------------------- GPU arm
def run_ours(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))

    import post_quantized_linear_b200 as pq
    from synth import workloads as W

    if args.small_m_only:
        dev = torch.device("cuda", local)
        hbm_peak = peaks()[1]
        print(json.dumps({"small_m": {"peak_gbs": hbm_peak, "cases": small_m_measure(
            dev, L2Flush(dev), args.steps, hbm_peak)}}), flush=True)
        return 0

    wl = W.WORKLOADS[args.workload]
    import dataclasses
    wl_rank = dataclasses.replace(wl, seed=wl.seed + rank)
    x, w, b = W.generate(wl_rank)
    dev = torch.device("cuda", local)
    xd, wd = x.to(dev), w.to(dev)
    bd = None if b is None else b.to(dev)
    out_dtype = torch.float32 if wl.out == "f32" else torch.bfloat16
    J = len(wl.kseg) - 1
    sp = torch.empty(J, dtype=torch.float32, device=dev)
    sn = torch.empty(J, dtype=torch.float32, device=dev)
    qw = pq.quantize_weights(wd, wl.kseg, wl.nseg, bits=wl.bits)
    y = torch.empty((wl.M, wl.N), dtype=out_dtype, device=dev)
    calib = xd if wl.calib_rows is None else xd[: wl.calib_rows]
    use_codes = args.path in ("codes", "combined")
    combined = args.path == "combined"
    if use_codes:
        ldq = (wl.K + 15) // 16 * 16
        qp_buf = torch.empty((wl.M, ldq), dtype=torch.int8, device=dev)[:, : wl.K]
        qn_buf = None if combined else torch.empty((wl.M, ldq), dtype=torch.int8, device=dev)[:, : wl.K]
    stream = torch.cuda.current_stream()
    flush = L2Flush(dev)

    def step(xs=xd, ws=wd, ys=y, gemm_events=None):
        pq.calibrate(calib if xs is xd else (xs if wl.calib_rows is None else xs[: wl.calib_rows]),
                     wl.kseg, sp, sn)
        pq.quantize_weights(ws, wl.kseg, wl.nseg, bits=wl.bits, out=qw)
        forward(xs, ys, gemm_events)

    def gemm(xs, ys):
        if combined:
            pq.linear_from_combined(qp_buf, qw, sp, sn, bd, out=ys)
        elif use_codes:
            pq.linear_from_codes(qp_buf, qn_buf, qw, sp, sn, bd, out=ys)
        else:
            pq.linear(xs, qw, sp, sn, bd, out=ys)

    def forward(xs, ys, gemm_events=None):
        if combined:
            pq.quantize_activations_combined(xs, wl.kseg, sp, sn, out=qp_buf)
        elif use_codes:
            pq.quantize_activations(xs, wl.kseg, sp, sn, out=(qp_buf, qn_buf))
        if gemm_events:
            gemm_events[0].record(stream)
        gemm(xs, ys)
        if gemm_events:
            gemm_events[1].record(stream)

    def events(n):
        return [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                for _ in range(n)]

    launches_per_step = 4 if use_codes else 3
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if pq.stream_status() != 0:
        raise RuntimeError("device status word set during warm-up")

    # The step, the forward and the GEMM alone are each captured once into a
    # CUDA graph and replayed: one launch per step, no host gaps between the
    # step's kernels.
    def capture(fn):
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            fn()
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            fn()
        torch.cuda.synchronize()
        return graph

    def gemm_only():
        gemm(xd, y)

    step_graph = capture(step)
    fwd_graph = capture(lambda: forward(xd, y))
    gemm_graph = capture(gemm_only)
    fused_graph = capture(lambda: pq.linear(xd, qw, sp, sn, bd, out=y)) if use_codes else None
    # The single-scale baseline (one symmetric scale per K segment) of the same
    # forward: its codes, then one int8 product per unit.
    single_graph = None
    if wl.bits == 8:
        ldc = (wl.K + 15) // 16 * 16
        c1_buf = torch.empty((wl.M, ldc), dtype=torch.int8, device=dev)[:, : wl.K]

        def single_forward():
            pq.quantize_activations_single(xd, wl.kseg, sp, sn, out=c1_buf)
            pq.linear_from_single(c1_buf, qw, sp, sn, bd, out=y)
        single_graph = capture(single_forward)
    # int4 weights: the block-Hadamard variant (HQ-DM) of the same forward --
    # codes of XH, then the product with the rotated int4 codes.  Its scales
    # and the weight rotation are offline steps, made once here.
    had_graph = None
    if wl.bits == 4:
        hsp = torch.empty(J, dtype=torch.float32, device=dev)
        hsn = torch.empty(J, dtype=torch.float32, device=dev)
        pq.calibrate_hadamard(calib, wl.kseg, hsp, hsn)
        w_rot = pq.rotate_weights_hadamard(qw)
        ldh = (wl.K + 15) // 16 * 16
        hq_p = torch.empty((wl.M, ldh), dtype=torch.int8, device=dev)[:, : wl.K]
        hq_n = torch.empty((wl.M, ldh), dtype=torch.int8, device=dev)[:, : wl.K]

        def hadamard_forward():
            pq.quantize_activations_hadamard(xd, wl.kseg, hsp, hsn, out=(hq_p, hq_n))
            pq.linear_from_codes_hadamard(hq_p, hq_n, qw, w_rot, hsp, hsn, bd, out=y)
        had_graph = capture(hadamard_forward)

    def timed(graph, n, salt):
        evs = events(n)
        for i in range(n):
            flush(i + salt)
            evs[i][0].record(stream)
            graph.replay()
            evs[i][1].record(stream)
        torch.cuda.synchronize()
        return [a.elapsed_time(b) for a, b in evs]

    timed(step_graph, 2, 0)
    sampler = None if args.no_clocks else ClockSampler(local)
    if sampler:
        sampler.start()
        time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    step_ms = timed(step_graph, args.steps, 1)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop() if sampler else None
    total_ms = sum(step_ms)
    gemm_ms = timed(gemm_graph, args.steps, 3)
    fwd_ms = timed(fwd_graph, args.steps, 5)
    fused_ms = timed(fused_graph, args.steps, 7) if fused_graph is not None else None
    single_ms = timed(single_graph, args.steps, 9) if single_graph is not None else None
    had_ms = timed(had_graph, args.steps, 11) if had_graph is not None else None
    if pq.stream_status() != 0:
        raise RuntimeError("device status word set during the timed region")
    del step_graph, fwd_graph, gemm_graph, fused_graph, single_graph, had_graph

    # end to end through the API: host inputs in, host result out, every step
    e2e = None
    if not args.no_e2e:
        xh = x.pin_memory()
        wh = w.pin_memory()
        yh = torch.empty((wl.M, wl.N), dtype=out_dtype).pin_memory()
        xdd = torch.empty_like(xd)
        wdd = torch.empty_like(wd)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

        def e2e_step():
            xdd.copy_(xh, non_blocking=True)
            wdd.copy_(wh, non_blocking=True)
            step(xs=xdd, ws=wdd)
            yh.copy_(y, non_blocking=True)

        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e0.record(stream)
        for _ in range(args.steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_total = e0.elapsed_time(e1)
        bi = xh.numel() * xh.element_size() + wh.numel() * wh.element_size()
        bo = yh.numel() * yh.element_size()
        e2e = {"ms": e2e_total, "bi": bi, "bo": bo}

    # max over ranks
    vals = [total_ms, statistics.mean(gemm_ms), statistics.mean(fwd_ms),
            e2e["ms"] if e2e else 0.0, statistics.mean(fused_ms) if fused_ms else 0.0,
            statistics.mean(single_ms) if single_ms else 0.0,
            statistics.mean(had_ms) if had_ms else 0.0]
    if world > 1:
        t = torch.tensor(vals, dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        vals = t.tolist()
    total_ms, gemm_avg_ms, fwd_avg_ms, e2e_ms, fused_avg_ms, single_avg_ms, had_avg_ms = vals

    if rank == 0:
        int8_peak_tops, hbm_peak, peak_kind = peaks()
        ops = wl.exec_ops
        value = world * args.steps * ops / (total_ms * 1e-3) / 1e12
        gemm_tops = ops / (gemm_avg_ms * 1e-3) / 1e12
        line = {
            "metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8",
            "data": "synthetic",
            "config": config_of(wl, "flushed (256 MiB write + 256 MiB read between steps)", args.path),
            "roofline": {
                "bound": "tensor", "kernel": gemm_kernel_name(args.path, wl.bits, wl.x_dtype),
                "achieved": gemm_tops, "peak": int8_peak_tops, "unit": "TOPS",
                "frac": gemm_tops / int8_peak_tops,
                "traffic": NCU_TRAFFIC_BYTES.get((wl.name, args.path)),
                "peak_source": f"{peak_kind} bf16 burst x {INT8_PER_BF16:g} (nominal int8/bf16)",
                "algorithmic_ops_per_launch": ops,
                "algorithmic_bytes_per_launch": wl.alg_bytes(),
                "achieved_gbs": wl.alg_bytes() / (gemm_avg_ms * 1e-3) / 1e9,
                "avg_launch_us": gemm_avg_ms * 1e3,
            },
            "forward_only": {
                "us": fwd_avg_ms * 1e3, "exec_tops": ops / (fwd_avg_ms * 1e-3) / 1e12,
                "linear_equiv_tops": ops / 2 / (fwd_avg_ms * 1e-3) / 1e12,
                "frac_int8_peak": ops / (fwd_avg_ms * 1e-3) / 1e12 / int8_peak_tops,
            },
            "gpu_launches": launches_per_step * args.steps,
            "timing": "each step one CUDA-graph replay, CUDA events on the launching stream",
            "clocks": clocks,
        }
        if had_ms:
            line["hadamard_forward"] = {
                "us": had_avg_ms * 1e3,
                "exec_tops": ops / (had_avg_ms * 1e-3) / 1e12,
                "over_dualscale_forward": had_avg_ms / fwd_avg_ms,
                "note": "block-Hadamard activations (blocks of 16): codes of XH, then the product "
                        "with the Hadamard-rotated int4 codes (rotation and its scales offline)"}
        if single_ms:
            line["single_scale_forward"] = {
                "us": single_avg_ms * 1e3,
                "exec_tops": ops / 2 / (single_avg_ms * 1e-3) / 1e12,
                "dualscale_over_single": fwd_avg_ms / single_avg_ms,
                "note": "naive baseline: one symmetric scale per K segment, its codes, then one "
                        "int8 product (half the MMA work of DualScale)",
            }
        if fused_ms:
            line["fused_forward"] = {
                "us": fused_avg_ms * 1e3, "exec_tops": ops / (fused_avg_ms * 1e-3) / 1e12,
                "frac_int8_peak": ops / (fused_avg_ms * 1e-3) / 1e12 / int8_peak_tops,
                "note": "sq_linear_forward: activations quantized inside the GEMM"}
        if e2e:
            line["e2e"] = {"value": world * args.steps * ops / (e2e_ms * 1e-3) / 1e12,
                           "unit": "TOPS", "h2d_bytes_per_step": e2e["bi"],
                           "d2h_bytes_per_step": e2e["bo"]}
        if world == 1 and not args.no_small_m:
            line["small_m"] = {
                "note": "HBM-bound forwards at M <= 128 (median of L2-flushed graph replays; "
                        "one_pass_layers: per layer of 8 back-to-back layers with distinct "
                        "weights); bytes = weight codes + scales + q+/q- codes + Y; peak = "
                        "measured HBM copy",
                "peak_gbs": hbm_peak,
                "cases": small_m_measure(dev, flush, args.steps, hbm_peak)}
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(wl, x, w, b)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
