#!/usr/bin/env python
"""Benchmark of the DualScale / SegLinear quantized linear layer on B200.

One step = one pass of the whole path over one batch: static calibration on
the workload's calibration rows (token-sharded across ranks: each rank
calibrates its own rows and the 2*J scales are all-reduced with MAX), weight
quantization, and the forward.  With the default `--path codes` the forward
writes the DualScale codes q+/q- once and runs the GEMM from codes (two int8
tensor-core products per k step, fused epilogue); `--path fused` quantizes
inside the GEMM, `--path combined` goes through the combined code.  The metric
counts the executed int8 work of the forward, 4*M*N*K ops (two products, one
per polarity), per second of step time.

The default workload is the largest one that fits one GPU, the MMDiT MLP
up-projection (M = 16384, K = 3072, N = 12288).  The same JSON line reports the
dominant kernel against its roofline, the fused, single-scale and (int4
weights) block-Hadamard forwards beside it, every workload configuration
(`configs`: GEMM, forward and step times with their roofline fractions), the
small-M forwards, the host latency of one call, the end-to-end rate through
the API with host buffers, and the CPU oracle on the host cores.

Timing: W warm-up steps, then K timed steps on the device with CUDA events on
the launching stream; before every timed step the L2 is flushed (a 256 MiB
write, then a 256 MiB read, outside the events) so that every step starts from
a cold L2.  `--gpus N` runs N ranks (one process per GPU, launched through
torch.distributed.run when WORLD_SIZE is not set); each rank runs its own batch
(independent problems), the step time is the max over ranks, and the value is
the whole-job rate.

`--impl reference` times the CPU oracle (the plain C implementation in
oracle/) on the host cores, each step on a bounded sample of the workload's
rows.
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import socket
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "quantized-linear int8 TOPS and % of B200 int8 tensor peak (GB/s at small M)"
DEFAULT_WORKLOAD = "mmdit_mlp_up"
CONFIG_ORDER = ("tiny_w8a8", "dit_xl2_fc2_cfg", "seglinear_qkv", "mmdit_mlp_up", "w4a8")
FALLBACK_BF16_TFLOPS = 1590.0
FALLBACK_HBM_GBS = 6650.0
INT8_PER_BF16 = 2.0  # nominal dense ratio: 4.5 POPS int8 / 2.25 PFLOP/s bf16
# tcgen05.mma.kind::i8 with M = 128 and N >= 128 completes 8192 int8 MACs per
# clock per SM (measured with an issue-rate probe on this machine's B200s):
# 16384 int8 ops per clock per SM.
MMA_I8_OPS_PER_CLK_SM = 16384

# DRAM bytes (read + write) of one launch of the dominant kernel, from one ncu
# capture of the current kernel build (profiles/*.md); keyed by (workload,
# path).  Absent: no capture of the current build.
NCU_TRAFFIC_BYTES = {
    ("mmdit_mlp_up", "codes"): 161485056 + 381627392,     # dualscale_gemm_codes_kernel
    ("dit_xl2_fc2_cfg", "codes"): 91399680 + 11276032,    # dualscale_gemm_codes_kernel
    ("seglinear_qkv", "codes"): 56157696 + 30311936,      # dualscale_gemm_codes_kernel
    ("w4a8", "codes"): 105579776 + 67246080,              # dualscale_gemm_codes_kernel (int4)
}


def gemm_kernel_name(path: str, bits: int, x_dtype: str) -> str:
    """The GEMM kernel a forward of this path launches (product library)."""
    if path == "codes":          # int8 and int4 weights alike
        return "dualscale_gemm_codes_kernel"
    if bits == 4:
        return "dualscale_gemm_kernel"
    if path == "combined":
        return "dualscale_gemm_combined_kernel"
    return "dualscale_gemm_inplace_kernel" if x_dtype == "bf16" else "dualscale_gemm_kernel"


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--path", choices=["fused", "codes", "combined"], default="codes",
                    help="fused: quantize X inside the GEMM; codes: quantize X once into "
                         "q+/q- code tensors, then the GEMM loads the codes; combined: quantize "
                         "X once into c = q+ + q- (one byte per activation), then the GEMM "
                         "loads c and splits it")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the per-configuration table (every workload's GEMM/forward/step)")
    ap.add_argument("--no-small-m", action="store_true",
                    help="skip the small-M (M <= 128, HBM-bound) measurements")
    ap.add_argument("--small-m-only", action="store_true",
                    help="run only the small-M measurements (one GPU) and print them as one "
                         "JSON line; not a bench line")
    ap.add_argument("--fused-act-only", action="store_true",
                    help="run only the fused-activation measurements (one GPU) and print them "
                         "as one JSON line; not a bench line")
    return ap.parse_args(argv)


def peaks():
    """(int8 TOPS denominator, HBM GB/s, source): the measured bf16 burst
    figure times the nominal int8/bf16 ratio and the measured copy bandwidth,
    else the recipe's fallback."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["bf16_tflops"]) * INT8_PER_BF16, float(p["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_BF16_TFLOPS * INT8_PER_BF16, FALLBACK_HBM_GBS, "fallback"


def mma_rate_tops(sms: int, sm_mhz: float) -> float:
    """The tcgen05 int8 MMA issue rate of `sms` SMs at `sm_mhz` (TOPS)."""
    return MMA_I8_OPS_PER_CLK_SM * sms * sm_mhz * 1e6 / 1e12


# fp32 lanes per SM (four sub-partitions of 32).  A packed f32x2 instruction
# holds its pipe for two cycles (instruction-mix counters of the int4 GEMM), so
# pairs do not raise this rate.
FP32_LANES_SM = 128
# int4 groups: per output element and 128-wide group the fold takes two exact
# seed subtractions, one product and two fused multiply-adds.
FOLD_OPS_PER_OUTPUT_GROUP = 5


def fold_roofline(wl, gemm_us: float, mma_peak: float) -> dict:
    """The per-group fold of an int4 GEMM against the SMs' fp32 lane rate (an
    FMA counted as one operation), at the clock the MMA rate was taken at."""
    ops = wl.M * wl.N * (wl.K // 128) * FOLD_OPS_PER_OUTPUT_GROUP
    peak = mma_peak * FP32_LANES_SM / MMA_I8_OPS_PER_CLK_SM      # T fp32 ops/s
    achieved = ops / (gemm_us * 1e-6) / 1e12
    return {"bound": "alu", "achieved": achieved, "peak": peak, "unit": "T fp32 ops/s",
            "frac": achieved / peak, "ops_per_launch": ops,
            "floor_us": ops / (peak * 1e12) * 1e6,
            "peak_source": f"{FP32_LANES_SM} fp32 lanes/clk/SM x SMs x the MMA rate's clock"}


# ------------------------------------------------------------ rank launch
def free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def rank_env():
    """(world, rank, local rank) from the torch.distributed launcher's environment."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def relaunch_command(argv, gpus: int, port: int):
    """The torch.distributed.run command that starts `gpus` ranks of this script."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
            f"--nproc-per-node={gpus}", "--master-addr=127.0.0.1", f"--master-port={port}",
            os.path.abspath(__file__), *argv]


def check_world(gpus: int):
    """None when the launch matches --gpus; else the reason it does not."""
    if "WORLD_SIZE" in os.environ and int(os.environ["WORLD_SIZE"]) != gpus:
        return f"WORLD_SIZE={os.environ['WORLD_SIZE']} but --gpus {gpus}"
    return None


def max_over_ranks(vals, world: int, device):
    """Element-wise max of a list of floats over the ranks (identity at world 1)."""
    if world == 1:
        return list(vals)
    import torch
    import torch.distributed as dist
    t = torch.tensor(vals, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def rank_workload(wl, rank: int):
    """The batch of rank r: the workload drawn with seed + r (independent problems)."""
    import dataclasses
    return dataclasses.replace(wl, seed=wl.seed + rank)


def whole_job_tops(world: int, steps: int, ops: int, total_ms: float) -> float:
    """Executed int8 TOPS of the whole job: every rank's steps over the slowest rank's time."""
    return world * steps * ops / (total_ms * 1e-3) / 1e12


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


def timed_graph(graph, n: int, salt: int, flush, stream):
    """Device times (ms) of n replays, each after an L2 flush, CUDA events on `stream`."""
    import torch
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(n)]
    for i in range(n):
        flush(i + salt)
        evs[i][0].record(stream)
        graph.replay()
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in evs]


def capture(fn):
    """fn captured once into a CUDA graph (after one run on a side stream)."""
    import torch
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
    stream = torch.cuda.current_stream()
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
            byts = N * K + 4 * N + 2 * M * K + 2 * M * N
            for name, fn in (("splitk", lambda: pq.linear_from_codes_splitk(qp, qn, qw, sp, sn, ws, out=y)),
                             ("one_pass", lambda: pq.linear_from_codes(qp, qn, qw, sp, sn, out=y))):
                g = capture(fn)
                us = statistics.median(timed_graph(g, max(steps, 5), 0, flush, stream)) * 1e3
                res[name] = {"us": us, "gbs": byts / (us * 1e-6) / 1e9,
                             "frac_hbm": byts / (us * 1e-6) / 1e9 / hbm_peak}
                del g
            qws = [qw] + [pq.quantize_weights(wd, wl.kseg, wl.nseg, bits=8)
                          for _ in range(SMALL_M_LAYERS - 1)]
            ys = [torch.empty((M, N), dtype=torch.bfloat16, device=dev) for _ in qws]

            def layers():
                for q_l, y_l in zip(qws, ys):
                    pq.linear_from_codes(qp, qn, q_l, sp, sn, out=y_l)
            g = capture(layers)
            us = statistics.median(timed_graph(g, max(steps, 5), 0, flush, stream)) * 1e3 / len(qws)
            res["one_pass_layers"] = {"layers": len(qws), "us_per_layer": us,
                                      "gbs": byts / (us * 1e-6) / 1e9,
                                      "frac_hbm": byts / (us * 1e-6) / 1e9 / hbm_peak}
            del g, qws, ys
            out.append(res)
    return out


FUSED_ACT_CASES = (("dit_xl2_fc2_cfg", "gelu"), ("w4a8", "silu"))


def fused_act_measure(dev, flush, steps: int, hbm_peak: float):
    """The activation fused into the combined-code producer on the DiT fc2 input
    (GELU) and the W4A8 input (SiLU), against the unfused pair (the framework's
    activation kernel writing X in bf16, then the combined-code quantizer).
    Bytes: fused = Z read (bf16) + codes written; unfused = Z read + X written
    + X read + codes written.  Each a CUDA-graph replay after an L2 flush."""
    import torch
    import post_quantized_linear_b200 as pq
    from synth import workloads as W
    stream = torch.cuda.current_stream()
    out = []
    for name, act in FUSED_ACT_CASES:
        wl = W.WORKLOADS[name]
        g = torch.Generator().manual_seed(wl.seed)
        z = torch.randn((wl.M, wl.K), generator=g).to(torch.bfloat16).to(dev)
        x = torch.empty_like(z)
        ldc = (wl.K + 15) // 16 * 16
        c = torch.empty((wl.M, ldc), dtype=torch.int8, device=dev)[:, : wl.K]
        sp, sn = pq.calibrate_act(z, act, wl.kseg)
        fn = torch.nn.functional.silu if act == "silu" else torch.nn.functional.gelu

        def fused():
            pq.quantize_activations_combined_act(z, act, wl.kseg, sp, sn, out=c)

        def unfused():
            x.copy_(fn(z))
            pq.quantize_activations_combined(x, wl.kseg, sp, sn, out=c)
        res = {"workload": name, "act": act, "M": wl.M, "K": wl.K}
        for key, f, byts in (("fused", fused, 3 * wl.M * wl.K), ("unfused", unfused, 7 * wl.M * wl.K)):
            gph = capture(f)
            us = statistics.median(timed_graph(gph, max(steps, 5), 0, flush, stream)) * 1e3
            res[key] = {"us": us, "gbs": byts / (us * 1e-6) / 1e9,
                        "frac_hbm": byts / (us * 1e-6) / 1e9 / hbm_peak,
                        "bytes": byts}
            del gph
        res["fused_over_unfused"] = res["fused"]["us"] / res["unfused"]["us"]
        out.append(res)
        del z, x, c
    return out


def per_call_measure(dev, calls: int = 200):
    """Host cost of one forward call outside a CUDA graph, the cost a small-M
    caller pays: the GEMM from codes at M = 16, (K, N) = (3072, 12288), called
    `calls` times back to back.  host_us: time for the API call to return
    (argument marshalling, validation, tensor-map encoding, launch); eager_us:
    device time per call of the back-to-back eager launches."""
    import torch
    import post_quantized_linear_b200 as pq
    from synth import workloads as W
    M, K, N = 16, 3072, 12288
    wl = W.small_case(M, K, N, seed=7, act="silu", bias=False, out="bf16")
    x, w, _ = W.generate(wl)
    xd, wd = x.to(dev), w.to(dev)
    sp, sn = pq.calibrate(xd, wl.kseg)
    qw = pq.quantize_weights(wd, wl.kseg, wl.nseg, bits=8)
    qp, qn = pq.quantize_activations(xd, wl.kseg, sp, sn)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    for _ in range(10):
        pq.linear_from_codes(qp, qn, qw, sp, sn, out=y)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    t0 = time.perf_counter()
    for _ in range(calls):
        pq.linear_from_codes(qp, qn, qw, sp, sn, out=y)
    t1 = time.perf_counter()
    e1.record(stream)
    torch.cuda.synchronize()
    return {"M": M, "K": K, "N": N, "calls": calls,
            "host_us": (t1 - t0) / calls * 1e6,
            "eager_us": e0.elapsed_time(e1) / calls * 1e3,
            "note": "sq_linear_forward_codes through the Python binding, outside a CUDA graph"}


# ------------------------------------------------------------------ clocks
REASON_BITS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}


class ClockSampler:
    """SM clock and clock-event reasons sampled while the timed region runs:
    NVML polled every 2 ms (the GPU this process uses, matched by PCI bus id),
    else nvidia-smi every 200 ms."""

    def __init__(self, gpu_index: int, period_s: float = 0.002):
        self.gpu = gpu_index
        self.period = period_s
        self.rows = []
        self.proc = None
        self.thread = None
        self.halt = threading.Event()

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        try:
            import torch
            pr = torch.cuda.get_device_properties(self.gpu)
            bus = f"{pr.pci_domain_id:08x}:{pr.pci_bus_id:02x}:{pr.pci_device_id:02x}.0"
            return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId_v2(bus)
        except Exception:
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.gpu)

    def _poll(self, pynvml, h):
        reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
        mx = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
        while not self.halt.is_set():
            try:
                sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                r = reasons(h)
                self.rows.append([str(sm), str(mx), "", f"{r:x}"])
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        try:
            pynvml, h = self._nvml_handle()
            self.proc = "nvml"
            self.thread = threading.Thread(target=self._poll, args=(pynvml, h), daemon=True)
            self.thread.start()
            return
        except Exception:
            pass
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
        if self.proc == "nvml":
            self.halt.set()
            self.thread.join(timeout=5)
        else:
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
def oracle_step(wl, xn, wn, bn, rows: int):
    """One oracle step on a sample: calibration on the workload's calibration
    rows, quantization of the whole weight, forward of the first `rows` rows.
    Returns (seconds, executed int8 ops of the sampled forward)."""
    import numpy as np
    import oracle as O
    t0 = time.perf_counter()
    calib = xn if wl.calib_rows is None else xn[: wl.calib_rows]
    sp, sn = O.calibrate(calib, wl.kseg)
    if wl.bits == 8:
        wc, ws = O.quantize_weights_w8(wn, wl.kseg)
    else:
        wc, ws = O.quantize_weights_w4(wn)
    O.linear_forward(np.ascontiguousarray(xn[:rows]), wl.kseg, sp, sn, wl.bits, wc, ws, bn,
                     out="f32" if wl.out == "f32" else "bf16")
    return time.perf_counter() - t0, 4 * rows * wl.N * wl.K


def oracle_sample_rows(wl, xn, wn, bn, step_budget_s: float) -> int:
    """Rows of the sampled forward that keep one oracle step near the budget.
    The oracle runs the rows in parallel on the host threads, so the cost per
    row is taken between one and four rows per thread."""
    r1 = min(wl.M, host_threads())
    r2 = min(wl.M, 4 * r1)
    t1, _ = oracle_step(wl, xn, wn, bn, r1)
    t2, _ = oracle_step(wl, xn, wn, bn, r2)
    per_row = max((t2 - t1) / max(r2 - r1, 1), 1e-7)
    fixed = max(t1 - r1 * per_row, 0.0)
    return int(max(r1, min(wl.M, (step_budget_s - fixed) / per_row)))


def host_threads() -> int:
    cores = len(os.sched_getaffinity(0))
    return int(os.environ.get("OMP_NUM_THREADS", cores))


def cpu_baseline(wl, x, w, b, target_s=20.0):
    """The oracle, as it stands, timed on the host cores on a bounded sample."""
    import oracle as O
    from synth import workloads as W
    O.build()
    xn, wn = W.to_numpy_x(x), w.numpy()
    bn = None if b is None else b.numpy()
    rows = oracle_sample_rows(wl, xn, wn, bn, target_s)
    t, ops = oracle_step(wl, xn, wn, bn, rows)
    return {
        "value": ops / t / 1e12, "unit": "TOPS", "cores": host_threads(), "kind": "oracle",
        "sample": (f"one step: calibration on the workload's calibration rows, quantization of "
                   f"the whole [{wl.N},{wl.K}] weight, forward of {rows}/{wl.M} rows; "
                   f"{t:.2f} s measured; value = executed ops of the sampled forward / step time"),
    }


def run_reference(args):
    """The reference arm: the CPU oracle, as it stands, on the host cores; each
    step a bounded sample of the workload's rows, sized so that the whole run
    stays within a few minutes.  Every number is measured (no scaling)."""
    world, rank, _ = rank_env()
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
    rows = oracle_sample_rows(wl, xn, wn, bn, budget_s / max(1, steps + warm))
    for _ in range(warm):
        oracle_step(wl, xn, wn, bn, rows)
    ts = []
    ops = 0
    for _ in range(steps):
        t, ops = oracle_step(wl, xn, wn, bn, rows)
        ts.append(t)
    total = sum(ts)
    value = steps * ops / total / 1e12 if steps else 0.0
    sample = (f"each step: calibration on the workload's calibration rows, quantization of the "
              f"whole [{wl.N},{wl.K}] weight, forward of {rows}/{wl.M} rows; value = executed "
              "ops of the sampled forwards / measured step time")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": world,
        "steps": steps, "warmup": warm, "ms_per_step": total / max(1, steps) * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8",
        "data": "synthetic",
        "config": config_of(wl, "host cores, no L2 flush", "oracle", world, sample_rows=rows),
        "cpu_baseline": {"value": value, "unit": "TOPS", "cores": host_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def config_of(wl, l2, path="codes", world=1, sample_rows=None):
    c = {"workload": wl.name, "path": path, "M": wl.M, "K": wl.K, "N": wl.N, "bits": wl.bits,
         "x_dtype": wl.x_dtype, "out_dtype": wl.out, "k_segments": list(wl.kseg),
         "n_segments": list(wl.nseg), "calib_rows": wl.calib_rows or wl.M,
         "global_batch": wl.M * world, "l2": l2, "parallelism": f"dp{world}"}
    if sample_rows is not None:
        c["sample_rows"] = sample_rows
    return c


# ------------------------------------------------------------- GPU arm
class Layer:
    """One workload's device state and its captured CUDA graphs.

    step():      calibration (token-sharded: local calibration, then the MAX
                 all-reduce of the scales when several ranks run) followed by
                 `rest`, one graph replay of weight quantization + forward;
    fwd_graph:   activation codes + the GEMM (the forward alone);
    gemm_graph:  the GEMM alone (the dominant kernel)."""

    def __init__(self, wl, dev, path: str, rank: int = 0, extras: bool = True):
        import torch
        import post_quantized_linear_b200 as pq
        from synth import workloads as W
        self.wl, self.dev, self.path = wl, dev, path
        x, w, b = W.generate(rank_workload(wl, rank))
        self.x_host, self.w_host = x, w
        self.xd, self.wd = x.to(dev), w.to(dev)
        self.bd = None if b is None else b.to(dev)
        self.out_dtype = torch.float32 if wl.out == "f32" else torch.bfloat16
        J = len(wl.kseg) - 1
        self.sp = torch.empty(J, dtype=torch.float32, device=dev)
        self.sn = torch.empty(J, dtype=torch.float32, device=dev)
        self.qw = pq.quantize_weights(self.wd, wl.kseg, wl.nseg, bits=wl.bits)
        self.y = torch.empty((wl.M, wl.N), dtype=self.out_dtype, device=dev)
        self.calib = self.xd if wl.calib_rows is None else self.xd[: wl.calib_rows]
        self.codes = path in ("codes", "combined")
        self.combined = path == "combined"
        ldq = (wl.K + 15) // 16 * 16
        if self.codes:
            self.qp = torch.empty((wl.M, ldq), dtype=torch.int8, device=dev)[:, : wl.K]
            self.qn = (None if self.combined else
                       torch.empty((wl.M, ldq), dtype=torch.int8, device=dev)[:, : wl.K])
        self.launches_per_step = 4 if self.codes else 3
        self.calibrate()
        torch.cuda.synchronize()
        self.rest_graph = capture(self.rest)
        self.fwd_graph = capture(lambda: self.forward(self.xd, self.y))
        self.gemm_graph = capture(lambda: self.gemm(self.xd, self.y))
        self.fused_graph = self.single_graph = self.had_graph = None
        if not extras:
            return
        if self.codes:
            self.fused_graph = capture(lambda: pq.linear(self.xd, self.qw, self.sp, self.sn,
                                                         self.bd, out=self.y))
        # the single-scale baseline (one symmetric scale per K segment): its
        # codes, then one int8 product per unit
        if wl.bits == 8:
            self.c1 = torch.empty((wl.M, ldq), dtype=torch.int8, device=dev)[:, : wl.K]

            def single_forward():
                pq.quantize_activations_single(self.xd, wl.kseg, self.sp, self.sn, out=self.c1)
                pq.linear_from_single(self.c1, self.qw, self.sp, self.sn, self.bd, out=self.y)
            self.single_graph = capture(single_forward)
        # int4 weights: the block-Hadamard variant (HQ-DM) of the same forward:
        # codes of XH, then the product with the rotated int4 codes (its scales
        # and the weight rotation are offline steps, made once here)
        if wl.bits == 4:
            self.hsp = torch.empty(J, dtype=torch.float32, device=dev)
            self.hsn = torch.empty(J, dtype=torch.float32, device=dev)
            pq.calibrate_hadamard(self.calib, wl.kseg, self.hsp, self.hsn)
            self.w_rot = pq.rotate_weights_hadamard(self.qw)
            self.hq_p = torch.empty((wl.M, ldq), dtype=torch.int8, device=dev)[:, : wl.K]
            self.hq_n = torch.empty((wl.M, ldq), dtype=torch.int8, device=dev)[:, : wl.K]

            def hadamard_forward():
                pq.quantize_activations_hadamard(self.xd, wl.kseg, self.hsp, self.hsn,
                                                 out=(self.hq_p, self.hq_n))
                pq.linear_from_codes_hadamard(self.hq_p, self.hq_n, self.qw, self.w_rot, self.hsp,
                                              self.hsn, self.bd, out=self.y)
            self.had_graph = capture(hadamard_forward)

    def calibrate(self, calib=None):
        from post_quantized_linear_b200 import parallel
        parallel.calibrate_sharded(self.calib if calib is None else calib, self.wl.kseg,
                                   s_pos=self.sp, s_neg=self.sn)

    def gemm(self, xs, ys):
        import post_quantized_linear_b200 as pq
        if self.combined:
            pq.linear_from_combined(self.qp, self.qw, self.sp, self.sn, self.bd, out=ys)
        elif self.codes:
            pq.linear_from_codes(self.qp, self.qn, self.qw, self.sp, self.sn, self.bd, out=ys)
        else:
            pq.linear(xs, self.qw, self.sp, self.sn, self.bd, out=ys)

    def forward(self, xs, ys):
        import post_quantized_linear_b200 as pq
        if self.combined:
            pq.quantize_activations_combined(xs, self.wl.kseg, self.sp, self.sn, out=self.qp)
        elif self.codes:
            pq.quantize_activations(xs, self.wl.kseg, self.sp, self.sn, out=(self.qp, self.qn))
        self.gemm(xs, ys)

    def rest(self, xs=None, ws=None, ys=None):
        import post_quantized_linear_b200 as pq
        pq.quantize_weights(self.wd if ws is None else ws, self.wl.kseg, self.wl.nseg,
                            bits=self.wl.bits, out=self.qw)
        self.forward(self.xd if xs is None else xs, self.y if ys is None else ys)

    def step(self):
        self.calibrate()
        self.rest_graph.replay()

    def timed_steps(self, n: int, salt: int, flush, stream, world: int):
        """Device times (ms) of n steps, each after an L2 flush; ranks enter each
        step together."""
        import torch
        import torch.distributed as dist
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(n)]
        for i in range(n):
            flush(i + salt)
            evs[i][0].record(stream)
            self.step()
            evs[i][1].record(stream)
        torch.cuda.synchronize()
        return [a.elapsed_time(b) for a, b in evs]

    def release(self):
        self.rest_graph = self.fwd_graph = self.gemm_graph = None
        self.fused_graph = self.single_graph = self.had_graph = None


def measure_config(wl, dev, flush, steps: int, warmup: int, int8_peak: float, mma_peak: float,
                   hbm_peak: float, path: str = "codes"):
    """GEMM, forward and step times of one workload configuration (one GPU)."""
    import torch
    stream = torch.cuda.current_stream()
    L = Layer(wl, dev, path, extras=False)
    for _ in range(warmup):
        L.step()
    torch.cuda.synchronize()
    step_ms = statistics.mean(L.timed_steps(steps, 1, flush, stream, 1))
    gemm_ms = statistics.mean(timed_graph(L.gemm_graph, steps, 3, flush, stream))
    fwd_ms = statistics.mean(timed_graph(L.fwd_graph, steps, 5, flush, stream))
    L.release()
    ops, byts = wl.exec_ops, codes_gemm_bytes(wl, path)
    gemm_tops = ops / (gemm_ms * 1e-3) / 1e12
    # a problem of a few MB and tens of MFLOP is launch-latency bound, not tensor bound
    bound = "latency" if byts < 16 * 2 ** 20 and ops < 10 ** 10 else "tensor"
    return {
        "M": wl.M, "K": wl.K, "N": wl.N, "bits": wl.bits, "k_segments": list(wl.kseg),
        "gemm_us": gemm_ms * 1e3, "forward_us": fwd_ms * 1e3, "step_us": step_ms * 1e3,
        "gemm_tops": gemm_tops, "step_tops": ops / (step_ms * 1e-3) / 1e12,
        "roofline": {
            "bound": bound, "kernel": gemm_kernel_name(path, wl.bits, wl.x_dtype),
            "achieved": gemm_tops, "peak": int8_peak, "unit": "TOPS",
            "frac": gemm_tops / int8_peak, "frac_mma_rate": gemm_tops / mma_peak,
            "traffic": NCU_TRAFFIC_BYTES.get((wl.name, path)),
            "algorithmic_bytes_per_launch": byts,
            "achieved_gbs": byts / (gemm_ms * 1e-3) / 1e9,
            "frac_hbm": byts / (gemm_ms * 1e-3) / 1e9 / hbm_peak,
            **({"fold": fold_roofline(wl, gemm_ms * 1e3, mma_peak)} if wl.bits == 4 else {}),
        },
    }


def codes_gemm_bytes(wl, path: str = "codes") -> int:
    """Algorithmic bytes of one launch of the GEMM from codes: q+ and q- codes
    (or the one combined code), weight codes and scales, activation scales,
    bias, Y."""
    J = len(wl.kseg) - 1
    ye = 4 if wl.out == "f32" else 2
    if wl.bits == 8:
        wb = wl.N * wl.K + 4 * J * wl.N
    else:
        wb = wl.N * wl.K // 2 + 2 * wl.N * (wl.K // 128)
    bb = 4 * wl.N if wl.bias_sigma is not None else 0
    codes = (1 if path == "combined" else 2) * wl.M * wl.K
    return codes + wb + 8 * J + bb + wl.M * wl.N * ye


def num_sms(dev) -> int:
    import torch
    return torch.cuda.get_device_properties(dev).multi_processor_count


def run_ours(args):
    import torch
    import torch.distributed as dist

    world, rank, local = rank_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    import post_quantized_linear_b200 as pq
    from synth import workloads as W

    int8_peak, hbm_peak, peak_kind = peaks()
    if args.small_m_only:
        print(json.dumps({"small_m": {"peak_gbs": hbm_peak, "cases": small_m_measure(
            dev, L2Flush(dev), args.steps, hbm_peak)}}), flush=True)
        return 0
    if args.fused_act_only:
        print(json.dumps({"fused_activation": {"peak_gbs": hbm_peak, "cases": fused_act_measure(
            dev, L2Flush(dev), args.steps, hbm_peak)}}), flush=True)
        return 0

    wl = W.WORKLOADS[args.workload]
    stream = torch.cuda.current_stream()
    flush = L2Flush(dev)
    L = Layer(wl, dev, args.path, rank=rank)
    for _ in range(args.warmup):
        L.step()
    torch.cuda.synchronize()
    if pq.stream_status() != 0:
        raise RuntimeError("device status word set during warm-up")
    L.timed_steps(2, 0, flush, stream, world)

    sampler = None if args.no_clocks else ClockSampler(local)
    if sampler:
        sampler.start()
        time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    step_ms = L.timed_steps(args.steps, 1, flush, stream, world)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop() if sampler else None
    total_ms = sum(step_ms)
    gemm_ms = timed_graph(L.gemm_graph, args.steps, 3, flush, stream)
    fwd_ms = timed_graph(L.fwd_graph, args.steps, 5, flush, stream)
    fused_ms = timed_graph(L.fused_graph, args.steps, 7, flush, stream) if L.fused_graph else None
    single_ms = timed_graph(L.single_graph, args.steps, 9, flush, stream) if L.single_graph else None
    had_ms = timed_graph(L.had_graph, args.steps, 11, flush, stream) if L.had_graph else None
    if pq.stream_status() != 0:
        raise RuntimeError("device status word set during the timed region")
    L.release()

    # end to end through the API: host inputs in (pinned), host result out, every
    # step.  Steps are pipelined over two sets of device buffers: step i's
    # inputs are copied in (copy-in stream) while step i-1 computes and step
    # i-2's result is copied out (copy-out stream); PCIe carries both
    # directions at once.  Every step's copies lie inside the timed region.
    e2e = None
    if not args.no_e2e:
        xh = L.x_host.pin_memory()
        wh = L.w_host.pin_memory()
        yh = [torch.empty((wl.M, wl.N), dtype=L.out_dtype).pin_memory() for _ in range(2)]
        xdd = [torch.empty_like(L.xd) for _ in range(2)]
        wdd = [torch.empty_like(L.wd) for _ in range(2)]
        ydd = [L.y, torch.empty_like(L.y)]
        s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()

        def e2e_run(n: int):
            start = torch.cuda.Event()
            start.record(stream)
            done_in = [torch.cuda.Event() for _ in range(n)]
            done_comp = [torch.cuda.Event() for _ in range(n)]
            done_out = [torch.cuda.Event() for _ in range(n)]
            s_in.wait_event(start)
            for i in range(n):
                b = i % 2
                with torch.cuda.stream(s_in):
                    if i >= 2:
                        s_in.wait_event(done_comp[i - 2])   # the compute read buffer b
                    xdd[b].copy_(xh, non_blocking=True)
                    wdd[b].copy_(wh, non_blocking=True)
                    done_in[i].record(s_in)
                stream.wait_event(done_in[i])
                if i >= 2:
                    stream.wait_event(done_out[i - 2])      # ydd[b] was copied out
                L.calibrate(xdd[b] if wl.calib_rows is None else xdd[b][: wl.calib_rows])
                L.rest(xs=xdd[b], ws=wdd[b], ys=ydd[b])
                done_comp[i].record(stream)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(done_comp[i])
                    yh[b].copy_(ydd[b], non_blocking=True)
                    done_out[i].record(s_out)
            stream.wait_event(done_out[n - 1])
            stream.wait_event(done_in[n - 1])

        e2e_run(2)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        e2e_run(args.steps)
        e1.record(stream)
        torch.cuda.synchronize()
        e2e = {"ms": e0.elapsed_time(e1),
               "bi": xh.numel() * xh.element_size() + wh.numel() * wh.element_size(),
               "bo": yh[0].numel() * yh[0].element_size()}

    mean = lambda v: statistics.mean(v) if v else 0.0   # noqa: E731
    vals = max_over_ranks([total_ms, mean(gemm_ms), mean(fwd_ms), e2e["ms"] if e2e else 0.0,
                           mean(fused_ms), mean(single_ms), mean(had_ms)], world, dev)
    total_ms, gemm_avg_ms, fwd_avg_ms, e2e_ms, fused_avg_ms, single_avg_ms, had_avg_ms = vals

    line = None
    if rank == 0:
        sm_mhz = (clocks or {}).get("sm_mhz") or 1965.0
        mma_peak = mma_rate_tops(num_sms(dev), sm_mhz)
        ops = wl.exec_ops
        gemm_tops = ops / (gemm_avg_ms * 1e-3) / 1e12
        byts = codes_gemm_bytes(wl, args.path) if L.codes else wl.alg_bytes()
        line = {
            "metric": METRIC, "value": whole_job_tops(world, args.steps, ops, total_ms),
            "unit": "TOPS", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": total_ms / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "int8", "data": "synthetic",
            "config": config_of(wl, "flushed (256 MiB write + 256 MiB read between steps)",
                                args.path, world),
            "roofline": {
                "bound": "tensor", "kernel": gemm_kernel_name(args.path, wl.bits, wl.x_dtype),
                "achieved": gemm_tops, "peak": int8_peak, "unit": "TOPS",
                "frac": gemm_tops / int8_peak,
                "traffic": NCU_TRAFFIC_BYTES.get((wl.name, args.path)),
                "peak_source": f"{peak_kind} bf16 burst x {INT8_PER_BF16:g} (nominal int8/bf16)",
                "mma_rate_tops": mma_peak, "frac_mma_rate": gemm_tops / mma_peak,
                "mma_rate_source": (f"{MMA_I8_OPS_PER_CLK_SM} int8 ops/clk/SM (measured "
                                    f"tcgen05 kind::i8 issue rate) x {num_sms(dev)} SMs x "
                                    f"{sm_mhz:g} MHz"),
                "algorithmic_ops_per_launch": ops,
                "algorithmic_bytes_per_launch": byts,
                "achieved_gbs": byts / (gemm_avg_ms * 1e-3) / 1e9,
                "avg_launch_us": gemm_avg_ms * 1e3,
                **({"fold": fold_roofline(wl, gemm_avg_ms * 1e3, mma_peak)} if wl.bits == 4 else {}),
            },
            "forward_only": {
                "us": fwd_avg_ms * 1e3, "exec_tops": ops / (fwd_avg_ms * 1e-3) / 1e12,
                "linear_equiv_tops": ops / 2 / (fwd_avg_ms * 1e-3) / 1e12,
                "frac_int8_peak": ops / (fwd_avg_ms * 1e-3) / 1e12 / int8_peak,
            },
            "gpu_launches": L.launches_per_step * args.steps,
            "timing": ("each step: the calibration launch (+ the MAX all-reduce of the scales "
                       "over ranks), then one CUDA-graph replay of weight quantization and the "
                       "forward; CUDA events on the launching stream"),
            "clocks": clocks,
        }
        if had_ms:
            line["hadamard_forward"] = {
                "us": had_avg_ms * 1e3, "exec_tops": ops / (had_avg_ms * 1e-3) / 1e12,
                "over_dualscale_forward": had_avg_ms / fwd_avg_ms,
                "note": "block-Hadamard activations (blocks of 16): codes of XH, then the product "
                        "with the Hadamard-rotated int4 codes (rotation and its scales offline)"}
        if single_ms:
            line["single_scale_forward"] = {
                "us": single_avg_ms * 1e3,
                "exec_tops": ops / 2 / (single_avg_ms * 1e-3) / 1e12,
                "dualscale_over_single": fwd_avg_ms / single_avg_ms,
                "note": "naive baseline: one symmetric scale per K segment, its codes, then one "
                        "int8 product (half the MMA work of DualScale)"}
        if fused_ms:
            line["fused_forward"] = {
                "us": fused_avg_ms * 1e3, "exec_tops": ops / (fused_avg_ms * 1e-3) / 1e12,
                "frac_int8_peak": ops / (fused_avg_ms * 1e-3) / 1e12 / int8_peak,
                "note": "sq_linear_forward: activations quantized inside the GEMM"}
        if e2e:
            line["e2e"] = {"value": whole_job_tops(world, args.steps, ops, e2e_ms),
                           "unit": "TOPS", "h2d_bytes_per_step": e2e["bi"],
                           "d2h_bytes_per_step": e2e["bo"],
                           "note": "inputs copied from pinned host memory and Y copied back "
                                   "every step, around the library's calls (device pointers); "
                                   "steps pipelined over two buffer sets, copies in and out on "
                                   "their own streams"}
    del L
    torch.cuda.empty_cache()
    if rank == 0 and world == 1:
        if not args.no_configs:
            table = {}
            mma_peak = line["roofline"]["mma_rate_tops"]
            for name in CONFIG_ORDER:
                table[name] = measure_config(W.WORKLOADS[name], dev, flush, args.steps,
                                             args.warmup, int8_peak, mma_peak, hbm_peak)
                torch.cuda.empty_cache()
            line["configs"] = table
        if not args.no_small_m:
            line["small_m"] = {
                "note": "forwards at M <= 128 (median of L2-flushed graph replays; "
                        "one_pass_layers: per layer of 8 back-to-back layers with distinct "
                        "weights, which hides part of each launch); bytes = weight codes + "
                        "scales + q+/q- codes + Y; peak = the HBM copy bandwidth (measured "
                        "figure, else the fallback). (3072, 12288) streams its weight at "
                        "~4.6 TB/s in steady state, the rest of a layer being launch, "
                        "first-load latency and epilogue; (4608, 1152) is a 5.3 MB weight "
                        "whose time follows the k blocks each CTA streams, cut by sharing "
                        "each N tile's k blocks over a cluster of CTAs",
                "peak_gbs": hbm_peak,
                "cases": small_m_measure(dev, flush, args.steps, hbm_peak)}
            line["per_call_us"] = per_call_measure(dev)
            line["fused_activation"] = {
                "note": "SiLU / GELU fused into the combined-code producer (x = bf16_RN(act(z)) "
                        "never stored) against the framework's activation kernel + the "
                        "combined-code quantizer; bytes are the algorithmic traffic of each",
                "peak_gbs": hbm_peak, "cases": fused_act_measure(dev, flush, args.steps, hbm_peak)}
        if not args.no_cpu_baseline:
            from synth import workloads as W2
            x, w, b = W2.generate(wl)
            line["cpu_baseline"] = cpu_baseline(wl, x, w, b)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main(argv=None):
    argv = list(sys.argv[1:] if argv is None else argv)
    args = parse_args(argv)
    bad = check_world(args.gpus)
    if bad is not None:
        print(f"bench.py: {bad}", file=sys.stderr)
        return 2
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        # one process per GPU: start the ranks and wait for them
        cmd = relaunch_command(argv, args.gpus, free_port())
        return subprocess.run(cmd, timeout=3600).returncode
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
