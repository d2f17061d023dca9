"""Host-side checks of bench.py (no GPU): the reference arm's JSON line (the
CPU oracle on the host cores), the roofline denominators read from the
measured-peaks file, and the kernel each path times."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_reference_arm_prints_one_contract_line():
    env = dict(os.environ, OMP_NUM_THREADS="2")
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--workload", "tiny_w8a8", "--steps", "1", "--warmup", "0"],
                         capture_output=True, text=True, timeout=600, env=env, cwd=ROOT)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [l for l in res.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0 and line["unit"] == "TOPS"
    assert line["config"]["workload"] == "tiny_w8a8"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0


def test_peaks_come_from_the_measured_file():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if not os.path.exists(path):
        pytest.skip("no measured peaks on this machine")
    p = json.load(open(path))
    int8, hbm, kind = bench.peaks()
    assert kind == "measured"
    assert int8 == pytest.approx(float(p["bf16_tflops"]) * bench.INT8_PER_BF16)
    assert hbm == pytest.approx(float(p["hbm_gbs"]))


def test_timed_kernel_of_each_path():
    assert bench.gemm_kernel_name("codes", 8, "bf16") == "dualscale_gemm_codes_kernel"
    assert bench.gemm_kernel_name("codes", 4, "bf16") == "dualscale_gemm_codes_kernel"
    assert bench.gemm_kernel_name("fused", 4, "bf16") == "dualscale_gemm_kernel"
    assert bench.gemm_kernel_name("combined", 8, "bf16") == "dualscale_gemm_combined_kernel"
    assert bench.gemm_kernel_name("fused", 8, "bf16") == "dualscale_gemm_inplace_kernel"
    assert bench.gemm_kernel_name("fused", 8, "f32") == "dualscale_gemm_kernel"


def test_clock_sampler_reads_nvml(monkeypatch):
    """The sampler polls NVML (a fake module here): idle samples are dropped,
    the SM clock is the median of the busy samples, and the reasons are the
    names of the bits seen while busy."""
    import types
    fake = types.ModuleType("pynvml")
    fake.NVML_CLOCK_SM = 1
    seq = iter([(1965, 0x0), (1965, 0x4), (1800, 0x4), (300, 0x1)] * 1000)
    state = {"v": (1965, 0)}

    def clock(h, kind):
        state["v"] = next(seq)
        return state["v"][0]
    fake.nvmlInit = lambda: None
    fake.nvmlDeviceGetHandleByIndex = lambda i: "h%d" % i
    fake.nvmlDeviceGetHandleByPciBusId_v2 = lambda bus: "bus"
    fake.nvmlDeviceGetMaxClockInfo = lambda h, kind: 1965
    fake.nvmlDeviceGetClockInfo = clock
    fake.nvmlDeviceGetCurrentClocksEventReasons = lambda h: state["v"][1]
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    s = bench.ClockSampler(0, period_s=0.0005)
    s.start()
    import time
    time.sleep(0.05)
    out = s.stop()
    assert out["samples"] > 10 and out["sm_max_mhz"] == 1965
    assert out["sm_mhz"] in (1800, 1965)
    assert out["reasons"] == ["sw_power_cap"]


def test_fold_roofline_of_int4_groups():
    """w4a8: 16384 x 3072 outputs, 24 groups, five fp32 operations each; the
    fp32 lane rate of 148 SMs at 1965 MHz is 128 x 148 x 1.965e9 /s."""
    from synth import workloads as W
    wl = W.WORKLOADS["w4a8"]
    r = bench.fold_roofline(wl, 550.0, bench.mma_rate_tops(148, 1965.0))
    assert r["ops_per_launch"] == 16384 * 3072 * 24 * 5
    assert r["peak"] == pytest.approx(128 * 148 * 1.965e9 / 1e12)
    assert r["floor_us"] == pytest.approx(6039797760 / (128 * 148 * 1.965e9) * 1e6)
    assert r["frac"] == pytest.approx(6039797760 / 550e-6 / 1e12 / r["peak"])
    assert r["bound"] == "alu"
