"""Shared helpers of the GPU-vs-oracle parity tests.

Tolerances (from the workload specification, applied as written):
  * codes, scales and int32 accumulators: bit-exact;
  * fp32 outputs: |y_gpu - y_oracle| <= 1e-6 * D, where D is the magnitude sum
    sum_u |sw_u| (|s+ F(acc+_u)| + |s- F(acc-_u)|) + |b| (a relative bound on
    the terms avoids a blow-up when they cancel);
  * bf16 outputs: within one bf16 ulp of the oracle's bf16 value.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle as O
from synth import workloads as W


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def bf16_ulp(vals: np.ndarray) -> np.ndarray:
    """Spacing of bf16 numbers at |vals| (8 significant bits)."""
    a = np.abs(vals)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, -126)
    return np.where(a > 0, 2.0 ** (e - 7), 2.0 ** -133)


def assert_bf16_within_1ulp(got_bits: np.ndarray, ref_bits: np.ndarray):
    g = bf16_to_f64(got_bits)
    r = bf16_to_f64(ref_bits)
    bad = np.abs(g - r) > bf16_ulp(r) * (1 + 1e-12)
    if bad.any():
        idx = np.argwhere(bad)[:5]
        raise AssertionError(f"{int(bad.sum())} bf16 outputs beyond 1 ulp, e.g. {idx.tolist()}: "
                             f"got {g[tuple(idx[0])]} ref {r[tuple(idx[0])]}")


def magnitude_sum(acc, unit_seg, s_pos, s_neg, unit_scales, bias):
    acc = acc.astype(np.float64)
    D = np.zeros(acc.shape[2:])
    for u in range(acc.shape[0]):
        j = unit_seg[u]
        D += np.abs(unit_scales[u].astype(np.float64))[None, :] * (
            np.abs(np.float64(s_pos[j]) * acc[u, 0]) + np.abs(np.float64(s_neg[j]) * acc[u, 1]))
    if bias is not None:
        D += np.abs(bias.astype(np.float64))[None, :]
    return D


def assert_f32_within(got: np.ndarray, ref: np.ndarray, D: np.ndarray, rel: float = 1e-6):
    err = np.abs(got.astype(np.float64) - ref.astype(np.float64))
    bad = err > rel * D + 1e-37
    if bad.any():
        i = tuple(np.argwhere(bad)[0])
        raise AssertionError(f"{int(bad.sum())} fp32 outputs beyond {rel}*D, e.g. {i}: "
                             f"got {got[i]} ref {ref[i]} D {D[i]}")


class Case:
    """Inputs of one workload on host and device, the oracle's scales and
    weights, and the GPU path's results."""

    def __init__(self, wl: W.Workload, device="cuda"):
        import post_quantized_linear_b200 as pq
        self.wl = wl
        x, w, b = W.generate(wl)
        self.x_cpu, self.w_cpu, self.b_cpu = x, w, b
        self.x_np = W.to_numpy_x(x)
        self.w_np = w.numpy()
        self.b_np = None if b is None else b.numpy()
        calib_np = self.x_np if wl.calib_rows is None else self.x_np[: wl.calib_rows]
        self.o_sp, self.o_sn = O.calibrate(calib_np, wl.kseg)
        if wl.bits == 8:
            self.o_wc, self.o_ws = O.quantize_weights_w8(self.w_np, wl.kseg)
        else:
            self.o_wc, self.o_ws = O.quantize_weights_w4(self.w_np)
        # device
        self.x = x.to(device)
        self.w = w.to(device)
        self.b = None if b is None else b.to(device)
        calib = self.x if wl.calib_rows is None else self.x[: wl.calib_rows]
        self.sp, self.sn = pq.calibrate(calib, wl.kseg)
        self.qw = pq.quantize_weights(self.w, wl.kseg, wl.nseg, bits=wl.bits)
        self.out_dtype = torch.float32 if wl.out == "f32" else torch.bfloat16

    def check_scales_and_weights(self):
        import post_quantized_linear_b200 as pq
        torch.cuda.synchronize()
        assert pq.stream_status() == 0
        np.testing.assert_array_equal(self.sp.cpu().numpy(), self.o_sp)
        np.testing.assert_array_equal(self.sn.cpu().numpy(), self.o_sn)
        if self.wl.bits == 8:
            np.testing.assert_array_equal(self.qw.codes.cpu().numpy(), self.o_wc)
            np.testing.assert_array_equal(self.qw.scales.cpu().numpy(), self.o_ws)
        else:
            np.testing.assert_array_equal(self.qw.codes.cpu().numpy(), self.o_wc)
            np.testing.assert_array_equal(self.qw.scales.cpu().numpy().view(np.uint16),
                                          self.o_ws.view(np.uint16))

    def forward(self):
        import post_quantized_linear_b200 as pq
        return pq.linear(self.x, self.qw, self.sp, self.sn, self.b, out_dtype=self.out_dtype)

    def oracle_rows(self, rows: np.ndarray):
        """Oracle forward of the given rows, with the oracle's own scales/weights."""
        xr = np.ascontiguousarray(self.x_np[rows])
        out = "f32" if self.wl.out == "f32" else "bf16"
        y, acc, _ = O.linear_forward(xr, self.wl.kseg, self.o_sp, self.o_sn, self.wl.bits,
                                     self.o_wc, self.o_ws, self.b_np, out=out, return_acc=True)
        return y, acc

    def compare_rows(self, y_gpu: torch.Tensor, rows: np.ndarray):
        y_ref, acc = self.oracle_rows(rows)
        g = y_gpu[torch.as_tensor(rows, device=y_gpu.device)]
        if self.wl.out == "f32":
            ub, useg = O.units_of(self.wl.bits, self.wl.K, self.wl.kseg)
            D = magnitude_sum(acc, useg, self.o_sp, self.o_sn,
                              O.unit_weight_scales(self.wl.bits, self.o_ws), self.b_np)
            assert_f32_within(g.cpu().numpy(), y_ref, D)
        else:
            assert_bf16_within_1ulp(bf16_bits(g), y_ref)
        return y_ref, acc


def compare_rows_single(case: "Case", y_gpu: torch.Tensor, rows: np.ndarray):
    """The single-scale baseline's rows against the oracle (same tolerances)."""
    wl = case.wl
    xr = np.ascontiguousarray(case.x_np[rows])
    out = "f32" if wl.out == "f32" else "bf16"
    y_ref, acc, _ = O.linear_forward_single(xr, wl.kseg, case.o_sp, case.o_sn, case.o_wc,
                                            case.o_ws, case.b_np, out=out, return_acc=True)
    g = y_gpu[torch.as_tensor(rows, device=y_gpu.device)]
    if wl.out == "f32":
        ub, useg = O.units_of(8, wl.K, wl.kseg)
        s = np.maximum(case.o_sp, case.o_sn)
        acc2 = np.stack([acc, np.zeros_like(acc)], axis=1)
        D = magnitude_sum(acc2, useg, s, s, O.unit_weight_scales(8, case.o_ws), case.b_np)
        assert_f32_within(g.cpu().numpy(), y_ref, D)
    else:
        assert_bf16_within_1ulp(bf16_bits(g), y_ref)
    return y_ref, acc


def sample_rows(M: int, n: int, seed: int = 0) -> np.ndarray:
    """First and last tile rows, tile edges and a random spread."""
    fixed = [0, 1, 31, 32, 63, 64, 127, 128, M - 1, M - 2, M - 128, M - 129]
    rng = np.random.default_rng(seed)
    rest = rng.choice(M, size=max(0, n - len(fixed)), replace=False)
    rows = np.unique(np.clip(np.concatenate([fixed, rest]), 0, M - 1))
    return rows.astype(np.int64)
