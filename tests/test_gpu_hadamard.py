"""GPU-vs-oracle parity of the block-Hadamard variant (HQ-DM, "HQ-DM: Single
Hadamard Transformation-Based Quantization-Aware Training for Low-Bit
Diffusion Models", Spanish technical summary 2.1), called through the C ABI.

Bit-exact: the scales of XH, the XH codes, the rotated weight codes; outputs:
fp32 bit-exact (the fixed epilogue order) and within 1e-6 of the magnitude
sum, bf16 within one ulp."""
import numpy as np
import pytest
import torch

import oracle as O
from synth import workloads as W

from parity_util import (Case, assert_bf16_within_1ulp, assert_f32_within, bf16_bits,
                         magnitude_sum)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _setup():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import post_quantized_linear_b200 as pq  # noqa: F401  (fails loudly without the library)
    O.build()
    yield


class HCase:
    """A W4A8 workload through the Hadamard path: device results and the
    oracle's scales of XH."""

    def __init__(self, wl):
        import post_quantized_linear_b200 as pq
        self.c = c = Case(wl)
        self.wl = wl
        calib_np = c.x_np if wl.calib_rows is None else c.x_np[: wl.calib_rows]
        self.o_sp, self.o_sn = O.calibrate_hadamard(calib_np, wl.kseg)
        calib = c.x if wl.calib_rows is None else c.x[: wl.calib_rows]
        self.sp, self.sn = pq.calibrate_hadamard(calib, wl.kseg)
        self.qp, self.qn = pq.quantize_activations_hadamard(c.x, wl.kseg, self.sp, self.sn)
        self.rot = pq.rotate_weights_hadamard(c.qw)

    def forward(self):
        import post_quantized_linear_b200 as pq
        return pq.linear_from_codes_hadamard(self.qp, self.qn, self.c.qw, self.rot, self.sp,
                                             self.sn, self.c.b, out_dtype=self.c.out_dtype)

    def compare_rows(self, y_gpu, rows):
        wl, c = self.wl, self.c
        out = "f32" if wl.out == "f32" else "bf16"
        y_ref, acc, _, _ = O.linear_forward_hadamard(np.ascontiguousarray(c.x_np[rows]), wl.kseg,
                                                     self.o_sp, self.o_sn, c.o_wc, c.o_ws, c.b_np,
                                                     out=out, return_acc=True)
        g = y_gpu[torch.as_tensor(rows, device=y_gpu.device)]
        if out == "f32":
            ub, useg = O.units_of(4, wl.K, wl.kseg)
            D = magnitude_sum(acc, useg, self.o_sp * O.HADAMARD_NORM, self.o_sn * O.HADAMARD_NORM,
                              O.unit_weight_scales(4, c.o_ws), c.b_np)
            assert_f32_within(g.cpu().numpy(), y_ref, D)
            np.testing.assert_array_equal(g.cpu().numpy(), y_ref)   # fixed fp32 order
        else:
            assert_bf16_within_1ulp(bf16_bits(g), y_ref)


CASES = [
    dict(M=300, K=640, N=272, kseg=[0, 256, 640], x_sigmas=[1.0, 5.0], x_dtype="bf16", out="bf16"),
    dict(M=129, K=384, N=144, kseg=[0, 384], x_dtype="f32", out="f32"),
    dict(M=64, K=1024, N=512, kseg=[0, 1024], x_dtype="bf16", out="f32"),
    dict(M=1, K=256, N=96, kseg=[0, 256], x_dtype="bf16", out="bf16"),
    dict(M=257, K=1152, N=128, kseg=[0, 128, 640, 1152], x_sigmas=[1.0, 3.0, 0.5],
         x_dtype="bf16", out="f32"),
    dict(M=16, K=3072, N=1024, kseg=[0, 3072], x_dtype="bf16", out="bf16"),
    # several row tiles and output tiles (ragged both ways), fp32 out: bit-exact
    dict(M=300, K=1024, N=400, kseg=[0, 512, 1024], x_sigmas=[1.0, 4.0], x_dtype="bf16",
         out="f32"),
]


def _case(i):
    p = dict(CASES[i])
    return W.small_case(p.pop("M"), p.pop("K"), p.pop("N"), seed=300 + i, bits=4, **p)


@pytest.mark.parametrize("i", range(len(CASES)))
def test_hadamard_scales_codes_and_rotated_weights_bit_exact(i):
    import post_quantized_linear_b200 as pq
    h = HCase(_case(i))
    torch.cuda.synchronize()
    assert pq.stream_status() == 0
    np.testing.assert_array_equal(h.sp.cpu().numpy(), h.o_sp)
    np.testing.assert_array_equal(h.sn.cpu().numpy(), h.o_sn)
    op, on = O.quantize_activations_hadamard(h.c.x_np, h.wl.kseg, h.o_sp, h.o_sn)
    np.testing.assert_array_equal(h.qp.cpu().numpy(), op)
    np.testing.assert_array_equal(h.qn.cpu().numpy(), on)
    np.testing.assert_array_equal(h.rot.cpu().numpy(),
                                  O.rotate_weight_codes(O.unpack_w4(h.c.o_wc, h.wl.K)))


@pytest.mark.parametrize("i", range(len(CASES)))
def test_hadamard_forward_matches_oracle(i):
    import post_quantized_linear_b200 as pq
    h = HCase(_case(i))
    y = h.forward()
    torch.cuda.synchronize()
    assert pq.stream_status() == 0
    h.compare_rows(y, np.arange(h.wl.M))


def test_hadamard_full_size_every_row():
    """The W4A8 workload (M = 16384, K = N = 3072) in the bench's launch
    configuration: bit-exact scales, every XH code and the rotated weights;
    every output row against the oracle (in chunks of rows)."""
    import post_quantized_linear_b200 as pq
    h = HCase(W.WORKLOADS["w4a8"])
    y = h.forward()
    torch.cuda.synchronize()
    assert pq.stream_status() == 0
    np.testing.assert_array_equal(h.sp.cpu().numpy(), h.o_sp)
    np.testing.assert_array_equal(h.sn.cpu().numpy(), h.o_sn)
    chunk = 2048
    for r0 in range(0, h.wl.M, chunk):
        rows = np.arange(r0, min(h.wl.M, r0 + chunk))
        op, on = O.quantize_activations_hadamard(np.ascontiguousarray(h.c.x_np[rows]), h.wl.kseg,
                                                 h.o_sp, h.o_sn)
        np.testing.assert_array_equal(h.qp[r0:r0 + len(rows)].cpu().numpy(), op)
        np.testing.assert_array_equal(h.qn[r0:r0 + len(rows)].cpu().numpy(), on)
        h.compare_rows(y, rows)


def test_hadamard_starved_pipeline_times_out_and_context_recovers(dev_lib):
    import post_quantized_linear_b200 as pq
    from post_quantized_linear_b200 import _lib
    h = HCase(_case(0))
    torch.cuda.synchronize()
    assert pq.stream_status() == _lib.SQ_OK
    pq.set_wait_budget(2_000_000)
    pq.debug_starve_pipeline(True)
    try:
        h.forward()
        assert pq.stream_status() == _lib.SQ_ERR_TIMEOUT
    finally:
        pq.debug_starve_pipeline(False)
        pq.set_wait_budget(0)
    y = h.forward()
    torch.cuda.synchronize()
    assert pq.stream_status() == _lib.SQ_OK
    h.compare_rows(y, np.arange(h.wl.M))
