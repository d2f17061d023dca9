"""Single-scale baseline (one symmetric scale per K segment, s = max(s+, s-)):
codes and forward against the oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle as O
from synth import workloads as W

from parity_util import Case, compare_rows_single, sample_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _setup():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import post_quantized_linear_b200 as pq  # noqa: F401  (fails loudly without the library)
    O.build()
    yield


CASES = [
    dict(M=300, K=640, N=272, kseg=[0, 256, 640], x_sigmas=[1.0, 5.0], x_dtype="bf16", out="bf16"),
    dict(M=300, K=640, N=272, kseg=[0, 256, 640], x_sigmas=[1.0, 5.0], x_dtype="bf16", out="f32"),
    dict(M=129, K=384, N=144, kseg=[0, 384], x_dtype="f32", out="f32"),
    dict(M=1, K=16, N=16, kseg=[0, 16], x_dtype="bf16", out="bf16"),
    dict(M=390, K=768, N=656, kseg=[0, 768], x_dtype="bf16", out="bf16"),
    dict(M=257, K=1040, N=128, kseg=[0, 128, 512, 1040], x_sigmas=[1.0, 3.0, 0.5], x_dtype="bf16",
         out="f32"),
]


def _case(i):
    p = dict(CASES[i])
    return W.small_case(p.pop("M"), p.pop("K"), p.pop("N"), seed=80 + i, **p)


@pytest.mark.parametrize("i", range(len(CASES)))
def test_single_codes_bit_exact(i):
    import post_quantized_linear_b200 as pq
    c = Case(_case(i))
    code = pq.quantize_activations_single(c.x, c.wl.kseg, c.sp, c.sn)
    ref = O.quantize_activations_single(c.x_np, c.wl.kseg, c.o_sp, c.o_sn)
    np.testing.assert_array_equal(code.cpu().numpy(), ref)


@pytest.mark.parametrize("bn", ["128", "192", "256"])
@pytest.mark.parametrize("i", range(len(CASES)))
def test_single_forward_matches_oracle(i, bn, monkeypatch, dev_lib):
    import post_quantized_linear_b200 as pq
    monkeypatch.setenv("SEGQUANT_BN", bn)
    c = Case(_case(i))
    code = pq.quantize_activations_single(c.x, c.wl.kseg, c.sp, c.sn)
    y = pq.linear_from_single(code, c.qw, c.sp, c.sn, c.b, out_dtype=c.out_dtype)
    torch.cuda.synchronize()
    assert pq.stream_status() == 0
    compare_rows_single(c, y, np.arange(c.wl.M))


def test_single_forward_fp32_bit_exact():
    """fp32 output follows the fixed epilogue order: bit-exact with the oracle."""
    import post_quantized_linear_b200 as pq
    c = Case(_case(1))
    code = pq.quantize_activations_single(c.x, c.wl.kseg, c.sp, c.sn)
    y = pq.linear_from_single(code, c.qw, c.sp, c.sn, c.b, out_dtype=torch.float32)
    ref = O.linear_forward_single(c.x_np, c.wl.kseg, c.o_sp, c.o_sn, c.o_wc, c.o_ws, c.b_np,
                                  out="f32")
    np.testing.assert_array_equal(y.cpu().numpy(), ref)


def test_single_starved_pipeline_times_out_and_context_recovers(dev_lib):
    import post_quantized_linear_b200 as pq
    from post_quantized_linear_b200 import _lib
    c = Case(_case(0))
    code = pq.quantize_activations_single(c.x, c.wl.kseg, c.sp, c.sn)
    assert pq.stream_status() == _lib.SQ_OK
    pq.set_wait_budget(2_000_000)
    pq.debug_starve_pipeline(True)
    try:
        pq.linear_from_single(code, c.qw, c.sp, c.sn, c.b, out_dtype=c.out_dtype)
        assert pq.stream_status() == _lib.SQ_ERR_TIMEOUT
    finally:
        pq.debug_starve_pipeline(False)
        pq.set_wait_budget(0)
    y = pq.linear_from_single(code, c.qw, c.sp, c.sn, c.b, out_dtype=c.out_dtype)
    torch.cuda.synchronize()
    assert pq.stream_status() == _lib.SQ_OK
    compare_rows_single(c, y, np.arange(c.wl.M))


@pytest.mark.parametrize("name", ["dit_xl2_fc2_cfg", "seglinear_qkv", "mmdit_mlp_up"])
def test_single_full_size_sampled_rows(name):
    import post_quantized_linear_b200 as pq
    wl = W.WORKLOADS[name]
    c = Case(wl)
    code = pq.quantize_activations_single(c.x, wl.kseg, c.sp, c.sn)
    y = pq.linear_from_single(code, c.qw, c.sp, c.sn, c.b, out_dtype=c.out_dtype)
    torch.cuda.synchronize()
    assert pq.stream_status() == 0
    rows = sample_rows(wl.M, 96 if wl.N > 4096 else 160)
    ref = O.quantize_activations_single(np.ascontiguousarray(c.x_np[rows]), wl.kseg, c.o_sp, c.o_sn)
    np.testing.assert_array_equal(code.cpu().numpy()[rows], ref)
    compare_rows_single(c, y, rows)
