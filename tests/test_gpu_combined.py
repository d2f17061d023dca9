"""Combined DualScale codes (c = q+ + q-, one byte per activation) and the GEMM
that splits them in shared memory, against the oracle, through the C ABI.

Bit-exact: the combined codes.  Outputs: bit-identical to the fused forward and
to the forward from (q+, q-) codes, and within the parity tolerance of the
oracle (fp32 within 1e-6 of the magnitude sum, bf16 within one ulp)."""
import numpy as np
import pytest
import torch

import oracle as O
from synth import workloads as W

from parity_util import Case, sample_rows

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
    dict(M=257, K=1040, N=128, kseg=[0, 128, 512, 1040], x_sigmas=[1.0, 3.0, 0.5], x_dtype="bf16",
         out="f32"),
    dict(M=390, K=768, N=656, kseg=[0, 768], x_dtype="bf16", out="bf16"),
]


def _case(i):
    p = dict(CASES[i])
    return W.small_case(p.pop("M"), p.pop("K"), p.pop("N"), seed=60 + i, **p)


def _bits(y):
    return y.view(torch.int16) if y.dtype == torch.bfloat16 else y.view(torch.int32)


@pytest.mark.parametrize("i", range(len(CASES)))
def test_combined_codes_bit_exact(i):
    import post_quantized_linear_b200 as pq
    c = Case(_case(i))
    code = pq.quantize_activations_combined(c.x, c.wl.kseg, c.sp, c.sn)
    ref = O.quantize_activations_combined(c.x_np, c.wl.kseg, c.o_sp, c.o_sn)
    np.testing.assert_array_equal(code.cpu().numpy(), ref)


@pytest.mark.parametrize("bn", ["128", "192", "256"])
@pytest.mark.parametrize("i", range(len(CASES)))
def test_forward_from_combined_matches_oracle_and_fused(i, bn, monkeypatch, dev_lib):
    import post_quantized_linear_b200 as pq
    monkeypatch.setenv("SEGQUANT_BN", bn)
    c = Case(_case(i))
    code = pq.quantize_activations_combined(c.x, c.wl.kseg, c.sp, c.sn)
    y = pq.linear_from_combined(code, c.qw, c.sp, c.sn, c.b, out_dtype=c.out_dtype)
    torch.cuda.synchronize()
    assert pq.stream_status() == 0
    c.compare_rows(y, np.arange(c.wl.M))
    assert torch.equal(_bits(y), _bits(c.forward()))


def test_combined_strided_codes_and_output():
    """Row strides larger than K for the codes and for Y."""
    import post_quantized_linear_b200 as pq
    wl = W.small_case(200, 384, 160, seed=70, out="bf16")
    c = Case(wl)
    buf = torch.zeros((wl.M, 512), dtype=torch.int8, device="cuda")
    code = pq.quantize_activations_combined(c.x, wl.kseg, c.sp, c.sn, out=buf[:, :wl.K])
    ybuf = torch.full((wl.M, 208), 7.0, dtype=torch.bfloat16, device="cuda")
    y = pq.linear_from_combined(code, c.qw, c.sp, c.sn, c.b, out=ybuf[:, :wl.N])
    torch.cuda.synchronize()
    c.compare_rows(y, np.arange(wl.M))
    assert torch.all(ybuf[:, wl.N:] == 7.0)
    assert not buf[:, wl.K:].any()


def test_combined_empty_batch_is_noop():
    import post_quantized_linear_b200 as pq
    c = Case(_case(0))
    code = torch.empty((0, c.wl.K), dtype=torch.int8, device="cuda")
    y = pq.linear_from_combined(code, c.qw, c.sp, c.sn, c.b)
    torch.cuda.synchronize()
    assert y.shape == (0, c.wl.N)


def test_combined_rejects_int4_weights():
    import post_quantized_linear_b200 as pq
    wl = W.small_case(64, 256, 64, seed=71, bits=4, out="bf16")
    c = Case(wl)
    code = pq.quantize_activations_combined(c.x, wl.kseg, c.sp, c.sn)
    with pytest.raises(pq.SegQuantError):
        pq.linear_from_combined(code, c.qw, c.sp, c.sn, c.b)


def test_combined_starved_pipeline_times_out_and_context_recovers(dev_lib):
    import post_quantized_linear_b200 as pq
    from post_quantized_linear_b200 import _lib
    c = Case(_case(0))
    code = pq.quantize_activations_combined(c.x, c.wl.kseg, c.sp, c.sn)
    assert pq.stream_status() == _lib.SQ_OK
    pq.set_wait_budget(2_000_000)
    pq.debug_starve_pipeline(True)
    try:
        pq.linear_from_combined(code, c.qw, c.sp, c.sn, c.b, out_dtype=c.out_dtype)
        assert pq.stream_status() == _lib.SQ_ERR_TIMEOUT
    finally:
        pq.debug_starve_pipeline(False)
        pq.set_wait_budget(0)
    y = pq.linear_from_combined(code, c.qw, c.sp, c.sn, c.b, out_dtype=c.out_dtype)
    torch.cuda.synchronize()
    assert pq.stream_status() == _lib.SQ_OK
    c.compare_rows(y, np.arange(c.wl.M))


@pytest.mark.parametrize("name", ["dit_xl2_fc2_cfg", "seglinear_qkv", "mmdit_mlp_up"])
def test_combined_full_size_sampled_rows(name):
    """Full-size workloads in the launch configuration the benchmark times:
    sampled rows against the oracle, every row against the (q+, q-) path."""
    import post_quantized_linear_b200 as pq
    wl = W.WORKLOADS[name]
    c = Case(wl)
    code = pq.quantize_activations_combined(c.x, wl.kseg, c.sp, c.sn)
    y = pq.linear_from_combined(code, c.qw, c.sp, c.sn, c.b, out_dtype=c.out_dtype)
    qp, qn = pq.quantize_activations(c.x, wl.kseg, c.sp, c.sn)
    y2 = pq.linear_from_codes(qp, qn, c.qw, c.sp, c.sn, c.b, out_dtype=c.out_dtype)
    torch.cuda.synchronize()
    assert pq.stream_status() == 0
    assert torch.equal(_bits(y), _bits(y2))
    assert torch.equal(code, (qp.to(torch.int16) + qn.to(torch.int16)).to(torch.int8))
    c.compare_rows(y, sample_rows(wl.M, 96 if wl.N > 4096 else 160))
