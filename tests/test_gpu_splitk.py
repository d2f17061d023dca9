"""Small-M split-K forward from DualScale codes, against the oracle and the
one-pass kernel, through the C ABI."""
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


def _bits(y):
    return y.view(torch.int16) if y.dtype == torch.bfloat16 else y.view(torch.int32)


CASES = [
    dict(M=64, K=640, N=272, out="bf16"),            # ragged N tail, BN 128
    dict(M=1, K=256, N=128, out="f32"),              # one row
    dict(M=100, K=1024, N=400, out="f32"),           # ragged M inside a row group
    dict(M=128, K=3072, N=2304, out="bf16"),         # BN 256, a full row tile
    dict(M=16, K=4608, N=1152, out="bf16", x_dtype="bf16"),
    dict(M=33, K=384, N=4096, out="bf16"),           # few k blocks, many N tiles
]


def _case(i):
    p = dict(CASES[i])
    return W.small_case(p.pop("M"), p.pop("K"), p.pop("N"), seed=120 + i, bias=True, **p)


@pytest.mark.parametrize("i", range(len(CASES)))
def test_splitk_matches_oracle_and_one_pass_kernel(i):
    import post_quantized_linear_b200 as pq
    c = Case(_case(i))
    wl = c.wl
    qp, qn = pq.quantize_activations(c.x, wl.kseg, c.sp, c.sn)
    ws = pq.splitk_workspace(wl.M, wl.N, wl.K, device="cuda")
    y = pq.linear_from_codes_splitk(qp, qn, c.qw, c.sp, c.sn, ws, c.b, out_dtype=c.out_dtype)
    y1 = pq.linear_from_codes(qp, qn, c.qw, c.sp, c.sn, c.b, out_dtype=c.out_dtype)
    torch.cuda.synchronize()
    assert pq.stream_status() == 0
    c.compare_rows(y, np.arange(wl.M))
    assert torch.equal(_bits(y), _bits(y1))
    # the counters are back to zero: a second call on the same workspace agrees
    y2 = pq.linear_from_codes_splitk(qp, qn, c.qw, c.sp, c.sn, ws, c.b, out_dtype=c.out_dtype)
    torch.cuda.synchronize()
    assert torch.equal(_bits(y2), _bits(y))


def test_splitk_repeated_calls_reuse_the_workspace():
    """Three calls in a row, the last after clobbering the partial slices (only
    the counters must start at zero)."""
    import post_quantized_linear_b200 as pq
    wl = W.small_case(64, 3072, 2048, seed=130, out="bf16")
    c = Case(wl)
    qp, qn = pq.quantize_activations(c.x, wl.kseg, c.sp, c.sn)
    ws = pq.splitk_workspace(wl.M, wl.N, wl.K, device="cuda")
    ys = [pq.linear_from_codes_splitk(qp, qn, c.qw, c.sp, c.sn, ws, c.b) for _ in range(2)]
    n_tiles = (wl.N + 255) // 256
    cnt = (n_tiles * 8 * 4 + 255) // 256 * 256
    ws[cnt:].fill_(0x5A)
    ys.append(pq.linear_from_codes_splitk(qp, qn, c.qw, c.sp, c.sn, ws, c.b))
    torch.cuda.synchronize()
    assert not ws[:cnt].any()
    for y in ys[1:]:
        assert torch.equal(_bits(y), _bits(ys[0]))
    c.compare_rows(ys[0], np.arange(wl.M))


def test_splitk_rejects_large_m_and_segments():
    import post_quantized_linear_b200 as pq
    wl = W.small_case(200, 256, 128, seed=131, out="bf16")
    c = Case(wl)
    qp, qn = pq.quantize_activations(c.x, wl.kseg, c.sp, c.sn)
    ws = torch.zeros(1 << 20, dtype=torch.uint8, device="cuda")
    with pytest.raises(pq.SegQuantError):
        pq.linear_from_codes_splitk(qp, qn, c.qw, c.sp, c.sn, ws)
    wl2 = W.small_case(64, 512, 128, seed=132, kseg=[0, 256, 512], x_sigmas=[1.0, 2.0], out="bf16")
    c2 = Case(wl2)
    qp2, qn2 = pq.quantize_activations(c2.x, wl2.kseg, c2.sp, c2.sn)
    with pytest.raises(pq.SegQuantError):
        pq.linear_from_codes_splitk(qp2, qn2, c2.qw, c2.sp, c2.sn, ws)


def test_splitk_starved_pipeline_times_out_and_recovers(dev_lib):
    import post_quantized_linear_b200 as pq
    from post_quantized_linear_b200 import _lib
    wl = W.small_case(64, 1024, 512, seed=133, out="bf16")
    c = Case(wl)
    qp, qn = pq.quantize_activations(c.x, wl.kseg, c.sp, c.sn)
    ws = pq.splitk_workspace(wl.M, wl.N, wl.K, device="cuda")
    assert pq.stream_status() == _lib.SQ_OK
    pq.set_wait_budget(2_000_000)
    pq.debug_starve_pipeline(True)
    try:
        pq.linear_from_codes_splitk(qp, qn, c.qw, c.sp, c.sn, ws, c.b)
        assert pq.stream_status() == _lib.SQ_ERR_TIMEOUT
    finally:
        pq.debug_starve_pipeline(False)
        pq.set_wait_budget(0)
    ws.zero_()        # after a timeout the caller clears the workspace
    y = pq.linear_from_codes_splitk(qp, qn, c.qw, c.sp, c.sn, ws, c.b)
    torch.cuda.synchronize()
    assert pq.stream_status() == _lib.SQ_OK
    c.compare_rows(y, np.arange(wl.M))


@pytest.mark.parametrize("KN", [(3072, 12288), (4608, 1152)])
@pytest.mark.parametrize("M", [16, 64, 128])
def test_splitk_small_m_configs(M, KN):
    """The small-M configurations the benchmark measures (SiLU activations, one
    segment): every row against the one-pass kernel, sampled rows against the oracle."""
    import post_quantized_linear_b200 as pq
    K, N = KN
    wl = W.small_case(M, K, N, seed=140 + M, act="silu", out="bf16")
    c = Case(wl)
    qp, qn = pq.quantize_activations(c.x, wl.kseg, c.sp, c.sn)
    ws = pq.splitk_workspace(M, N, K, device="cuda")
    y = pq.linear_from_codes_splitk(qp, qn, c.qw, c.sp, c.sn, ws, c.b)
    y1 = pq.linear_from_codes(qp, qn, c.qw, c.sp, c.sn, c.b)
    torch.cuda.synchronize()
    assert pq.stream_status() == 0
    assert torch.equal(_bits(y), _bits(y1))
    c.compare_rows(y, sample_rows(M, 16) if M > 16 else np.arange(M))


@pytest.mark.parametrize("bn", ["32", "64", "96", "128", "-1"])
@pytest.mark.parametrize("MKN", [(100, 640, 272), (1, 384, 96), (128, 1024, 1024), (64, 3072, 12288)])
def test_small_m_narrow_tiles_match_oracle(MKN, bn, monkeypatch, dev_lib):
    """One row tile: the GEMM from codes with narrow tiles and four epilogue
    warps (forced widths, and -1 for the regular choice) against the oracle,
    and bit-identical to the fused forward; also the single-scale kernel."""
    import post_quantized_linear_b200 as pq
    from parity_util import compare_rows_single
    monkeypatch.setenv("SEGQUANT_BN_SMALL", bn)
    M, K, N = MKN
    wl = W.small_case(M, K, N, seed=150 + M, out="bf16")
    c = Case(wl)
    qp, qn = pq.quantize_activations(c.x, wl.kseg, c.sp, c.sn)
    y = pq.linear_from_codes(qp, qn, c.qw, c.sp, c.sn, c.b)
    yf = c.forward()
    c1 = pq.quantize_activations_single(c.x, wl.kseg, c.sp, c.sn)
    ys = pq.linear_from_single(c1, c.qw, c.sp, c.sn, c.b)
    torch.cuda.synchronize()
    assert pq.stream_status() == 0
    rows = np.arange(M) if M <= 16 else sample_rows(M, 24)
    c.compare_rows(y, rows)
    assert torch.equal(_bits(y), _bits(yf))
    compare_rows_single(c, ys, rows)
