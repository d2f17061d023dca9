"""GPU-vs-oracle parity of every step of the path, called through the C ABI.

Bit-exact: calibration scales, weight codes and scales, DualScale activation
codes, int32 accumulators.  Outputs: fp32 within 1e-6 of the magnitude sum,
bf16 within one ulp (see tests/parity_util.py)."""
import numpy as np
import pytest
import torch

import oracle as O
from synth import workloads as W

from parity_util import (Case, assert_bf16_within_1ulp, assert_f32_within, bf16_bits,
                         magnitude_sum, sample_rows)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _setup():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import post_quantized_linear_b200 as pq  # noqa: F401  (fails loudly without the library)
    O.build()
    yield


# Small shapes that span several tiles in M, N and K with ragged tails.
SMALL = [
    dict(M=300, K=640, N=272, kseg=[0, 256, 640], x_sigmas=[1.0, 5.0], x_dtype="bf16", out="bf16"),
    dict(M=300, K=640, N=272, kseg=[0, 256, 640], x_sigmas=[1.0, 5.0], x_dtype="bf16", out="f32"),
    dict(M=129, K=384, N=144, kseg=[0, 384], x_dtype="f32", out="f32"),
    dict(M=64, K=256, N=256, kseg=[0, 256], x_dtype="f32", out="bf16"),
    dict(M=1, K=16, N=16, kseg=[0, 16], x_dtype="bf16", out="bf16"),
    dict(M=257, K=1040, N=128, kseg=[0, 128, 512, 1040], x_sigmas=[1.0, 3.0, 0.5], x_dtype="bf16",
         out="f32"),
    # int4 weights (group 128): several groups, K segments, ragged M and N
    dict(M=300, K=640, N=272, kseg=[0, 256, 640], x_sigmas=[1.0, 5.0], x_dtype="bf16", out="bf16",
         bits=4),
    dict(M=129, K=384, N=144, kseg=[0, 384], x_dtype="f32", out="f32", bits=4),
    dict(M=200, K=1024, N=400, kseg=[0, 1024], x_dtype="bf16", out="f32", bits=4),
]


def _small(i, **over):
    p = dict(SMALL[i])
    p.update(over)
    return W.small_case(p.pop("M"), p.pop("K"), p.pop("N"), seed=10 + i, **p)


@pytest.mark.parametrize("i", range(len(SMALL)))
def test_scales_and_weights_bit_exact(i):
    c = Case(_small(i))
    c.check_scales_and_weights()


@pytest.mark.parametrize("i", range(len(SMALL)))
def test_activation_codes_bit_exact(i):
    import post_quantized_linear_b200 as pq
    c = Case(_small(i))
    qp, qn = pq.quantize_activations(c.x, c.wl.kseg, c.sp, c.sn)
    op, on = O.quantize_activations(c.x_np, c.wl.kseg, c.o_sp, c.o_sn)
    np.testing.assert_array_equal(qp.cpu().numpy(), op)
    np.testing.assert_array_equal(qn.cpu().numpy(), on)


@pytest.mark.parametrize("i", range(len(SMALL)))
def test_accumulators_bit_exact(i):
    import post_quantized_linear_b200 as pq
    c = Case(_small(i))
    acc = pq.linear_accumulators(c.x, c.qw, c.sp, c.sn)
    _, o_acc = c.oracle_rows(np.arange(c.wl.M))
    np.testing.assert_array_equal(acc.cpu().numpy(), o_acc)


@pytest.mark.parametrize("i", range(len(SMALL)))
def test_forward_matches_oracle(i):
    c = Case(_small(i))
    c.check_scales_and_weights()
    y = c.forward()
    torch.cuda.synchronize()
    c.compare_rows(y, np.arange(c.wl.M))


@pytest.mark.parametrize("i", range(len(SMALL)))
def test_forward_from_codes_equals_fused(i):
    """Pre-quantized codes through TMA give the same bits as the fused quantizer."""
    import post_quantized_linear_b200 as pq
    c = Case(_small(i))
    y = c.forward()
    qp, qn = pq.quantize_activations(c.x, c.wl.kseg, c.sp, c.sn)
    y2 = pq.linear_from_codes(qp, qn, c.qw, c.sp, c.sn, c.b, out_dtype=c.out_dtype)
    assert torch.equal(y.view(torch.int16) if y.dtype == torch.bfloat16 else y.view(torch.int32),
                       y2.view(torch.int16) if y2.dtype == torch.bfloat16 else y2.view(torch.int32))


@pytest.mark.parametrize("bn", ["128", "192", "256"])
@pytest.mark.parametrize("codes", [False, True])
def test_tile_width_variants_match_oracle(bn, codes, monkeypatch, dev_lib):
    """Both output-tile widths (BN = 128 double-buffered TMEM, BN = 256 single
    buffer with the streaming epilogue), fused and from codes, on ragged shapes."""
    import post_quantized_linear_b200 as pq
    monkeypatch.setenv("SEGQUANT_BN", bn)
    wl = W.small_case(390, 768, 656, seed=21, out="bf16")
    c = Case(wl)
    if codes:
        qp, qn = pq.quantize_activations(c.x, wl.kseg, c.sp, c.sn)
        y = pq.linear_from_codes(qp, qn, c.qw, c.sp, c.sn, c.b)
    else:
        y = c.forward()
    torch.cuda.synchronize()
    c.compare_rows(y, np.arange(wl.M))


@pytest.mark.parametrize("N", [304, 336])
def test_narrow_tail_of_the_halved_buffer(N, monkeypatch, dev_lib):
    """BN = 256 from codes, where the one TMEM buffer goes back to the MMA in
    halves: a last tile column of 48 or 80 columns leaves some epilogue warps
    without columns (they hand both halves back at once) and the MMA fills
    only the first half; every row against the oracle."""
    import post_quantized_linear_b200 as pq
    monkeypatch.setenv("SEGQUANT_BN", "256")
    wl = W.small_case(390, 768, N, seed=23, out="bf16")
    c = Case(wl)
    qp, qn = pq.quantize_activations(c.x, wl.kseg, c.sp, c.sn)
    y = pq.linear_from_codes(qp, qn, c.qw, c.sp, c.sn, c.b)
    torch.cuda.synchronize()
    assert pq.stream_status() == 0
    c.compare_rows(y, np.arange(wl.M))


@pytest.mark.parametrize("bn", ["128", "192", "256"])
@pytest.mark.parametrize("i", [0, 1, 2, 5])
def test_codes_kernels_one_ring_and_two_rings_agree(i, bn, monkeypatch, dev_lib):
    """The GEMM from codes with one ring of stages (codes and weights in one
    stage) and with separate operand rings: the oracle's result, bit-identical
    to each other, on one and several K segments, bf16 and fp32 outputs."""
    import post_quantized_linear_b200 as pq
    monkeypatch.setenv("SEGQUANT_BN", bn)
    c = Case(_small(i))
    qp, qn = pq.quantize_activations(c.x, c.wl.kseg, c.sp, c.sn)
    monkeypatch.setenv("SEGQUANT_CODES_RING", "1")
    y1 = pq.linear_from_codes(qp, qn, c.qw, c.sp, c.sn, c.b, out_dtype=c.out_dtype)
    monkeypatch.setenv("SEGQUANT_CODES_RING", "0")
    y0 = pq.linear_from_codes(qp, qn, c.qw, c.sp, c.sn, c.b, out_dtype=c.out_dtype)
    torch.cuda.synchronize()
    assert pq.stream_status() == 0
    c.compare_rows(y1, np.arange(c.wl.M))
    iv = torch.int16 if y1.dtype == torch.bfloat16 else torch.int32
    assert torch.equal(y1.view(iv), y0.view(iv))


@pytest.mark.parametrize("bn", ["128", "192", "256"])
@pytest.mark.parametrize("MKN", [(390, 768, 656), (300, 640, 272), (64, 1024, 512), (1, 256, 96),
                                 (300, 640, 272, (0, 256, 640))])
def test_code_tiles_by_cp_async_or_tma_agree(MKN, bn, monkeypatch, dev_lib):
    """The GEMM from codes with the code tiles copied by cp.async loader warps
    and with every operand loaded by TMA: the oracle's result, identical bits,
    DualScale and single-scale, ragged M, N and K tails, one and two K segments."""
    import post_quantized_linear_b200 as pq
    from parity_util import compare_rows_single
    monkeypatch.setenv("SEGQUANT_BN", bn)
    M, K, N = MKN[:3]
    kseg = list(MKN[3]) if len(MKN) > 3 else None
    c = Case(W.small_case(M, K, N, seed=90 + M, out="bf16", kseg=kseg,
                          x_sigmas=[1.0, 4.0] if kseg else None))
    qp, qn = pq.quantize_activations(c.x, c.wl.kseg, c.sp, c.sn)
    c1 = pq.quantize_activations_single(c.x, c.wl.kseg, c.sp, c.sn)
    ys = {}
    for lda in ("1", "0"):
        monkeypatch.setenv("SEGQUANT_CODES_LDA", lda)
        ys[lda] = (pq.linear_from_codes(qp, qn, c.qw, c.sp, c.sn, c.b),
                   pq.linear_from_single(c1, c.qw, c.sp, c.sn, c.b))
    torch.cuda.synchronize()
    assert pq.stream_status() == 0
    c.compare_rows(ys["1"][0], np.arange(M))
    compare_rows_single(c, ys["1"][1], np.arange(M))
    for i in range(2):
        assert torch.equal(ys["1"][i].view(torch.int16), ys["0"][i].view(torch.int16))


@pytest.mark.parametrize("bn", ["128", "192"])
@pytest.mark.parametrize("MKN", [(390, 640, 656), (300, 1040, 272), (129, 768, 400), (64, 3072, 1024),
                                 (300, 640, 272, (0, 256, 640)),
                                 (257, 1040, 256, (0, 128, 512, 1040))])
def test_two_k_blocks_per_stage_agree(MKN, bn, monkeypatch, dev_lib):
    """The GEMM from codes with two k blocks per pipeline stage (one commit per
    stage; odd k-block counts end in a half stage; K tails; K segments that
    begin or end inside a stage) against the oracle and bit-identical to one k
    block per stage, DualScale and single-scale."""
    import post_quantized_linear_b200 as pq
    from parity_util import compare_rows_single
    monkeypatch.setenv("SEGQUANT_BN", bn)
    M, K, N = MKN[:3]
    kseg = list(MKN[3]) if len(MKN) > 3 else None
    sig = [1.0 + 2.0 * j for j in range(len(kseg) - 1)] if kseg else None
    c = Case(W.small_case(M, K, N, seed=110 + M, out="bf16", kseg=kseg, x_sigmas=sig))
    qp, qn = pq.quantize_activations(c.x, c.wl.kseg, c.sp, c.sn)
    c1 = pq.quantize_activations_single(c.x, c.wl.kseg, c.sp, c.sn)
    ys = {}
    for kps in ("2", "1"):
        monkeypatch.setenv("SEGQUANT_KPS", kps)
        ys[kps] = (pq.linear_from_codes(qp, qn, c.qw, c.sp, c.sn, c.b),
                   pq.linear_from_single(c1, c.qw, c.sp, c.sn, c.b))
    torch.cuda.synchronize()
    assert pq.stream_status() == 0
    c.compare_rows(ys["2"][0], np.arange(M))
    compare_rows_single(c, ys["2"][1], np.arange(M))
    for i in range(2):
        assert torch.equal(ys["2"][i].view(torch.int16), ys["1"][i].view(torch.int16))


@pytest.mark.parametrize("out", ["bf16", "f32"])
def test_wide_tiles_with_sixteen_epilogue_warps_agree(out, monkeypatch, dev_lib):
    """256-wide tiles drained by 16 epilogue warps: the oracle's result and the
    same bits as with 8 warps (ragged M, N tail)."""
    import post_quantized_linear_b200 as pq
    monkeypatch.setenv("SEGQUANT_BN", "256")
    c = Case(W.small_case(390, 768, 656, seed=77, out=out))
    qp, qn = pq.quantize_activations(c.x, c.wl.kseg, c.sp, c.sn)
    ys = {}
    for e in ("1", "0"):
        monkeypatch.setenv("SEGQUANT_EPW16", e)
        ys[e] = pq.linear_from_codes(qp, qn, c.qw, c.sp, c.sn, c.b, out_dtype=c.out_dtype)
    torch.cuda.synchronize()
    assert pq.stream_status() == 0
    c.compare_rows(ys["1"], np.arange(c.wl.M))
    iv = torch.int16 if out == "bf16" else torch.int32
    assert torch.equal(ys["1"].view(iv), ys["0"].view(iv))


@pytest.mark.parametrize("out", ["bf16", "f32"])
@pytest.mark.parametrize("MKN", [(300, 640, 272, (0, 256, 640)), (129, 384, 144), (200, 1024, 400),
                                 (64, 3072, 1024), (1, 256, 96), (16, 1024, 272, (0, 512, 1024)),
                                 (257, 1152, 128, (0, 128, 640, 1152))])
def test_int4_codes_kernel_and_operand_ring_kernel_agree(MKN, out, monkeypatch, dev_lib):
    """int4 weights (group 128) through the GEMM from codes (unpack warps, one
    ring of stages, seeded accumulators) and through the operand-ring kernel:
    the oracle's result on every row and identical bits; ragged M and N tails,
    one to three K segments, short row tiles."""
    import post_quantized_linear_b200 as pq
    M, K, N = MKN[:3]
    kseg = list(MKN[3]) if len(MKN) > 3 else None
    sig = [1.0, 4.0, 0.5][: len(kseg) - 1] if kseg else None
    c = Case(W.small_case(M, K, N, seed=200 + M, bits=4, out=out, kseg=kseg, x_sigmas=sig))
    qp, qn = pq.quantize_activations(c.x, c.wl.kseg, c.sp, c.sn)
    ys = {}
    for v in ("1", "0"):
        monkeypatch.setenv("SEGQUANT_W4_CODES", v)
        ys[v] = pq.linear_from_codes(qp, qn, c.qw, c.sp, c.sn, c.b, out_dtype=c.out_dtype)
    torch.cuda.synchronize()
    assert pq.stream_status() == 0
    c.compare_rows(ys["1"], np.arange(M))
    iv = torch.int16 if out == "bf16" else torch.int32
    assert torch.equal(ys["1"].view(iv), ys["0"].view(iv))


@pytest.mark.parametrize("kseg", [None, (0, 256, 640)])
@pytest.mark.parametrize("M", [1, 17, 48, 100, 127])
def test_code_boxes_sized_to_a_short_row_tile(M, kseg, monkeypatch, dev_lib):
    """Fewer than 128 rows: the GEMM from codes loads code boxes of M rows
    rounded up to 16 and the MMA's other rows read stale shared memory.  Every
    row against the oracle (DualScale and single-scale, one and two K
    segments), and the same bits as the fused forward (which quantizes from X)
    at every narrow tile width."""
    import post_quantized_linear_b200 as pq
    from parity_util import compare_rows_single
    K = 640 if kseg else 1024
    c = Case(W.small_case(M, K, 272, seed=170 + M, out="bf16", kseg=list(kseg) if kseg else None,
                          x_sigmas=[1.0, 4.0] if kseg else None))
    qp, qn = pq.quantize_activations(c.x, c.wl.kseg, c.sp, c.sn)
    c1 = pq.quantize_activations_single(c.x, c.wl.kseg, c.sp, c.sn)
    yf = c.forward()
    res = {}
    for bn in ("32", "96", "-1"):
        monkeypatch.setenv("SEGQUANT_BN_SMALL", bn)
        res[bn] = (pq.linear_from_codes(qp, qn, c.qw, c.sp, c.sn, c.b),
                   pq.linear_from_single(c1, c.qw, c.sp, c.sn, c.b))
    torch.cuda.synchronize()
    assert pq.stream_status() == 0
    y, ys = res["-1"]
    c.compare_rows(y, np.arange(M))
    compare_rows_single(c, ys, np.arange(M))
    assert torch.equal(y.view(torch.int16), yf.view(torch.int16))
    for (yd, yds) in res.values():
        assert torch.equal(yd.view(torch.int16), y.view(torch.int16))
        assert torch.equal(yds.view(torch.int16), ys.view(torch.int16))


def test_forward_exact_in_fp32():
    """With the fp32 epilogue order the kernel reproduces the oracle bit for bit."""
    c = Case(_small(1))
    y = c.forward().cpu().numpy()
    y_ref, _ = c.oracle_rows(np.arange(c.wl.M))
    np.testing.assert_array_equal(y, y_ref)


@pytest.mark.parametrize("i", [7, 8])
def test_int4_forward_exact_in_fp32(i):
    """int4 weights (one unit per 128-wide group, seeded accumulators) with
    fp32 outputs on several row and output tiles: the fused forward and the
    GEMM from codes reproduce the oracle bit for bit (the fixed fp32 order)."""
    import post_quantized_linear_b200 as pq
    c = Case(_small(i))
    assert c.wl.bits == 4 and c.wl.out == "f32"
    y = c.forward()
    qp, qn = pq.quantize_activations(c.x, c.wl.kseg, c.sp, c.sn)
    y2 = pq.linear_from_codes(qp, qn, c.qw, c.sp, c.sn, c.b, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert pq.stream_status() == 0
    y_ref, _ = c.oracle_rows(np.arange(c.wl.M))
    np.testing.assert_array_equal(y.cpu().numpy(), y_ref)
    np.testing.assert_array_equal(y2.cpu().numpy(), y_ref)


def test_nonnegative_input_and_zero_rows():
    import post_quantized_linear_b200 as pq
    wl = W.small_case(200, 256, 128, seed=3, act="none", bias=True, out="f32")
    x, w, b = W.generate(wl)
    x = x.abs().to(torch.float32)
    x[5] = 0.0
    xd, wd, bd = x.cuda().to(torch.bfloat16), w.cuda(), b.cuda()
    sp, sn = pq.calibrate(xd, wl.kseg)
    assert float(sn[0]) == 0.0
    qw = pq.quantize_weights(wd, wl.kseg)
    acc = pq.linear_accumulators(xd, qw, sp, sn)
    assert int(acc[:, 1].abs().max()) == 0
    y = pq.linear(xd, qw, sp, sn, bd, out_dtype=torch.float32)
    np.testing.assert_array_equal(y[5].cpu().numpy(), b.numpy())


def test_empty_batch_is_noop():
    import post_quantized_linear_b200 as pq
    c = Case(_small(3))
    x0 = c.x[:0]
    y = pq.linear(x0, c.qw, c.sp, c.sn, c.b, out_dtype=torch.float32)
    assert y.shape == (0, c.wl.N)


def test_output_segments_are_a_noop():
    """Quantizing and running q | k | v separately equals the fused N = 3 x 1152 layer."""
    import post_quantized_linear_b200 as pq
    wl = W.small_case(256, 512, 384, seed=4, kseg=[0, 256, 512], x_sigmas=[1.0, 5.0], out="bf16")
    x, w, _ = W.generate(wl)
    w[128:256] *= 2.5
    xd, wd = x.cuda(), w.cuda()
    sp, sn = pq.calibrate(xd, wl.kseg)
    full = pq.quantize_weights(wd, wl.kseg, (0, 128, 256, 384))
    y = pq.linear(xd, full, sp, sn)
    for n0, n1 in [(0, 128), (128, 256), (256, 384)]:
        part = pq.quantize_weights(wd[n0:n1].contiguous(), wl.kseg)
        assert torch.equal(part.codes, full.codes[n0:n1])
        assert torch.equal(part.scales, full.scales[:, n0:n1])
        assert torch.equal(pq.linear(xd, part, sp, sn), y[:, n0:n1])


def test_strided_activations_and_outputs():
    import post_quantized_linear_b200 as pq
    c = Case(_small(0))
    big = torch.zeros((c.wl.M, c.wl.K + 64), dtype=c.x.dtype, device="cuda")
    big[:, 16:16 + c.wl.K] = c.x
    xs = big[:, 16:16 + c.wl.K]
    ybig = torch.zeros((c.wl.M, c.wl.N + 32), dtype=torch.bfloat16, device="cuda")
    ys = ybig[:, 8:8 + c.wl.N]
    pq.linear(xs, c.qw, c.sp, c.sn, c.b, out=ys)
    assert torch.equal(ys, c.forward())
    assert int(ybig[:, :8].abs().sum()) == 0


@pytest.mark.parametrize("name", ["tiny_w8a8", "dit_xl2_fc2_cfg", "seglinear_qkv", "mmdit_mlp_up",
                                  "w4a8"])
def test_workloads_full_size_every_row(name):
    """Full-size workloads in the bench's launch configuration: bit-exact
    scales, weights and every DualScale code; every output row of the fused
    forward against the oracle (rows in chunks, so host memory stays bounded);
    the two-pass path (codes, then the GEMM from codes) bit-identical to it."""
    import post_quantized_linear_b200 as pq
    wl = W.WORKLOADS[name]
    c = Case(wl)
    c.check_scales_and_weights()
    y = c.forward()
    qp, qn = pq.quantize_activations(c.x, wl.kseg, c.sp, c.sn)
    y2 = pq.linear_from_codes(qp, qn, c.qw, c.sp, c.sn, c.b, out_dtype=c.out_dtype)
    torch.cuda.synchronize()
    assert pq.stream_status() == 0
    iv = torch.int16 if y.dtype == torch.bfloat16 else torch.int32
    assert torch.equal(y.view(iv), y2.view(iv))
    chunk = 2048
    for r0 in range(0, wl.M, chunk):
        rows = np.arange(r0, min(wl.M, r0 + chunk))
        op, on = O.quantize_activations(np.ascontiguousarray(c.x_np[rows]), wl.kseg, c.o_sp, c.o_sn)
        np.testing.assert_array_equal(qp[r0:r0 + len(rows)].cpu().numpy(), op)
        np.testing.assert_array_equal(qn[r0:r0 + len(rows)].cpu().numpy(), on)
        c.compare_rows(y, rows)


# ------------------------------------------------------------- status word
def test_calibration_non_finite_sets_range_status():
    import post_quantized_linear_b200 as pq
    from post_quantized_linear_b200 import _lib
    x = torch.randn(64, 256, device="cuda", dtype=torch.bfloat16)
    x[3, 17] = float("inf")
    pq.calibrate(x, [0, 256])
    assert pq.stream_status() == _lib.SQ_ERR_RANGE
    assert pq.stream_status() == _lib.SQ_OK          # the word is cleared by reading it
    x[3, 17] = float("nan")
    pq.calibrate(x, [0, 128, 256])
    assert pq.stream_status() == _lib.SQ_ERR_RANGE


def test_weight_quantization_range_status():
    import post_quantized_linear_b200 as pq
    from post_quantized_linear_b200 import _lib
    w = torch.randn(32, 256, device="cuda") * 0.02
    w[5, 9] = float("nan")
    pq.quantize_weights(w, [0, 256], bits=8)
    assert pq.stream_status() == _lib.SQ_ERR_RANGE
    w[5, 9] = 1.0e6                                  # 1e6 / 7 overflows binary16
    pq.quantize_weights(w, [0, 256], bits=4)
    assert pq.stream_status() == _lib.SQ_ERR_RANGE
    w[5, 9] = 0.01
    pq.quantize_weights(w, [0, 256], bits=4)
    assert pq.stream_status() == _lib.SQ_OK


@pytest.mark.parametrize("codes,i", [(False, 0), (True, 0), (True, 6)])
def test_starved_pipeline_times_out_and_context_recovers(codes, i, dev_lib):
    """Bounded waits: with the producer starved every wait expires; the kernel
    records SQ_ERR_TIMEOUT, frees its TMEM and exits, and the next launch on the
    same context is correct again (int8 and int4 weights)."""
    import post_quantized_linear_b200 as pq
    from post_quantized_linear_b200 import _lib
    c = Case(_small(i))
    qp, qn = pq.quantize_activations(c.x, c.wl.kseg, c.sp, c.sn)
    assert pq.stream_status() == _lib.SQ_OK
    pq.set_wait_budget(2_000_000)                   # about a millisecond
    pq.debug_starve_pipeline(True)
    try:
        if codes:
            pq.linear_from_codes(qp, qn, c.qw, c.sp, c.sn, c.b, out_dtype=c.out_dtype)
        else:
            c.forward()
        assert pq.stream_status() == _lib.SQ_ERR_TIMEOUT
    finally:
        pq.debug_starve_pipeline(False)
        pq.set_wait_budget(0)
    y = c.forward()
    torch.cuda.synchronize()
    assert pq.stream_status() == _lib.SQ_OK
    c.compare_rows(y, np.arange(c.wl.M))


# ---------------------------------------------------- 2-SM (CTA pair) GEMM
PAIR_CASES = [
    dict(M=300, K=640, N=288, kseg=[0, 640]),                       # ragged M, tail N = 32
    dict(M=513, K=1152, N=1152, kseg=[0, 1152]),                    # 3 pair rows, N = 4.5 x 256
    dict(M=256, K=384, N=64, kseg=[0, 384]),                        # one pair tile, narrow N
    dict(M=390, K=768, N=416, kseg=[0, 256, 768], x_sigmas=[1.0, 4.0]),  # two segments
    dict(M=100, K=256, N=256, kseg=[0, 256]),                       # the peer CTA's rows are all padding
]


@pytest.mark.parametrize("bn", ["128", "256"])
@pytest.mark.parametrize("i", range(len(PAIR_CASES)))
def test_pair_gemm_matches_oracle(i, bn, monkeypatch, dev_lib):
    """The GEMM from codes on CTA pairs (tcgen05.mma.cta_group::2) gives the
    oracle's result; several K segments use the double-buffered BN = 128 path."""
    import post_quantized_linear_b200 as pq
    monkeypatch.setenv("SEGQUANT_PAIR", "1")
    monkeypatch.setenv("SEGQUANT_BN", bn)
    p = dict(PAIR_CASES[i])
    wl = W.small_case(p.pop("M"), p.pop("K"), p.pop("N"), seed=40 + i, out="bf16", **p)
    c = Case(wl)
    qp, qn = pq.quantize_activations(c.x, wl.kseg, c.sp, c.sn)
    y = pq.linear_from_codes(qp, qn, c.qw, c.sp, c.sn, c.b)
    torch.cuda.synchronize()
    assert pq.stream_status() == 0
    c.compare_rows(y, np.arange(wl.M))
    # bit-identical to the one-CTA kernel
    monkeypatch.setenv("SEGQUANT_PAIR", "0")
    y1 = pq.linear_from_codes(qp, qn, c.qw, c.sp, c.sn, c.b)
    assert torch.equal(y.view(torch.int16), y1.view(torch.int16))


def test_pair_gemm_fp32_bit_exact(monkeypatch, dev_lib):
    import post_quantized_linear_b200 as pq
    monkeypatch.setenv("SEGQUANT_PAIR", "1")
    wl = W.small_case(300, 640, 288, seed=50, kseg=[0, 256, 640], x_sigmas=[1.0, 3.0], out="bf16")
    c = Case(wl)
    qp, qn = pq.quantize_activations(c.x, wl.kseg, c.sp, c.sn)
    # with fp32 output the fixed epilogue order makes the result bit-exact
    y = pq.linear_from_codes(qp, qn, c.qw, c.sp, c.sn, c.b, out_dtype=torch.float32)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(y.cpu().numpy(), O.epilogue(*_epi_args(c, wl)))


def _epi_args(c, wl):
    _, acc = c.oracle_rows(np.arange(wl.M))
    ub, useg = O.units_of(wl.bits, wl.K, wl.kseg)
    return (acc, useg, c.o_sp, c.o_sn, O.unit_weight_scales(wl.bits, c.o_ws), c.b_np, "f32")


@pytest.mark.parametrize("name", ["dit_xl2_fc2_cfg", "seglinear_qkv", "mmdit_mlp_up"])
def test_pair_gemm_full_size_sampled_rows(name, monkeypatch, dev_lib):
    import post_quantized_linear_b200 as pq
    monkeypatch.setenv("SEGQUANT_PAIR", "1")
    wl = W.WORKLOADS[name]
    c = Case(wl)
    qp, qn = pq.quantize_activations(c.x, wl.kseg, c.sp, c.sn)
    y = pq.linear_from_codes(qp, qn, c.qw, c.sp, c.sn, c.b, out_dtype=c.out_dtype)
    torch.cuda.synchronize()
    assert pq.stream_status() == 0
    c.compare_rows(y, sample_rows(wl.M, 96 if wl.N > 4096 else 160))
