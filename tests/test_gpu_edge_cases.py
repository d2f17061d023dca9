"""The method's constructed corner cases through every GPU quantizer, bit-exact
against the oracle (SegQuant DualScale, Spanish technical summary 2.B: the
non-negative part of each activation with s+, the negative part with s-;
round half to even and clamp to +-127 as the workload text fixes).

Inputs (tests/edge_inputs.py): exact round-half ties of each polarity's
reciprocal, signed zeros, the neighbours of the +-127.5 / r clamp thresholds,
+-inf where the polarity's scale is non-zero, +-FLT_MAX, subnormal inputs, a
subnormal scale, and a polarity with a zero scale, in four K segments with
different (s+, s-), fp32 and bf16 activations.

Quantizers covered:
  * standalone q+/q- (sq_quantize_activations), combined c = q+ + q-
    (sq_quantize_activations_combined), single scale
    (sq_quantize_activations_single) and block-Hadamard
    (sq_quantize_activations_hadamard): codes compared directly;
  * the quantizers inside the GEMMs -- in place over the bf16 stage (the
    default fused forward), the operand-producer warps (bf16 with int4
    weights, and with the in-place option off), and fp32 activations: their
    codes reach the int32 accumulators (sq_linear_accumulators), which are
    compared bit-exact, and the fp32 outputs, compared bit-exact too.  The
    weight has an identity block, so every code lands in an accumulator of
    its own.
"""
import numpy as np
import pytest
import torch

import oracle as O

import edge_inputs as E

pytestmark = pytest.mark.gpu

M = 300            # three row tiles, the last one ragged


@pytest.fixture(scope="module", autouse=True)
def _setup():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import post_quantized_linear_b200 as pq  # noqa: F401  (fails loudly without the library)
    O.build()
    yield


def _inputs(dtype: str, seed: int, kseg=E.EDGE_KSEG, sp=E.EDGE_SCALES_POS, sn=E.EDGE_SCALES_NEG,
            x32=None):
    """(device x, oracle x, device s+, device s-, oracle s+, oracle s-)."""
    if x32 is None:
        x32 = E.edge_activations(M, dtype, seed=seed, kseg=kseg, sp=sp, sn=sn)
    if dtype == "bf16":
        xo = E.to_bf16_bits(x32)
        xd = torch.from_numpy(xo.view(np.int16)).view(torch.bfloat16).cuda()
    else:
        xo = np.ascontiguousarray(x32)
        xd = torch.from_numpy(xo).cuda()
    osp = np.asarray(sp, np.float32)
    osn = np.asarray(sn, np.float32)
    return xd, xo, torch.from_numpy(osp).cuda(), torch.from_numpy(osn).cuda(), osp, osn


def _status_ok():
    import post_quantized_linear_b200 as pq
    torch.cuda.synchronize()
    assert pq.stream_status() == 0


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_standalone_quantizer_edge_codes(dtype):
    import post_quantized_linear_b200 as pq
    xd, xo, sp, sn, osp, osn = _inputs(dtype, 1)
    qp, qn = pq.quantize_activations(xd, E.EDGE_KSEG, sp, sn)
    _status_ok()
    op, on = O.quantize_activations(xo, E.EDGE_KSEG, osp, osn)
    np.testing.assert_array_equal(qp.cpu().numpy(), op)
    np.testing.assert_array_equal(qn.cpu().numpy(), on)
    # the constructed cases are really there: ties that went to even, saturation
    assert (op == 127).any() and (on == -127).any() and (op % 2 == 0).sum() > (op % 2 == 1).sum()


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_combined_quantizer_edge_codes(dtype):
    import post_quantized_linear_b200 as pq
    xd, xo, sp, sn, osp, osn = _inputs(dtype, 2)
    c = pq.quantize_activations_combined(xd, E.EDGE_KSEG, sp, sn)
    _status_ok()
    np.testing.assert_array_equal(c.cpu().numpy(),
                                  O.quantize_activations_combined(xo, E.EDGE_KSEG, osp, osn))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_single_scale_quantizer_edge_codes(dtype):
    import post_quantized_linear_b200 as pq
    xd, xo, sp, sn, osp, osn = _inputs(dtype, 3)
    c = pq.quantize_activations_single(xd, E.EDGE_KSEG, sp, sn)
    _status_ok()
    np.testing.assert_array_equal(c.cpu().numpy(),
                                  O.quantize_activations_single(xo, E.EDGE_KSEG, osp, osn))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_hadamard_quantizer_edge_codes(dtype):
    """Blocks that are single spikes 4t transform to +-t in every place, t an
    exact tie of the segment's s+ or s-; one segment has a zero s-."""
    import post_quantized_linear_b200 as pq
    kseg = [0, 256, 512]
    sp_l, sn_l = [2.0 ** -3, 2.0 ** -4], [2.0 ** -4, 0.0]
    x32 = E.hadamard_spikes(M, 512, 2.0 ** -3, 2.0 ** -4, seed=4)
    xd, xo, sp, sn, osp, osn = _inputs(dtype, 4, kseg=kseg, sp=sp_l, sn=sn_l, x32=x32)
    qp, qn = pq.quantize_activations_hadamard(xd, kseg, sp, sn)
    _status_ok()
    op, on = O.quantize_activations_hadamard(xo, kseg, osp, osn)
    np.testing.assert_array_equal(qp.cpu().numpy(), op)
    np.testing.assert_array_equal(qn.cpu().numpy(), on)
    assert (op % 2 == 0).sum() > (op % 2 == 1).sum()     # ties went to even


def _identity_plus_random_weight(K: int, n_extra: int, seed: int) -> torch.Tensor:
    """[K + n_extra, K]: an identity block with per-channel magnitudes (every
    activation code reaches its own accumulator), then random rows."""
    g = torch.Generator().manual_seed(seed)
    eye = torch.diag(0.5 + 0.001 * torch.arange(K, dtype=torch.float32))
    rnd = torch.randn((n_extra, K), generator=g) * 0.02
    return torch.cat([eye, rnd]).contiguous()


# (activation dtype, weight bits, in-place quantizer option) -> the GEMM's quantizer:
#   bf16, 8, on  : in place over the bf16 stage (dualscale_gemm_inplace_kernel)
#   bf16, 8, off : operand-producer warps (dualscale_gemm_kernel)
#   bf16, 4      : operand-producer warps with int4 unpack
#   f32,  8 / 4  : operand-producer warps reading fp32 stages
FUSED = [("bf16", 8, "1"), ("bf16", 8, "0"), ("bf16", 4, "1"), ("f32", 8, "1"), ("f32", 4, "1")]


@pytest.mark.parametrize("dtype,bits,inplace", FUSED)
def test_fused_quantizers_edge_accumulators_and_fp32_outputs(dtype, bits, inplace, monkeypatch):
    """The in-place option off is a measured alternative: it runs in the
    development build; every other case runs in the product library."""
    import contextlib
    import post_quantized_linear_b200 as pq
    from post_quantized_linear_b200 import _lib
    monkeypatch.setenv("SEGQUANT_INPLACE", inplace)
    xd, xo, sp, sn, osp, osn = _inputs(dtype, 5 + bits)
    K = E.EDGE_KSEG[-1]
    w = _identity_plus_random_weight(K, 48, seed=bits)           # N = 560: ragged N tail
    bias = torch.randn(w.shape[0], generator=torch.Generator().manual_seed(9)) * 0.01
    with (_lib.dev_library() if inplace == "0" else contextlib.nullcontext()):
        qw = pq.quantize_weights(w.cuda(), E.EDGE_KSEG, bits=bits)
        acc = pq.linear_accumulators(xd, qw, sp, sn)
        y = pq.linear(xd, qw, sp, sn, bias.cuda(), out_dtype=torch.float32)
        _status_ok()
    if bits == 8:
        wc, ws = O.quantize_weights_w8(w.numpy(), E.EDGE_KSEG)
    else:
        wc, ws = O.quantize_weights_w4(w.numpy())
    np.testing.assert_array_equal(qw.codes.cpu().numpy(), wc)
    y_ref, acc_ref, _ = O.linear_forward(xo, E.EDGE_KSEG, osp, osn, bits, wc, ws, bias.numpy(),
                                         out="f32", return_acc=True)
    np.testing.assert_array_equal(acc.cpu().numpy(), acc_ref)
    np.testing.assert_array_equal(y.cpu().numpy(), y_ref)


@pytest.mark.parametrize("dtype,bits", [("bf16", 8), ("f32", 8), ("bf16", 4)])
def test_gemm_from_codes_edge_fp32_outputs(dtype, bits):
    """The edge-case codes of the standalone quantizer through the GEMM from
    codes (the bench's path): fp32 outputs bit-exact against the oracle."""
    import post_quantized_linear_b200 as pq
    xd, xo, sp, sn, osp, osn = _inputs(dtype, 20 + bits)
    K = E.EDGE_KSEG[-1]
    w = _identity_plus_random_weight(K, 48, seed=30 + bits)
    qw = pq.quantize_weights(w.cuda(), E.EDGE_KSEG, bits=bits)
    qp, qn = pq.quantize_activations(xd, E.EDGE_KSEG, sp, sn)
    y = pq.linear_from_codes(qp, qn, qw, sp, sn, None, out_dtype=torch.float32)
    _status_ok()
    if bits == 8:
        wc, ws = O.quantize_weights_w8(w.numpy(), E.EDGE_KSEG)
    else:
        wc, ws = O.quantize_weights_w4(w.numpy())
    y_ref = O.linear_forward(xo, E.EDGE_KSEG, osp, osn, bits, wc, ws, None, out="f32")
    np.testing.assert_array_equal(y.cpu().numpy(), y_ref)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_calibration_of_subnormals_and_signed_zeros(dtype):
    """Calibration (a7) on columns whose values are all subnormal, signed zeros
    or a mix: the maxima are taken without flushing subnormals, so the scales
    equal the oracle's bit for bit (bf16 maxima are taken on packed pairs)."""
    import post_quantized_linear_b200 as pq
    rng = np.random.default_rng(31)
    M, K = 300, 512
    kseg = [0, 128, 256, 384, 512]
    if dtype == "bf16":
        mant = rng.integers(1, 128, size=(M, K)).astype(np.uint16)        # subnormal bf16
        sign = (rng.random((M, K)) < 0.5).astype(np.uint16) << 15
        bits = mant | sign
        bits[:, 128:256] = np.where(rng.random((M, 128)) < 0.5, 0x0000, 0x8000)   # +-0 only
        bits[:, 256:384] &= 0x807F                                          # subnormal, both signs
        bits[:, 384:448] |= 0x8000                                          # negatives only
        xo = bits
        xd = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()
    else:
        v = (rng.integers(1, 1 << 23, size=(M, K)).astype(np.uint32)).view(np.float32).copy()
        v[rng.random((M, K)) < 0.5] *= -1
        v[:, 128:256] = np.where(rng.random((M, 128)) < 0.5, 0.0, -0.0)
        v[:, 384:448] = -np.abs(v[:, 384:448])
        xo = np.ascontiguousarray(v)
        xd = torch.from_numpy(xo).cuda()
    sp, sn = pq.calibrate(xd, kseg)
    _status_ok()
    osp, osn = O.calibrate(xo, kseg)
    np.testing.assert_array_equal(sp.cpu().numpy(), osp)
    np.testing.assert_array_equal(sn.cpu().numpy(), osn)
