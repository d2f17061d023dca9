"""Pins of the oracle's single-scale baseline (no GPU needed).

The baseline is the standard single-scale quantization that DualScale replaces
("SegQuant: A Semantics-Aware and Generalizable Quantization Framework for
Diffusion Models", Spanish technical summary section 2.B), measured against
it in section 4 ("Eficiencia y Despliegue").  Reading: one symmetric scale per
K segment, s = max|x| / 127 = max(s+, s-).  Each test ties an oracle function
to an independent route: numpy's textbook rounding, the DualScale oracle with
equal scales, an int64 matmul, a hand-derived example and exact rational
arithmetic."""
from fractions import Fraction as Fr

import numpy as np
import pytest

import oracle as O
from test_oracle_pins import f32_of


def _silu_like(rng, shape, neg_scale=0.25):
    z = rng.standard_normal(shape).astype(np.float32)
    return np.where(z < 0, z * np.float32(neg_scale), z).astype(np.float32)


def test_single_scale_is_max_abs_over_127():
    rng = np.random.default_rng(31)
    x = _silu_like(rng, (40, 384)) * np.float32(3)
    kb = [0, 128, 384]
    sp, sn = O.calibrate(x, kb)
    for j in range(2):
        seg = x[:, kb[j]:kb[j + 1]]
        s_direct = np.float32(np.abs(seg).max()) / np.float32(127)
        assert max(sp[j], sn[j]) == s_direct


def test_single_codes_are_textbook_symmetric_codes():
    rng = np.random.default_rng(32)
    x = _silu_like(rng, (24, 384)) * np.float32(2)
    kb = [0, 256, 384]
    sp, sn = O.calibrate(x[2:], kb)        # rows 0-1 lie outside the calibration range
    x[0, :4] = [np.inf, -np.inf, 1e30, -1e30]
    x[1, :2] = [np.nan, -0.0]
    c = O.quantize_activations_single(x, kb, sp, sn)
    for j in range(2):
        s = max(sp[j], sn[j])
        r = np.float32(1) / np.float32(s)
        seg = x[:, kb[j]:kb[j + 1]].astype(np.float64)
        with np.errstate(invalid="ignore"):
            ref = np.clip(np.rint(seg * np.float64(r)), -127, 127)
        ref = np.where(np.isnan(ref), 0, ref).astype(np.int64)
        np.testing.assert_array_equal(c[:, kb[j]:kb[j + 1]].astype(np.int64), ref)
    assert list(c[0, :4]) == [127, -127, 127, -127] and list(c[1, :2]) == [0, 0]


def test_single_equals_dualscale_with_equal_scales():
    """With s+ = s- = s the DualScale pair collapses to the single-scale code,
    and the two accumulators sum to the single-scale accumulator."""
    rng = np.random.default_rng(33)
    x = _silu_like(rng, (16, 256))
    kb = [0, 128, 256]
    sp, sn = O.calibrate(x, kb)
    s = np.maximum(sp, sn)
    c = O.quantize_activations_single(x, kb, sp, sn)
    np.testing.assert_array_equal(c, O.quantize_activations_combined(x, kb, s, s))
    w = (rng.standard_normal((20, 256)) * 0.02).astype(np.float32)
    wc, ws = O.quantize_weights_w8(w, kb)
    qp, qn = O.quantize_activations(x, kb, s, s)
    acc2 = O.accumulate(qp, qn, wc, kb)
    acc1 = O.accumulate_single(c, wc, kb)
    np.testing.assert_array_equal(acc1, acc2[:, 0] + acc2[:, 1])


def test_single_accumulators_equal_int64_matmul():
    rng = np.random.default_rng(34)
    c = rng.integers(-127, 128, size=(9, 384)).astype(np.int8)
    wc = rng.integers(-127, 128, size=(13, 384)).astype(np.int8)
    kb = [0, 128, 384]
    acc = O.accumulate_single(c, wc, kb)
    for j in range(2):
        ref = c[:, kb[j]:kb[j + 1]].astype(np.int64) @ wc[:, kb[j]:kb[j + 1]].astype(np.int64).T
        np.testing.assert_array_equal(acc[j], ref)


def test_single_hand_worked_example():
    """The DualScale hand-worked example under one scale s = max(2^-4, 2^-6) = 2^-4:
    c = [[127, 16, -32, -8], [0, 2, 0, 0]] (-127/64*16 = -31.75 -> -32,
    -1/2*16 = -8, 1/32*16 = 1/2 -> 0, 3/32*16 = 3/2 -> 2, -1/8 -> 0, -3/8 -> 0);
    with q_w = [[127,-64,32,-1],[0,127,-64,32]]:
    acc = [[16129-1024-1024+8, 2032+2048-256], [-128, 254]] = [[14089, 3824], [-128, 254]];
    y = s_w * 2^-4 * acc + b, s_w = [2^-7, 2^-8], b = [1/4, -1/2]."""
    x = np.array([[127 / 16, 1.0, -127 / 64, -0.5], [1 / 32, 3 / 32, -1 / 128, -3 / 128]],
                 dtype=np.float32)
    w = np.array([[127 / 128, -0.5, 0.25, -1 / 128], [0.0, 127 / 256, -0.25, 0.125]],
                 dtype=np.float32)
    b = np.array([0.25, -0.5], dtype=np.float32)
    kb = [0, 4]
    sp, sn = O.calibrate(x, kb)
    wc, ws = O.quantize_weights_w8(w, kb)
    y, acc, c = O.linear_forward_single(x, kb, sp, sn, wc, ws, b, out="f32", return_acc=True)
    np.testing.assert_array_equal(c, [[127, 16, -32, -8], [0, 2, 0, 0]])
    np.testing.assert_array_equal(acc[0], [[14089, 3824], [-128, 254]])
    expect = np.array([[14089 * 2.0 ** -11 + 0.25, 3824 * 2.0 ** -12 - 0.5],
                       [-128 * 2.0 ** -11 + 0.25, 254 * 2.0 ** -12 - 0.5]])
    np.testing.assert_array_equal(y.astype(np.float64), expect)


@pytest.mark.parametrize("seed", range(4))
def test_single_epilogue_rounding_order_and_bound(seed):
    """Bitwise against the stated fp32 order evaluated in exact arithmetic with
    explicit roundings, and within the rounding bound of the exact real value
    y = sum_u sw_u s_u acc_u + b."""
    rng = np.random.default_rng(40 + seed)
    U, M, N = 1 + seed % 3, 3, 5
    acc = rng.integers(-2 ** 20, 2 ** 20, size=(U, M, N)).astype(np.int32)
    useg = np.arange(U, dtype=np.int32)
    sp = (rng.random(U) * 0.01 + 1e-4).astype(np.float32)
    sn = (rng.random(U) * 0.01 + 1e-4).astype(np.float32)
    sw = (rng.random((U, N)) * 1e-3 + 1e-5).astype(np.float32)
    b = (rng.standard_normal(N) * 0.1).astype(np.float32)
    y = O.epilogue_single(acc, useg, sp, sn, sw, b, out="f32")
    for m in range(M):
        for n in range(N):
            yr, exact, D = Fr(0), Fr(0), Fr(0)
            for u in range(U):
                s = Fr(float(max(sp[u], sn[u])))
                t = f32_of(s * int(acc[u, m, n]))
                yr = f32_of(Fr(float(sw[u, n])) * t + yr)
                exact += Fr(float(sw[u, n])) * s * int(acc[u, m, n])
                D += abs(Fr(float(sw[u, n])) * s * int(acc[u, m, n]))
            yr = f32_of(yr + Fr(float(b[n])))
            exact += Fr(float(b[n]))
            D += abs(Fr(float(b[n])))
            assert Fr(float(y[m, n])) == yr, (m, n)
            assert abs(Fr(float(y[m, n])) - exact) <= (2 * U + 2) * D * Fr(2) ** -24
