"""Pins of the CPU oracle to things other than itself (no GPU needed).

Each test ties one oracle function to the SegQuant definitions ("SegQuant: A
Semantics-Aware and Generalizable Quantization Framework for Diffusion
Models"; Spanish technical summary section 2.B DualScale and 2.A SegLinear,
Korean technical summary section 2) through an independent route:

* exact rational arithmetic (fractions.Fraction) on tiny inputs, written from
  the definitions, including constructed round-half ties;
* a hand-derived closed-form example with power-of-two scales;
* invariants that reduce the method to a textbook routine (single-scale
  symmetric quantization via numpy.rint, plain per-channel quantization, an
  int64 numpy matmul);
* closed-form error bounds (weights within half a step; outputs within the
  fp32 rounding bound of the exact rational value);
* library conversions (torch bf16 casts, numpy float16 casts).

A plausible slip in the oracle (a dropped bias or polarity term, a sign error,
a transposed operand, a wrong rounding tie, an off-by-one segment bound) fails
at least one of these.
"""
from fractions import Fraction as Fr

import numpy as np
import pytest
import torch

import oracle as O

TWO = Fr(2)


# ---------------------------------------------------------------- exact helpers
def f32_of(q: Fr) -> Fr:
    """Round a rational to binary32, nearest-even (finite range only)."""
    if q == 0:
        return Fr(0)
    sgn = -1 if q < 0 else 1
    a = abs(q)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while TWO ** e > a:
        e -= 1
    while TWO ** (e + 1) <= a:
        e += 1
    e = max(e, -126)
    ulp = TWO ** (e - 23)
    n = round(a / ulp)  # Fraction.__round__ is half-to-even
    v = n * ulp
    assert v < TWO ** 128
    return sgn * v


def recip32(s: Fr) -> Fr:
    return f32_of(1 / s) if s > 0 else Fr(0)


def code(x: Fr, r: Fr, lo: int, hi: int) -> int:
    return int(min(max(round(x * r), lo), hi))


def exact_forward(x, kb, w, bias, bits):
    """Everything from the definitions in exact arithmetic.

    x: list of rows of Fractions; w: list of rows (N) of Fractions.
    Returns dict with s_pos, s_neg, q_pos, q_neg, wcodes, wscale (per unit),
    acc (per unit), y (exact rational), D (magnitude sum per output)."""
    M, K, N = len(x), len(x[0]), len(w)
    J = len(kb) - 1
    sp, sn = [], []
    for j in range(J):
        P = max([max(x[m][k], 0) for m in range(M) for k in range(kb[j], kb[j + 1])])
        Q = max([max(-x[m][k], 0) for m in range(M) for k in range(kb[j], kb[j + 1])])
        sp.append(f32_of(Fr(P) / 127))
        sn.append(f32_of(Fr(Q) / 127))
    seg_of_k = [max(j for j in range(J) if kb[j] <= k) for k in range(K)]
    qp = [[0] * K for _ in range(M)]
    qn = [[0] * K for _ in range(M)]
    for m in range(M):
        for k in range(K):
            j = seg_of_k[k]
            v = x[m][k]
            if v >= 0:
                qp[m][k] = code(v, recip32(sp[j]), 0, 127)
            else:
                qn[m][k] = code(v, recip32(sn[j]), -127, 0)
    if bits == 8:
        units = [(kb[j], kb[j + 1]) for j in range(J)]
        useg = list(range(J))
        wsc = [[None] * N for _ in range(J)]
        wq = [[0] * K for _ in range(N)]
        for n in range(N):
            for j in range(J):
                amax = max(abs(w[n][k]) for k in range(kb[j], kb[j + 1]))
                s = f32_of(Fr(amax) / 127)
                wsc[j][n] = s
                for k in range(kb[j], kb[j + 1]):
                    wq[n][k] = code(w[n][k], recip32(s), -127, 127)
    else:
        G = K // 128
        units = [(g * 128, (g + 1) * 128) for g in range(G)]
        useg = [seg_of_k[g * 128] for g in range(G)]
        wsc = [[None] * N for _ in range(G)]
        wq = [[0] * K for _ in range(N)]
        for n in range(N):
            for g in range(G):
                amax = max(abs(w[n][k]) for k in range(g * 128, (g + 1) * 128))
                s32 = f32_of(Fr(amax) / 7)
                s16 = Fr(float(np.float16(float(s32))))  # numpy's binary16 cast (RNE)
                wsc[g][n] = s16
                for k in range(g * 128, (g + 1) * 128):
                    wq[n][k] = code(w[n][k], recip32(s16), -7, 7)
    U = len(units)
    acc = np.zeros((U, 2, M, N), dtype=np.int64)
    y = [[Fr(0)] * N for _ in range(M)]
    D = [[Fr(0)] * N for _ in range(M)]
    for u, (k0, k1) in enumerate(units):
        j = useg[u]
        for m in range(M):
            for n in range(N):
                a_p = sum(qp[m][k] * wq[n][k] for k in range(k0, k1))
                a_n = sum(qn[m][k] * wq[n][k] for k in range(k0, k1))
                acc[u, 0, m, n] = a_p
                acc[u, 1, m, n] = a_n
                y[m][n] += wsc[u][n] * (sp[j] * a_p + sn[j] * a_n)
                D[m][n] += abs(wsc[u][n]) * (abs(sp[j] * a_p) + abs(sn[j] * a_n))
    if bias is not None:
        for m in range(M):
            for n in range(N):
                y[m][n] += bias[n]
                D[m][n] += abs(bias[n])
    return dict(sp=sp, sn=sn, qp=np.array(qp), qn=np.array(qn), wq=np.array(wq), wsc=wsc,
                acc=acc, y=y, D=D, U=U)


def run_oracle(x32, kb, w32, b32, bits):
    sp, sn = O.calibrate(x32, kb)
    if bits == 8:
        wc, ws = O.quantize_weights_w8(w32, kb)
        codes = wc
    else:
        wc, ws = O.quantize_weights_w4(w32)
        codes = O.unpack_w4(wc, x32.shape[1])
    y, acc, (qp, qn) = O.linear_forward(x32, kb, sp, sn, bits, wc, ws, b32, out="f32",
                                        return_acc=True)
    return dict(sp=sp, sn=sn, wc=wc, ws=ws, codes=codes, y=y, acc=acc, qp=qp, qn=qn)


def fp32_bound(U: int, D: Fr) -> float:
    # R9 evaluates, per unit, one product, one fma and one fma into y (plus the
    # int->fp32 conversions, exact here since |acc| < 2^24), then one bias add:
    # at most 2U + 2 roundings, each <= 2^-24 of a partial sum bounded by D.
    return float((2 * U + 4) * D) * 2.0 ** -24


def _rand_f32(rng, shape, scale):
    return (rng.standard_normal(shape) * scale).astype(np.float32)


# ------------------------------------------------------- exact brute force pins
@pytest.mark.parametrize("seed", range(6))
def test_bruteforce_w8_exact(seed):
    rng = np.random.default_rng(100 + seed)
    M, K, N = int(rng.integers(1, 5)), int(rng.integers(2, 9)), int(rng.integers(1, 6))
    J = 1 if K < 4 or seed % 2 == 0 else 2
    kb = [0, K] if J == 1 else [0, int(rng.integers(1, K)), K]
    x = _rand_f32(rng, (M, K), 1.0)
    x = np.where(x < 0, x * np.float32(0.1), x).astype(np.float32)  # SiLU-like asymmetry
    w = _rand_f32(rng, (N, K), 0.02)
    b = _rand_f32(rng, (N,), 0.05)
    ex = exact_forward([[Fr(float(v)) for v in r] for r in x], kb,
                       [[Fr(float(v)) for v in r] for r in w], [Fr(float(v)) for v in b], 8)
    o = run_oracle(x, kb, w, b, 8)
    assert [Fr(float(v)) for v in o["sp"]] == ex["sp"]
    assert [Fr(float(v)) for v in o["sn"]] == ex["sn"]
    np.testing.assert_array_equal(o["qp"], ex["qp"])
    np.testing.assert_array_equal(o["qn"], ex["qn"])
    np.testing.assert_array_equal(o["codes"], ex["wq"])
    for j in range(J):
        assert [Fr(float(v)) for v in o["ws"][j]] == ex["wsc"][j]
    np.testing.assert_array_equal(o["acc"], ex["acc"])
    for m in range(M):
        for n in range(N):
            err = abs(Fr(float(o["y"][m, n])) - ex["y"][m][n])
            assert float(err) <= fp32_bound(ex["U"], ex["D"][m][n]), (m, n)


@pytest.mark.parametrize("seed", range(3))
def test_bruteforce_w4_exact(seed):
    rng = np.random.default_rng(200 + seed)
    M, K, N = 2, 256, 3
    kb = [0, 128, 256] if seed == 1 else [0, 256]
    x = _rand_f32(rng, (M, K), 1.0)
    x = np.where(x < 0, x * np.float32(0.2), x).astype(np.float32)
    w = _rand_f32(rng, (N, K), 0.02)
    b = None if seed == 2 else _rand_f32(rng, (N,), 0.05)
    ex = exact_forward([[Fr(float(v)) for v in r] for r in x], kb,
                       [[Fr(float(v)) for v in r] for r in w],
                       None if b is None else [Fr(float(v)) for v in b], 4)
    o = run_oracle(x, kb, w, b, 4)
    np.testing.assert_array_equal(o["codes"], ex["wq"])
    G = K // 128
    for g in range(G):
        assert [Fr(float(v)) for v in o["ws"][g]] == ex["wsc"][g]
    np.testing.assert_array_equal(o["qp"], ex["qp"])
    np.testing.assert_array_equal(o["qn"], ex["qn"])
    np.testing.assert_array_equal(o["acc"], ex["acc"])
    for m in range(M):
        for n in range(N):
            err = abs(Fr(float(o["y"][m, n])) - ex["y"][m][n])
            assert float(err) <= fp32_bound(ex["U"], ex["D"][m][n])


def test_round_half_to_even_ties():
    # s+ = 2^-4 (max(X+) = 127/16), s- = 2^-6 (max|X-| = 127/64): r+ = 16, r- = 64,
    # so every x below is an exact tie x*r = i + 1/2 (or an exact integer).
    pos = [7.9375] + [(i + 0.5) / 16 for i in range(0, 9)]
    neg = [-1.984375] + [-(i + 0.5) / 64 for i in range(0, 9)]
    x = np.array([pos + neg], dtype=np.float32)
    kb = [0, x.shape[1]]
    sp, sn = O.calibrate(x, kb)
    assert sp[0] == np.float32(2.0 ** -4) and sn[0] == np.float32(2.0 ** -6)
    qp, qn = O.quantize_activations(x, kb, sp, sn)
    expect_p = [127] + [0, 2, 2, 4, 4, 6, 6, 8, 8]          # 0.5->0, 1.5->2, 2.5->2, ...
    expect_n = [-127] + [0, -2, -2, -4, -4, -6, -6, -8, -8]
    assert list(qp[0, :10]) == expect_p and list(qn[0, :10]) == [0] * 10
    assert list(qn[0, 10:]) == expect_n and list(qp[0, 10:]) == [0] * 10


def test_hand_worked_example():
    """Closed form derived by hand with power-of-two scales (every value exact).

    X = [[127/16, 1, -127/64, -1/2], [1/32, 3/32, -1/128, -3/128]]
      -> s+ = 2^-4, s- = 2^-6; q+ = [[127,16,0,0],[0,2,0,0]] (1/32*16 = 1/2 -> 0,
         3/32*16 = 3/2 -> 2), q- = [[0,0,-127,-32],[0,0,0,-2]] (-1/2 -> -0, -3/2 -> -2).
    W = [[127/128, -1/2, 1/4, -1/128], [0, 127/256, -1/4, 1/8]]
      -> s_w = [2^-7, 2^-8]; q_w = [[127,-64,32,-1],[0,127,-64,32]].
    acc+ = [[15105, 2032], [-128, 254]], acc- = [[-4032, 7104], [2, -64]].
    y = s_w * (s+ acc+ + s- acc-) + b with b = [1/4, -1/2]:
      y00 = 2^-7 (15105/16 - 4032/64) + 1/4 = 14097/2048 + 1/4
      y01 = 2^-8 (2032/16 + 7104/64) - 1/2 = 238/256 - 1/2
      y10 = 2^-7 (-128/16 + 2/64) + 1/4 = -7.96875/128 + 1/4
      y11 = 2^-8 (254/16 - 64/64) - 1/2 = 14.875/256 - 1/2
    """
    x = np.array([[127 / 16, 1.0, -127 / 64, -0.5], [1 / 32, 3 / 32, -1 / 128, -3 / 128]],
                 dtype=np.float32)
    w = np.array([[127 / 128, -0.5, 0.25, -1 / 128], [0.0, 127 / 256, -0.25, 0.125]],
                 dtype=np.float32)
    b = np.array([0.25, -0.5], dtype=np.float32)
    o = run_oracle(x, [0, 4], w, b, 8)
    assert o["sp"][0] == 2.0 ** -4 and o["sn"][0] == 2.0 ** -6
    np.testing.assert_array_equal(o["qp"], [[127, 16, 0, 0], [0, 2, 0, 0]])
    np.testing.assert_array_equal(o["qn"], [[0, 0, -127, -32], [0, 0, 0, -2]])
    np.testing.assert_array_equal(o["codes"], [[127, -64, 32, -1], [0, 127, -64, 32]])
    np.testing.assert_array_equal(o["ws"][0], [2.0 ** -7, 2.0 ** -8])
    np.testing.assert_array_equal(o["acc"][0, 0], [[15105, 2032], [-128, 254]])
    np.testing.assert_array_equal(o["acc"][0, 1], [[-4032, 7104], [2, -64]])
    expect = np.array([[14097 / 2048 + 0.25, 238 / 256 - 0.5],
                       [-7.96875 / 128 + 0.25, 14.875 / 256 - 0.5]], dtype=np.float64)
    np.testing.assert_array_equal(o["y"].astype(np.float64), expect)
    # combined code c = q+ + q- of the same example, from the hand-derived codes
    c = O.quantize_activations_combined(x, [0, 4], o["sp"], o["sn"])
    np.testing.assert_array_equal(c, [[127, 16, -127, -32], [0, 2, 0, -2]])


# ------------------------------------------------------------------ invariants
def _silu_like(rng, shape, neg_scale=0.25):
    z = rng.standard_normal(shape).astype(np.float32)
    return np.where(z < 0, z * np.float32(neg_scale), z).astype(np.float32)


def test_I1_equal_scales_is_single_scale():
    """s+ = s- = s reduces DualScale to ordinary symmetric quantization."""
    rng = np.random.default_rng(1)
    x = _silu_like(rng, (16, 384))
    s = np.float32(np.abs(x).max() / np.float32(127))
    kb = [0, 384]
    qp, qn = O.quantize_activations(x, kb, [s], [s])
    r = np.float32(1) / s
    single = np.clip(np.rint(x.astype(np.float64) * np.float64(r)), -127, 127).astype(np.int64)
    np.testing.assert_array_equal(qp.astype(np.int64) + qn, single)
    # with one scale the combined code is the textbook symmetric code
    c = O.quantize_activations_combined(x, kb, [s], [s])
    np.testing.assert_array_equal(c.astype(np.int64), single)
    w = _rand_f32(rng, (24, 384), 0.02)
    wc, ws = O.quantize_weights_w8(w, kb)
    acc = O.accumulate(qp, qn, wc, [0, 384])
    acc_single = single @ wc.astype(np.int64).T
    np.testing.assert_array_equal(acc[0, 0].astype(np.int64) + acc[0, 1], acc_single)
    y = O.epilogue(acc, [0], [s], [s], ws)
    y_single = (ws[0][None, :].astype(np.float64) * (np.float64(s) * acc_single))
    np.testing.assert_allclose(y, y_single, rtol=0, atol=4 * 2.0 ** -24 * np.abs(y_single).max())


def test_I2_nonnegative_inputs_zero_negative_branch():
    rng = np.random.default_rng(2)
    x = np.abs(rng.standard_normal((8, 256))).astype(np.float32)
    x[0, 0] = -0.0  # negative zero is non-negative
    kb = [0, 128, 256]
    sp, sn = O.calibrate(x, kb)
    assert np.all(sn == 0)
    qp, qn = O.quantize_activations(x, kb, sp, sn)
    assert not qn.any()
    w = _rand_f32(rng, (16, 256), 0.02)
    wc, _ = O.quantize_weights_w8(w, kb)
    acc = O.accumulate(qp, qn, wc, kb)
    assert not acc[:, 1].any()


def test_I3_single_segment_is_per_channel():
    rng = np.random.default_rng(3)
    w = _rand_f32(rng, (40, 200), 0.02)
    wc, ws = O.quantize_weights_w8(w, [0, 200])
    s = (np.abs(w).max(axis=1) / np.float32(127)).astype(np.float32)
    np.testing.assert_array_equal(ws[0], s)
    r = (np.float32(1) / s).astype(np.float32)
    q = np.clip(np.rint(w.astype(np.float64) * r[:, None].astype(np.float64)), -127, 127)
    np.testing.assert_array_equal(wc, q.astype(np.int8))


def test_I4_weight_error_within_half_step():
    rng = np.random.default_rng(4)
    w = _rand_f32(rng, (32, 512), 0.02)
    w[3, :] = 0.0  # an all-zero channel: scale 0, codes 0, exact
    wc, ws = O.quantize_weights_w8(w, [0, 256, 512])
    for j, (k0, k1) in enumerate([(0, 256), (256, 512)]):
        s = ws[j].astype(np.float64)[:, None]
        err = np.abs(w[:, k0:k1].astype(np.float64) - s * wc[:, k0:k1])
        assert np.all(err <= s / 2 * (1 + 2.0 ** -20))
    packed, s16 = O.quantize_weights_w4(w)
    codes = O.unpack_w4(packed, 512)
    assert codes.min() >= -7 and codes.max() <= 7
    sf = s16.astype(np.float64)  # [G, N]
    for g in range(4):
        blk = slice(g * 128, (g + 1) * 128)
        err = np.abs(w[:, blk].astype(np.float64) - sf[g][:, None] * codes[:, blk])
        assert np.all(err <= sf[g][:, None] / 2 * (1 + 2.0 ** -10))


def test_I5_sign_symmetry():
    """Codes of -X with the scales swapped are the negated, swapped codes of X."""
    rng = np.random.default_rng(5)
    x = _silu_like(rng, (12, 256))
    kb = [0, 256]
    sp, sn = O.calibrate(x, kb)
    qp, qn = O.quantize_activations(x, kb, sp, sn)
    qp2, qn2 = O.quantize_activations(-x, kb, sn, sp)
    nz = x != 0  # +-0 both go to the positive branch with code 0
    np.testing.assert_array_equal(qp2[nz], -qn[nz])
    np.testing.assert_array_equal(qn2[nz], -qp[nz])


def test_I6_output_segments_change_nothing():
    """Per-channel weight scales make an N split (q | k | v) a numerical no-op."""
    rng = np.random.default_rng(6)
    x = _silu_like(rng, (8, 256))
    w = _rand_f32(rng, (48, 256), 0.02)
    w[16:32] *= 2.5
    kb = [0, 128, 256]
    sp, sn = O.calibrate(x, kb)
    wc, ws = O.quantize_weights_w8(w, kb)
    y = O.linear_forward(x, kb, sp, sn, 8, wc, ws)
    for n0, n1 in [(0, 16), (16, 32), (32, 48)]:
        wc_s, ws_s = O.quantize_weights_w8(w[n0:n1], kb)
        np.testing.assert_array_equal(wc_s, wc[n0:n1])
        np.testing.assert_array_equal(ws_s, ws[:, n0:n1])
        y_s = O.linear_forward(x, kb, sp, sn, 8, wc_s, ws_s)
        np.testing.assert_array_equal(y_s, y[:, n0:n1])


def test_I7_equal_segments_sum_to_single_segment():
    rng = np.random.default_rng(7)
    x = _silu_like(rng, (8, 256))
    x[:, :128] = x[:, 128:]  # identical halves: identical per-segment scales
    w = _rand_f32(rng, (16, 256), 0.02)
    w[:, :128] = w[:, 128:]
    kb2 = [0, 128, 256]
    sp2, sn2 = O.calibrate(x, kb2)
    sp1, sn1 = O.calibrate(x, [0, 256])
    assert sp2[0] == sp2[1] == sp1[0] and sn2[0] == sn2[1] == sn1[0]
    qp2, qn2 = O.quantize_activations(x, kb2, sp2, sn2)
    qp1, qn1 = O.quantize_activations(x, [0, 256], sp1, sn1)
    np.testing.assert_array_equal(qp2, qp1)
    wc2, _ = O.quantize_weights_w8(w, kb2)
    wc1, _ = O.quantize_weights_w8(w, [0, 256])
    np.testing.assert_array_equal(wc2, wc1)
    acc2 = O.accumulate(qp2, qn2, wc2, kb2)
    acc1 = O.accumulate(qp1, qn1, wc1, [0, 256])
    np.testing.assert_array_equal(acc2.sum(axis=0), acc1[0])


def test_I8_code_ranges_and_disjoint_support():
    rng = np.random.default_rng(8)
    x = _silu_like(rng, (32, 384)) * np.float32(3)
    x[0, :4] = [np.inf, -np.inf, 1e30, -1e30]
    kb = [0, 384]
    sp, sn = O.calibrate(x[1:], kb)  # forward rows beyond the calibration range saturate
    qp, qn = O.quantize_activations(x, kb, sp, sn)
    assert qp.min() >= 0 and qp.max() <= 127 and qn.min() >= -127 and qn.max() <= 0
    assert not (qp.astype(np.int32) * qn).any()
    assert list(qp[0, :4]) == [127, 0, 127, 0] and list(qn[0, :4]) == [0, -127, 0, -127]
    # disjoint support: the combined code splits back losslessly
    c = O.quantize_activations_combined(x, kb, sp, sn)
    assert c.min() >= -127 and c.max() <= 127
    np.testing.assert_array_equal(np.maximum(c, 0), qp)
    np.testing.assert_array_equal(np.minimum(c, 0), qn)


def test_I9_power_of_two_rescaling():
    rng = np.random.default_rng(9)
    x = _silu_like(rng, (8, 256))
    kb = [0, 256]
    sp, sn = O.calibrate(x, kb)
    qp, qn = O.quantize_activations(x, kb, sp, sn)
    for e in (-5, 3, 11):
        f = np.float32(2.0 ** e)
        sp_e, sn_e = O.calibrate(x * f, kb)
        np.testing.assert_array_equal(sp_e, sp * f)
        qp_e, qn_e = O.quantize_activations(x * f, kb, sp_e, sn_e)
        np.testing.assert_array_equal(qp_e, qp)
        np.testing.assert_array_equal(qn_e, qn)


def test_accumulators_equal_int64_matmul():
    rng = np.random.default_rng(10)
    x = _silu_like(rng, (24, 640))
    kb = [0, 256, 640]
    sp, sn = O.calibrate(x, kb)
    qp, qn = O.quantize_activations(x, kb, sp, sn)
    w = _rand_f32(rng, (20, 640), 0.02)
    wc, _ = O.quantize_weights_w8(w, kb)
    acc = O.accumulate(qp, qn, wc, kb)
    for u, (k0, k1) in enumerate([(0, 256), (256, 640)]):
        np.testing.assert_array_equal(acc[u, 0], qp[:, k0:k1].astype(np.int64) @ wc[:, k0:k1].astype(np.int64).T)
        np.testing.assert_array_equal(acc[u, 1], qn[:, k0:k1].astype(np.int64) @ wc[:, k0:k1].astype(np.int64).T)


@pytest.mark.parametrize("bits", [8, 4])
def test_outputs_within_fp32_bound_of_fp64_definition(bits):
    rng = np.random.default_rng(11 + bits)
    M, K, N = 24, 512, 40
    kb = [0, 256, 512]
    x = _silu_like(rng, (M, K))
    x[:, 256:] *= np.float32(5)
    w = _rand_f32(rng, (N, K), 0.02)
    b = _rand_f32(rng, (N,), 0.01)
    o = run_oracle(x, kb, w, b, bits)
    ub, useg = O.units_of(bits, K, kb)
    sw = O.unit_weight_scales(bits, o["ws"]).astype(np.float64)
    y64 = np.zeros((M, N))
    D = np.zeros((M, N))
    for u in range(len(ub) - 1):
        k0, k1 = ub[u], ub[u + 1]
        j = useg[u]
        ap = o["qp"][:, k0:k1].astype(np.float64) @ o["codes"][:, k0:k1].astype(np.float64).T
        an = o["qn"][:, k0:k1].astype(np.float64) @ o["codes"][:, k0:k1].astype(np.float64).T
        y64 += sw[u] * (np.float64(o["sp"][j]) * ap + np.float64(o["sn"][j]) * an)
        D += np.abs(sw[u]) * (np.abs(np.float64(o["sp"][j]) * ap) + np.abs(np.float64(o["sn"][j]) * an))
    y64 += b
    D += np.abs(b)
    U = len(ub) - 1
    assert np.all(np.abs(o["y"] - y64) <= (2 * U + 4) * 2.0 ** -24 * D + 1e-30)
    # a dropped negative branch would miss by far more than the bound
    assert np.max(np.abs(o["y"] - y64) / (D + 1e-30)) < 1e-6


# ------------------------------------------------------- packing & conversions
def test_int4_packing_layout_and_roundtrip():
    # a weight row whose codes are known in advance: s = 7/7 = 1 -> code = rne(w)
    k = np.arange(128)
    w = np.array([((k % 15) - 7).astype(np.float32)], dtype=np.float32)
    packed, s16 = O.quantize_weights_w4(w)
    assert s16.shape == (1, 1) and float(s16[0, 0]) == 1.0
    codes = ((k % 15) - 7)
    expect = [(int(codes[2 * i]) & 0xF) | ((int(codes[2 * i + 1]) & 0xF) << 4) for i in range(64)]
    assert list(packed[0]) == expect
    np.testing.assert_array_equal(O.unpack_w4(packed, 128)[0], codes)


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(12)
    v = rng.standard_normal(20000).astype(np.float32) * np.float32(10.0) ** rng.integers(-20, 20, 20000).astype(np.float32)
    # exact ties between bf16 neighbours
    base = np.array([1.0, 1.5, -3.0, 100.0], np.float32).view(np.uint32)
    ties = np.concatenate([(base + 0x8000).view(np.float32), (base + 0x18000).view(np.float32)])
    v = np.concatenate([v, ties, np.float32([0.0, -0.0, 3.4e38, -3.4e38])])
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([O.f32_to_bf16_bits(float(t)) for t in v], np.uint16)
    np.testing.assert_array_equal(got, ref)


def test_f16_rounding_matches_numpy():
    rng = np.random.default_rng(13)
    v = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * np.float32(10.0) ** rng.integers(-9, 5, 20000).astype(np.float32),
        np.float32([65504.0, 65519.0, 65520.0, 6.1035156e-05, 5.9604645e-08, 2.9802322e-08, 0.0]),
    ]).astype(np.float32)
    ref = v.astype(np.float16).view(np.uint16)
    got = np.array([O.f32_to_f16_bits(float(t)) for t in v], np.uint16)
    np.testing.assert_array_equal(got, ref)


def test_calibration_rejects_non_finite():
    x = np.ones((4, 8), np.float32)
    x[1, 2] = np.inf
    with pytest.raises(O.OracleError) as e:
        O.calibrate(x, [0, 8])
    assert e.value.code == O.ERR_RANGE
    x[1, 2] = np.nan
    with pytest.raises(O.OracleError):
        O.calibrate(x, [0, 8])


def test_calibration_is_per_segment_max_over_127():
    rng = np.random.default_rng(14)
    x = _silu_like(rng, (64, 384))
    x[:, 128:] *= np.float32(7)
    sp, sn = O.calibrate(x, [0, 128, 384])
    for j, (k0, k1) in enumerate([(0, 128), (128, 384)]):
        blk = x[:, k0:k1]
        assert Fr(float(sp[j])) == f32_of(Fr(float(blk.max())) / 127)
        assert Fr(float(sn[j])) == f32_of(Fr(float(-blk.min())) / 127)


def test_bf16_activations_widen_exactly():
    rng = np.random.default_rng(15)
    xt = torch.from_numpy(_silu_like(rng, (8, 256))).to(torch.bfloat16)
    xb = xt.view(torch.int16).numpy().view(np.uint16)
    xf = xt.to(torch.float32).numpy()
    kb = [0, 256]
    assert np.array_equal(np.array(O.calibrate(xb, kb)), np.array(O.calibrate(xf, kb)))
    sp, sn = O.calibrate(xf, kb)
    a = O.quantize_activations(xb, kb, sp, sn)
    b = O.quantize_activations(xf, kb, sp, sn)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])
