"""Pins of the oracle's activation for the fused producer (no GPU).

The activation in front of the layer (SegQuant, Spanish technical summary 1
and 2.B; Korean technical summary section 2: the negative tail DualScale keeps
comes from SiLU / GELU).  Reading: x = act(z) rounded once, to nearest with ties
to even, to bf16; SiLU(z) = z / (1 + e^-z), GELU(z) = z/2 (1 + erf(z / sqrt 2)).

The oracle evaluates act in double with the C library and rounds from there.
These tests pin it to an independent evaluation: the definitions summed as
series in 60-digit decimal arithmetic (exp by Python's decimal module, erf by
its Maclaurin series, pi by Machin's formula), rounded to bf16 with exact
rational arithmetic; plus closed forms at special values.
"""
from decimal import Decimal, getcontext
from fractions import Fraction

import numpy as np
import pytest

import oracle as O

getcontext().prec = 60


def _pi() -> Decimal:
    """pi = 16 atan(1/5) - 4 atan(1/239) (Machin), atan by its series."""
    def atan_inv(n):
        x = Decimal(1) / n
        x2 = x * x
        term, total, k = x, Decimal(0), 0
        while abs(term) > Decimal(10) ** -70:
            total += term / (2 * k + 1) if k % 2 == 0 else -term / (2 * k + 1)
            term *= x2
            k += 1
        return total
    return 16 * atan_inv(5) - 4 * atan_inv(239)


PI = _pi()
SQRT2 = Decimal(2).sqrt()


def _erf(x: Decimal) -> Decimal:
    """erf(x) = 2/sqrt(pi) * sum_n (-1)^n x^(2n+1) / (n! (2n+1))."""
    total, term, n = Decimal(0), x, 0      # term = (-1)^n x^(2n+1) / n!
    while True:
        add = term / (2 * n + 1)
        total += add
        if abs(add) < Decimal(10) ** -75:
            break
        n += 1
        term = -term * x * x / n
    return 2 / PI.sqrt() * total


def _act_exact(z: float, act: str) -> Decimal:
    zd = Decimal(z)
    if act == "silu":
        return zd / (1 + (-zd).exp())
    return zd / 2 * (1 + _erf(zd / SQRT2))


def _bf16_rne(v: Decimal) -> int:
    """bf16 bit pattern of v rounded to nearest, ties to even (exact)."""
    if v == 0:
        return 0x8000 if v.is_signed() else 0
    sign = 0x8000 if v < 0 else 0
    a = Fraction(abs(v))
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1                                  # a in [2^e, 2^(e+1))
    E = max(e, -126)
    ulp = Fraction(2) ** (E - 7)
    q = a / ulp
    r = round(q)                                # Fraction.__round__: ties to even
    val = float(r * ulp)
    bits = int(np.asarray([val], np.float32).view(np.uint32)[0]) >> 16
    return sign | bits


def _grid():
    rng = np.random.default_rng(5)
    bf = np.arange(0x3A00, 0x4110, 7, dtype=np.uint32)            # bf16 values 2^-11 .. 9
    zb = (bf << 16).view(np.float32)
    zr = rng.uniform(-6.0, 6.0, 400).astype(np.float32)
    return np.concatenate([zb, -zb, zr])


@pytest.mark.parametrize("act", ["silu", "gelu"])
def test_activation_matches_high_precision_definition(act):
    z = _grid()
    x, flags = O.activation_bf16(z, act)
    assert not flags.any()
    want = np.array([_bf16_rne(_act_exact(float(v), act)) for v in z], np.uint16)
    np.testing.assert_array_equal(x, want)


@pytest.mark.parametrize("act", ["silu", "gelu"])
def test_activation_special_values(act):
    z = np.float32([0.0, -0.0, 60.0, 1000.0, 32768.0, -200.0, -1.0e4])
    x, flags = O.activation_bf16(z, act)
    assert not flags.any()
    f = (x.astype(np.uint32) << 16).view(np.float32)
    assert x[0] == 0x0000 and x[1] == 0x8000                 # act(+-0) = +-0
    # act(z) = z (1 - tiny) for large z: the bf16 of z itself (z exact in bf16)
    np.testing.assert_array_equal(f[2:5], np.float32([60.0, 1000.0, 32768.0]))
    # act(z) -> -0 far below: the exact value is below bf16's smallest subnormal
    assert np.all(x[5:] == 0x8000)


def test_activation_from_bf16_and_fp32_inputs_agree():
    z = _grid()
    zb = (np.asarray(z, np.float32).view(np.uint32) >> 16).astype(np.uint16)
    z32 = (zb.astype(np.uint32) << 16).view(np.float32)      # the same values as fp32
    for act in ("silu", "gelu"):
        np.testing.assert_array_equal(O.activation_bf16(zb, act)[0], O.activation_bf16(z32, act)[0])


def test_fused_codes_are_the_codes_of_the_activation():
    """quantize_activations_combined_act = the combined codes of the bf16 x."""
    rng = np.random.default_rng(9)
    z = rng.standard_normal((40, 256)).astype(np.float32) * 2
    kseg = [0, 128, 256]
    for act in ("silu", "gelu"):
        x, _ = O.activation_bf16(z, act)
        sp, sn = O.calibrate_act(z, act, kseg)
        np.testing.assert_array_equal(sp, O.calibrate(x, kseg)[0])
        c, flags = O.quantize_activations_combined_act(z, act, kseg, sp, sn)
        assert not flags.any()
        np.testing.assert_array_equal(c, O.quantize_activations_combined(x, kseg, sp, sn))
        assert (c < 0).any() and (c > 0).any()      # the negative tail survives
