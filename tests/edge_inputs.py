"""Constructed activation inputs for the GPU edge-case parity tests.

Values are chosen where the quantization rule of the SegQuant DualScale step
(Spanish technical summary 2.B: the non-negative part with its own scale, the
negative part with another; round half to even and clamp to +-127 as the
workload text fixes) has its corner cases:

  * exact round-half ties x * r = i + 1/2 for i = 0..127, both signs, where r
    is the fp32 reciprocal of a polarity's scale;
  * -0.0 and +0.0;
  * the fp32 (or bf16) neighbours of the clamp thresholds +-127.5 / r;
  * +-inf (only where that polarity's scale is non-zero) and +-FLT_MAX;
  * subnormal inputs, and a subnormal scale whose reciprocal turns subnormal
    inputs into small codes (with ties);
  * a polarity whose scale is zero.

The module only builds inputs (no quantization arithmetic): the expected codes
always come from the oracle.
"""
from __future__ import annotations

from fractions import Fraction
from typing import List, Sequence

import numpy as np

F32 = np.float32


def recip(s: float) -> np.float32:
    """fp32 1/s (IEEE division), 0 for s = 0: the reciprocal every quantizer uses."""
    s = F32(s)
    return F32(0.0) if s == 0 else F32(1.0) / s


def bf16_exact(v: np.ndarray) -> np.ndarray:
    """Mask of fp32 values that bf16 holds exactly."""
    return (np.asarray(v, F32).view(np.uint32) & 0xFFFF) == 0


def _neighbours(v: float, dtype: str, n: int = 3) -> List[float]:
    """v and its n nearest representable neighbours on each side (fp32 or bf16)."""
    if dtype == "f32":
        out = [F32(v)]
        up = dn = F32(v)
        for _ in range(n):
            up = np.nextafter(up, F32(np.inf))
            dn = np.nextafter(dn, F32(-np.inf))
            out += [up, dn]
        return [float(x) for x in out]
    b = int(np.asarray([v], F32).view(np.uint32)[0]) >> 16   # truncated bf16 bits
    out = []
    for d in range(-n, n + 2):
        bits = np.uint32(((b + d) & 0xFFFF) << 16)
        val = float(np.asarray([bits], np.uint32).view(F32)[0])
        if np.isfinite(val):
            out.append(val)
    return out


def ties(s: float, dtype: str) -> List[float]:
    """Non-negative x with x * fl(1/s) = i + 1/2 exactly (i = 0..127) that the
    dtype represents exactly."""
    r = recip(s)
    if r == 0 or not np.isfinite(r):
        return []
    rf = Fraction(float(r))
    out = []
    for i in range(128):
        x = Fraction(2 * i + 1, 2) / rf
        xf = F32(float(x))
        if not np.isfinite(xf) or Fraction(float(xf)) != x:
            continue
        if dtype == "bf16" and not bf16_exact(np.asarray([xf]))[0]:
            continue
        out.append(float(xf))
    return out


def polarity_values(s: float, sign: float, dtype: str) -> List[float]:
    """Corner-case values of one polarity (sign +1 or -1) for scale s."""
    vals: List[float] = []
    r = recip(s)
    if r != 0 and np.isfinite(r):
        vals += [sign * t for t in ties(s, dtype)]
        thr = float(F32(127.5) / r)
        if np.isfinite(thr):
            vals += [sign * v for v in _neighbours(thr, dtype)]
            vals += [sign * v for v in _neighbours(float(F32(126.5) / r), dtype, 1)]
            vals += [sign * v for v in _neighbours(float(F32(0.5) / r), dtype, 1)]
        vals += [sign * float("inf")]
    vals += [sign * float(np.finfo(F32).max), sign * 2.0 ** -149, sign * 3 * 2.0 ** -140,
             sign * 2.0 ** -126, sign * 1.5 * 2.0 ** -127, sign * 2.5 * 2.0 ** -127]
    return vals


def segment_values(sp: float, sn: float, dtype: str, extra_scales: Sequence[float] = ()) -> np.ndarray:
    """Corner cases of one K segment with scales (s+, s-); extra_scales add the
    ties of other symmetric scales (the single-scale baseline's max(s+, s-))."""
    vals = [0.0, -0.0]
    vals += polarity_values(sp, +1.0, dtype)
    vals += polarity_values(sn, -1.0, dtype)
    for s in extra_scales:
        vals += [t for t in ties(s, dtype)] + [-t for t in ties(s, dtype)]
    v = np.asarray(vals, F32)
    if sn == 0:                      # -inf times a zero reciprocal: unspecified code
        v = v[~np.isneginf(v)]
    if sp == 0:
        v = v[~np.isposinf(v)]
    if dtype == "bf16":
        v = v[bf16_exact(v)]
    return v


# Scales of the edge-case segments (four K segments of 128): a power-of-two
# pair (every tie representable), reciprocals 12 and 10 (ties where 3 or 5
# divides 2i + 1), an arbitrary s+ with a zero s-, and a zero s+ with a
# subnormal s- (its reciprocal 2^127 maps subnormal inputs to codes -1, -2, ...).
EDGE_SCALES_POS = [2.0 ** -3, float(F32(1.0) / F32(12.0)), 0.0217, 0.0]
EDGE_SCALES_NEG = [2.0 ** -5, float(F32(1.0) / F32(10.0)), 0.0, 2.0 ** -127]
EDGE_KSEG = [0, 128, 256, 384, 512]


def edge_activations(M: int, dtype: str, seed: int = 0, kseg: Sequence[int] = EDGE_KSEG,
                     sp: Sequence[float] = EDGE_SCALES_POS, sn: Sequence[float] = EDGE_SCALES_NEG,
                     single: bool = True) -> np.ndarray:
    """fp32 [M, K] activations: every segment's columns hold its corner cases
    (each at several positions, every row tile) mixed with SiLU-like values.
    All values are exact in `dtype`."""
    rng = np.random.default_rng(seed)
    K = kseg[-1]
    x = np.empty((M, K), F32)
    for j in range(len(kseg) - 1):
        k0, k1 = kseg[j], kseg[j + 1]
        extra = [max(sp[j], sn[j])] if single else []
        corner = segment_values(sp[j], sn[j], dtype, extra)
        n = M * (k1 - k0)
        reps = max(1, (n // 2) // max(1, len(corner)))
        rand = _silu_like(rng, n, sp[j], sn[j])
        if dtype == "bf16":
            rand = (rand.view(np.uint32) & np.uint32(0xFFFF0000)).view(F32)
        pool = np.concatenate([np.tile(corner, reps), rand])
        rng.shuffle(pool)
        x[:, k0:k1] = pool[:n].reshape(M, k1 - k0)
    if dtype == "bf16":
        bits = x.view(np.uint32)
        assert np.all((bits & 0xFFFF) == 0)
    return x


def _silu_like(rng, n: int, sp: float, sn: float) -> np.ndarray:
    """Random values on the scale of the segment's codes (mostly in range)."""
    spread = max(sp, sn, 1e-30) * 127.0
    v = rng.standard_normal(n).astype(np.float64) * spread * 0.4
    return v.astype(F32)


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) of fp32 values that bf16 holds exactly."""
    b = np.asarray(x, F32).view(np.uint32)
    assert np.all((b & 0xFFFF) == 0)
    return (b >> 16).astype(np.uint16)


def hadamard_spikes(M: int, K: int, s_pos: float, s_neg: float, seed: int = 0) -> np.ndarray:
    """fp32 [M, K] whose 16-wide blocks are mostly single spikes 4t at one
    position: the block's transform (x H16 / 4) is then +-t in all 16 places,
    with t an exact round-half tie of s+ or of s- (so both polarities meet
    ties of their own scale); the rest are two-spike blocks and small random
    blocks.  Every value is exact in bf16."""
    rng = np.random.default_rng(seed)
    tt = ties(s_pos, "bf16") + ties(s_neg, "bf16")
    s = max(s_pos, s_neg)
    x = np.zeros((M, K), F32)
    for m in range(M):
        for b0 in range(0, K, 16):
            kind = rng.integers(0, 4)
            if kind <= 1:
                t = tt[rng.integers(len(tt))] * (1 if rng.integers(2) else -1)
                x[m, b0 + rng.integers(16)] = F32(4 * t)
            elif kind == 2:
                p = rng.choice(16, 2, replace=False)
                x[m, b0 + p[0]] = F32(4 * tt[rng.integers(len(tt))])
                x[m, b0 + p[1]] = F32(-4 * tt[rng.integers(len(tt))])
            else:
                v = (rng.standard_normal(16) * s * 40).astype(F32)
                x[m, b0:b0 + 16] = (v.view(np.uint32) & 0xFFFF0000).view(F32)
    return x
