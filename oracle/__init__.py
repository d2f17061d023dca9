"""CPU oracle for the SegQuant DualScale / SegLinear quantized linear layer.

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()`` and
the benchmark's CPU-baseline leg may import this package.  The product path
(``post_quantized_linear_b200``) never imports it and shares no code with it.

The arithmetic lives in ``segquant_oracle.c`` (plain C, compiled with
``-O2 -ffp-contract=off -fopenmp``); this module compiles it on demand and
exposes numpy-level wrappers.  Each wrapper follows the function of the same
name in the C file, whose comments cite the passage of the SegQuant summaries
("SegQuant: A Semantics-Aware and Generalizable Quantization Framework for
Diffusion Models", Spanish technical summary sections 2.A SegLinear and 2.B
DualScale; Korean technical summary section 2) that it restates.

Every function is pinned by the ``-m "not gpu"`` tests in
``tests/test_oracle_pins.py`` (exact-rational brute force, closed forms and
invariants); none is marked "parity unpinned" except agreement with the
paper's own kernel outputs, which the pages do not print.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "segquant_oracle.c")
_OUT_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_OUT_DIR, "libsegquant_oracle.so")
_lib = None

OK, ERR_ARG, ERR_RANGE = 0, 1, 4


def build(force: bool = False) -> str:
    """Compile the oracle's C source into a shared library (idempotent)."""
    os.makedirs(_OUT_DIR, exist_ok=True)
    stale = (not os.path.exists(_LIB_PATH)) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
               "-shared", "-fPIC", _SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        P = ctypes.c_void_p
        I64, I32, INT = ctypes.c_int64, ctypes.c_int32, ctypes.c_int
        lib.sqo_calibrate.argtypes = [P, INT, I64, I64, I64, I32, P, P, P]
        lib.sqo_quantize_activations.argtypes = [P, INT, I64, I64, I64, I32, P, P, P, P, P]
        lib.sqo_quantize_weights_w8.argtypes = [P, I64, I64, I64, I32, P, P, P]
        lib.sqo_quantize_weights_w4.argtypes = [P, I64, I64, I64, I32, P, P]
        lib.sqo_unpack_w4.argtypes = [P, I64, I64, P]
        lib.sqo_unpack_w4.restype = None
        lib.sqo_accumulate.argtypes = [P, P, I64, I64, P, I64, I32, P, P]
        lib.sqo_epilogue.argtypes = [P, I64, I64, I32, P, P, P, P, P, P, INT, I64]
        lib.sqo_quantize_activations_single.argtypes = [P, INT, I64, I64, I64, I32, P, P, P, P]
        lib.sqo_epilogue_single.argtypes = [P, I64, I64, I32, P, P, P, P, P, P, INT, I64]
        lib.sqo_f32_to_bf16.argtypes = [ctypes.c_float]
        lib.sqo_f32_to_bf16.restype = ctypes.c_uint16
        lib.sqo_f32_to_f16.argtypes = [ctypes.c_float]
        lib.sqo_f32_to_f16.restype = ctypes.c_uint16
        lib.sqo_f16_to_f32.argtypes = [ctypes.c_uint16]
        lib.sqo_f16_to_f32.restype = ctypes.c_float
        lib.sqo_activation_bf16.argtypes = [P, INT, I64, INT, P, P]
        for f in ("sqo_calibrate", "sqo_quantize_activations", "sqo_quantize_weights_w8",
                  "sqo_quantize_weights_w4", "sqo_accumulate", "sqo_epilogue",
                  "sqo_quantize_activations_single", "sqo_epilogue_single",
                  "sqo_activation_bf16"):
            getattr(lib, f).restype = ctypes.c_int
        _lib = lib
    return _lib


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _x_dtype(x: np.ndarray) -> int:
    """0 = fp32 values, 1 = bf16 stored as uint16 bit patterns."""
    if x.dtype == np.float32:
        return 0
    if x.dtype == np.uint16:
        return 1
    raise TypeError("activations must be float32 or bf16 bit patterns (uint16)")


def _bounds(b: Sequence[int]) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(b, dtype=np.int32))


class OracleError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} returned status {code}")
        self.code = code


def _check(fn: str, code: int, allow_range: bool = False):
    if code != OK and not (allow_range and code == ERR_RANGE):
        raise OracleError(fn, code)
    return code


def calibrate(x: np.ndarray, kbounds: Sequence[int]):
    """Static per-segment DualScale scales (s+, s-), each of shape [J]."""
    x = np.ascontiguousarray(x)
    rows, K = x.shape
    kb = _bounds(kbounds)
    J = len(kb) - 1
    sp = np.zeros(J, np.float32)
    sn = np.zeros(J, np.float32)
    _check("sqo_calibrate", _load().sqo_calibrate(_ptr(x), _x_dtype(x), rows, K, K, J, _ptr(kb),
                                                  _ptr(sp), _ptr(sn)))
    return sp, sn


def quantize_activations(x: np.ndarray, kbounds, s_pos, s_neg):
    """DualScale codes (q+, q-), each int8 [M, K]."""
    x = np.ascontiguousarray(x)
    M, K = x.shape
    kb = _bounds(kbounds)
    J = len(kb) - 1
    sp = np.ascontiguousarray(np.asarray(s_pos, np.float32))
    sn = np.ascontiguousarray(np.asarray(s_neg, np.float32))
    qp = np.zeros((M, K), np.int8)
    qn = np.zeros((M, K), np.int8)
    _check("sqo_quantize_activations",
           _load().sqo_quantize_activations(_ptr(x), _x_dtype(x), M, K, K, J, _ptr(kb), _ptr(sp),
                                            _ptr(sn), _ptr(qp), _ptr(qn)))
    return qp, qn


def quantize_activations_combined(x: np.ndarray, kbounds, s_pos, s_neg):
    """Combined DualScale codes c = q+ + q-, int8 [M, K] (SegQuant DualScale:
    X = X+ + X- with disjoint support, so at most one of q+, q- is non-zero)."""
    qp, qn = quantize_activations(x, kbounds, s_pos, s_neg)
    return (qp.astype(np.int16) + qn.astype(np.int16)).astype(np.int8)


def quantize_weights_w8(w: np.ndarray, kbounds):
    """Per-(channel, K-segment) int8 codes [N, K] and fp32 scales [J, N]."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    N, K = w.shape
    kb = _bounds(kbounds)
    J = len(kb) - 1
    codes = np.zeros((N, K), np.int8)
    scales = np.zeros((J, N), np.float32)
    _check("sqo_quantize_weights_w8",
           _load().sqo_quantize_weights_w8(_ptr(w), N, K, K, J, _ptr(kb), _ptr(codes), _ptr(scales)))
    return codes, scales


def quantize_weights_w4(w: np.ndarray, group: int = 128):
    """Packed int4 codes [N, K/2] (low nibble = even k) and fp16 scales [K/group, N]."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    N, K = w.shape
    packed = np.zeros((N, K // 2), np.uint8)
    scales = np.zeros((K // group, N), np.uint16)
    _check("sqo_quantize_weights_w4",
           _load().sqo_quantize_weights_w4(_ptr(w), N, K, K, group, _ptr(packed), _ptr(scales)))
    return packed, scales.view(np.float16)


def unpack_w4(packed: np.ndarray, K: int) -> np.ndarray:
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    N = packed.shape[0]
    codes = np.zeros((N, K), np.int8)
    _load().sqo_unpack_w4(_ptr(packed), N, K, _ptr(codes))
    return codes


def units_of(bits: int, K: int, kbounds: Sequence[int]):
    """Unit bounds and the K segment of each unit.

    int8 weights: one unit per K segment.  int4 weights: one unit per 128-wide
    K group (groups never straddle a segment bound, bounds being multiples of
    128)."""
    kb = list(kbounds)
    if bits == 8:
        ub = kb
        seg = list(range(len(kb) - 1))
    else:
        ub = list(range(0, K + 1, 128))
        seg = []
        for u in range(len(ub) - 1):
            j = max(i for i in range(len(kb) - 1) if kb[i] <= ub[u])
            seg.append(j)
    return np.asarray(ub, np.int32), np.asarray(seg, np.int32)


def accumulate(q_pos, q_neg, wcodes, ubounds) -> np.ndarray:
    """Per-unit int32 accumulators acc[u, polarity, m, n] (polarity 0 = +)."""
    q_pos = np.ascontiguousarray(q_pos, np.int8)
    q_neg = np.ascontiguousarray(q_neg, np.int8)
    wcodes = np.ascontiguousarray(wcodes, np.int8)
    M, K = q_pos.shape
    N = wcodes.shape[0]
    ub = _bounds(ubounds)
    U = len(ub) - 1
    acc = np.zeros((U, 2, M, N), np.int32)
    _check("sqo_accumulate", _load().sqo_accumulate(_ptr(q_pos), _ptr(q_neg), M, K, _ptr(wcodes), N,
                                                    U, _ptr(ub), _ptr(acc)))
    return acc


def epilogue(acc, unit_seg, s_pos, s_neg, unit_scales, bias=None, out: str = "f32") -> np.ndarray:
    """Fused DualScale epilogue.  unit_scales: [U, N] fp32.  out: 'f32' or 'bf16'
    (bf16 is returned as uint16 bit patterns)."""
    acc = np.ascontiguousarray(acc, np.int32)
    U, _, M, N = acc.shape
    us = np.ascontiguousarray(np.asarray(unit_seg, np.int32))
    sp = np.ascontiguousarray(np.asarray(s_pos, np.float32))
    sn = np.ascontiguousarray(np.asarray(s_neg, np.float32))
    sw = np.ascontiguousarray(np.asarray(unit_scales, np.float32))
    b = None if bias is None else np.ascontiguousarray(np.asarray(bias, np.float32))
    if out == "f32":
        y = np.zeros((M, N), np.float32)
        od = 0
    else:
        y = np.zeros((M, N), np.uint16)
        od = 1
    _check("sqo_epilogue", _load().sqo_epilogue(_ptr(acc), M, N, U, _ptr(us), _ptr(sp), _ptr(sn),
                                                _ptr(sw), _ptr(b), _ptr(y), od, N))
    return y


def unit_weight_scales(bits: int, scales: np.ndarray) -> np.ndarray:
    """Weight scale of every unit as fp32 [U, N]: the [J, N] int8 scales, or the
    widened [G, N] fp16 group scales."""
    if bits == 8:
        return np.ascontiguousarray(scales, np.float32)
    return np.ascontiguousarray(np.asarray(scales, np.float16).astype(np.float32))


def linear_forward(x, kbounds, s_pos, s_neg, bits, wcodes, wscales, bias=None, out="f32",
                   return_acc: bool = False):
    """The whole forward pass: codes, per-unit accumulators, epilogue.

    wcodes: int8 [N, K] (bits=8) or packed uint8 [N, K/2] (bits=4);
    wscales: fp32 [J, N] (bits=8) or fp16 [K/128, N] (bits=4)."""
    M, K = x.shape
    qp, qn = quantize_activations(x, kbounds, s_pos, s_neg)
    codes = wcodes if bits == 8 else unpack_w4(wcodes, K)
    ub, useg = units_of(bits, K, kbounds)
    acc = accumulate(qp, qn, codes, ub)
    y = epilogue(acc, useg, s_pos, s_neg, unit_weight_scales(bits, wscales), bias, out)
    if return_acc:
        return y, acc, (qp, qn)
    return y


def quantize_activations_single(x: np.ndarray, kbounds, s_pos, s_neg):
    """Single-scale baseline codes, int8 [M, K]: s_j = max(s+_j, s-_j)."""
    x = np.ascontiguousarray(x)
    M, K = x.shape
    kb = _bounds(kbounds)
    J = len(kb) - 1
    sp = np.ascontiguousarray(np.asarray(s_pos, np.float32))
    sn = np.ascontiguousarray(np.asarray(s_neg, np.float32))
    c = np.zeros((M, K), np.int8)
    _check("sqo_quantize_activations_single",
           _load().sqo_quantize_activations_single(_ptr(x), _x_dtype(x), M, K, K, J, _ptr(kb),
                                                   _ptr(sp), _ptr(sn), _ptr(c)))
    return c


def accumulate_single(c, wcodes, ubounds) -> np.ndarray:
    """Per-unit int32 accumulators acc[u, m, n] of single-scale codes."""
    c = np.ascontiguousarray(c, np.int8)
    return accumulate(c, np.zeros_like(c), wcodes, ubounds)[:, 0].copy()


def epilogue_single(acc, unit_seg, s_pos, s_neg, unit_scales, bias=None, out: str = "f32"):
    """Single-scale epilogue; acc int32 [U, M, N]; out 'f32' or 'bf16' (uint16 bits)."""
    acc = np.ascontiguousarray(acc, np.int32)
    U, M, N = acc.shape
    us = np.ascontiguousarray(np.asarray(unit_seg, np.int32))
    sp = np.ascontiguousarray(np.asarray(s_pos, np.float32))
    sn = np.ascontiguousarray(np.asarray(s_neg, np.float32))
    sw = np.ascontiguousarray(np.asarray(unit_scales, np.float32))
    b = None if bias is None else np.ascontiguousarray(np.asarray(bias, np.float32))
    y = np.zeros((M, N), np.float32 if out == "f32" else np.uint16)
    _check("sqo_epilogue_single",
           _load().sqo_epilogue_single(_ptr(acc), M, N, U, _ptr(us), _ptr(sp), _ptr(sn), _ptr(sw),
                                       _ptr(b), _ptr(y), 0 if out == "f32" else 1, N))
    return y


def linear_forward_single(x, kbounds, s_pos, s_neg, wcodes, wscales, bias=None, out="f32",
                          return_acc: bool = False):
    """The single-scale baseline forward (int8 weights): codes, accumulators, epilogue."""
    M, K = x.shape
    c = quantize_activations_single(x, kbounds, s_pos, s_neg)
    ub, useg = units_of(8, K, kbounds)
    acc = accumulate_single(c, wcodes, ub)
    y = epilogue_single(acc, useg, s_pos, s_neg, unit_weight_scales(8, wscales), bias, out)
    if return_acc:
        return y, acc, c
    return y


def f32_to_bf16_bits(v: float) -> int:
    return int(_load().sqo_f32_to_bf16(float(v)))


def f32_to_f16_bits(v: float) -> int:
    return int(_load().sqo_f32_to_f16(float(v)))


# ----------------------------------------------------------------------------
# Block-diagonal Hadamard transform of the activations ("HQ-DM: Single
# Hadamard Transformation-Based Quantization-Aware Training for Low-Bit
# Diffusion Models", Spanish technical summary section 2.1: the activation
# matrix X is multiplied by a block-diagonal matrix H built from standard
# Hadamard matrices and XH is quantized; the weights are left untransformed;
# because H is orthogonal and symmetric the activation is recovered as
# X^ = S * (XH)_int * H; the normalization 2^(-k/2) of a 2^k-point block is
# carried by the floating-point scales so the core stays integer).
#
# Readings (the page states the recovery step only as that formula):
# * blocks of b = 16 (k = 4) along K, so 2^(-k/2) = 1/4 is a power of two and
#   every scaling by it is exact; blocks never straddle a K-segment bound
#   (bounds are multiples of 128);
# * the transform is computed in fp32 by the radix-2 butterfly in Sylvester
#   order (one rounding per addition), then multiplied by 1/4;
# * the linear layer Y = X^ W^T with X^ = S (XH)_int H and the untransformed
#   int4 weight W^ = s_w W_int is evaluated exactly as the integer product of
#   the codes with the weight codes rotated into the same basis,
#   (XH)_int (W_int H16)^T with H16 the +-1 Sylvester matrix (H = H16 / 4):
#   Y = s_w * (S / 4) * (XH)_int (W_int H16)^T.  For int4 codes in [-7, 7] the
#   rotated codes lie in [-112, 112], so the product stays int8 x int8;
# * the factor 1/4 is applied to the activation scales (s+/4, s-/4) in the
#   DualScale epilogue, whose fixed fp32 order is otherwise unchanged.
HADAMARD_BLOCK = 16
HADAMARD_NORM = np.float32(0.25)      # 2^(-k/2) for b = 2^k = 16


def hadamard_matrix(b: int = HADAMARD_BLOCK) -> np.ndarray:
    """The b x b Sylvester Hadamard matrix (entries +-1, int64), b a power of 2:
    H_1 = [1], H_2n = [[H_n, H_n], [H_n, -H_n]]."""
    if b < 1 or b & (b - 1):
        raise ValueError("b must be a power of two")
    h = np.ones((1, 1), np.int64)
    while h.shape[0] < b:
        h = np.block([[h, h], [h, -h]])
    return h


def hadamard_transform(x: np.ndarray, b: int = HADAMARD_BLOCK) -> np.ndarray:
    """X H in fp32: each row split into blocks of b along K, each block
    replaced by its Sylvester-ordered butterfly (stage h = 1, 2, 4, ...: the
    pair (v[j], v[j+h]) becomes (v[j] + v[j+h], v[j] - v[j+h]), each rounded
    to fp32), then multiplied by 1/sqrt(b) (b = 16: 1/4, exact).  x: fp32
    values or bf16 stored as uint16 bit patterns, shape [M, K], K % b == 0."""
    if b != HADAMARD_BLOCK:
        raise ValueError("the transform uses blocks of 16")
    if x.dtype == np.uint16:
        x32 = (x.astype(np.uint32) << 16).view(np.float32)
    else:
        x32 = np.asarray(x, np.float32)
    M, K = x32.shape
    if K % b:
        raise ValueError("K must be a multiple of the block size")
    v = x32.reshape(M, K // b, b).copy()
    h = 1
    while h < b:
        for i in range(0, b, 2 * h):
            for j in range(i, i + h):
                a = v[..., j].copy()
                c = v[..., j + h].copy()
                v[..., j] = a + c
                v[..., j + h] = a - c
        h *= 2
    v *= HADAMARD_NORM
    return v.reshape(M, K)


def calibrate_hadamard(x: np.ndarray, kbounds, b: int = HADAMARD_BLOCK):
    """Static per-segment DualScale scales of the transformed activations XH."""
    return calibrate(hadamard_transform(x, b), kbounds)


def quantize_activations_hadamard(x: np.ndarray, kbounds, s_pos, s_neg, b: int = HADAMARD_BLOCK):
    """DualScale codes (q+, q-) of XH, each int8 [M, K]."""
    return quantize_activations(hadamard_transform(x, b), kbounds, s_pos, s_neg)


def rotate_weight_codes(codes: np.ndarray, b: int = HADAMARD_BLOCK) -> np.ndarray:
    """W_int H_b blockwise along K (exact integers), int8 [N, K]; raises if a
    rotated code leaves [-127, 127] (int4 codes in [-7, 7] stay within 112)."""
    c = np.asarray(codes, np.int64)
    N, K = c.shape
    r = (c.reshape(N, K // b, b) @ hadamard_matrix(b)).reshape(N, K)
    if np.abs(r).max(initial=0) > 127:
        raise ValueError("rotated weight codes exceed int8")
    return r.astype(np.int8)


def linear_forward_hadamard(x, kbounds, s_pos, s_neg, packed, scales, bias=None, out="f32",
                            b: int = HADAMARD_BLOCK, return_acc: bool = False):
    """The forward with Hadamard-transformed activations and untransformed int4
    weights (packed uint8 [N, K/2], fp16 group scales [K/128, N]): codes of XH,
    per-group int32 accumulators against the rotated weight codes, and the
    DualScale epilogue with the activation scales times 1/4.  s_pos/s_neg are
    the scales of XH (calibrate_hadamard)."""
    M, K = x.shape
    qp, qn = quantize_activations_hadamard(x, kbounds, s_pos, s_neg, b)
    rot = rotate_weight_codes(unpack_w4(packed, K), b)
    ub, useg = units_of(4, K, kbounds)
    acc = accumulate(qp, qn, rot, ub)
    sp = np.asarray(s_pos, np.float32) * HADAMARD_NORM
    sn = np.asarray(s_neg, np.float32) * HADAMARD_NORM
    y = epilogue(acc, useg, sp, sn, unit_weight_scales(4, scales), bias, out)
    if return_acc:
        return y, acc, (qp, qn), rot
    return y


# ----------------------------------------------------------------------------
# The activation in front of the layer, for the fused producer (SegQuant,
# Spanish technical summary 1 and 2.B, Korean technical summary section 2: the
# negative tail DualScale keeps comes from SiLU / GELU).  Reading: the layer
# input is x = act(z) rounded once to bf16; act is evaluated in double by the
# C library, and elements whose double lies within a relative 2^-40 of a bf16
# rounding midpoint are flagged (their rounding is not decided by a double).
ACTIVATIONS = {"silu": 1, "gelu": 2}


def activation_bf16(z: np.ndarray, act: str):
    """x = bf16_RN(act(z)) as bf16 bit patterns (uint16, z's shape) and a bool
    mask of the elements flagged as undecided by the double evaluation.
    z: fp32 values or bf16 bit patterns (uint16); act: 'silu' or 'gelu'."""
    z = np.ascontiguousarray(z)
    x = np.zeros(z.shape, np.uint16)
    flags = np.zeros(z.shape, np.uint8)
    _check("sqo_activation_bf16", _load().sqo_activation_bf16(
        _ptr(z), _x_dtype(z), z.size, ACTIVATIONS[act], _ptr(x), _ptr(flags)))
    return x, flags.astype(bool)


def calibrate_act(z: np.ndarray, act: str, kbounds):
    """Static DualScale scales of x = act(z) (calibrate applied to the bf16 x)."""
    x, _ = activation_bf16(z, act)
    return calibrate(x, kbounds)


def quantize_activations_combined_act(z: np.ndarray, act: str, kbounds, s_pos, s_neg):
    """Combined codes of x = act(z) and the flags of undecided elements."""
    x, flags = activation_bf16(z, act)
    return quantize_activations_combined(x, kbounds, s_pos, s_neg), flags
