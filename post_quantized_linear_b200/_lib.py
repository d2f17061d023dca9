"""ctypes declarations of the C ABI in ``include/segquant.h``.

Argument marshalling only: no arithmetic of the layer happens here.  Loading
fails loudly when the compiled library is missing; there is no fallback.
"""
from __future__ import annotations

import contextlib
import ctypes
import os

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG_DIR, "libsegquant.so")
# The development build of the same sources: environment switches for the
# measured alternative kernels and the two test hooks (tests only).
DEV_LIB_PATH = os.path.join(PKG_DIR, "libsegquant_dev.so")

SQ_OK, SQ_ERR_INVALID_ARG, SQ_ERR_ALIGNMENT, SQ_ERR_UNSUPPORTED = 0, 1, 2, 3
SQ_ERR_RANGE, SQ_ERR_CUDA, SQ_ERR_TIMEOUT = 4, 5, 6
SQ_F32, SQ_BF16 = 0, 1
SQ_ACT_SILU, SQ_ACT_GELU = 1, 2
SQ_MAX_SEGMENTS = 16
SQ_MAX_K = 131072

# Every function declared in include/segquant.h, with (restype, argtypes).
c_i32, c_i64, c_vp, c_size = ctypes.c_int32, ctypes.c_int64, ctypes.c_void_p, ctypes.c_size_t


class SqSegments(ctypes.Structure):
    _fields_ = [("count", ctypes.c_int32), ("bounds", ctypes.POINTER(ctypes.c_int32))]


class SqQWeight(ctypes.Structure):
    _fields_ = [("bits", ctypes.c_int32), ("group", ctypes.c_int32), ("N", ctypes.c_int64),
                ("K", ctypes.c_int64), ("kseg", SqSegments), ("nseg", SqSegments),
                ("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p)]


P_SEG = ctypes.POINTER(SqSegments)
P_QW = ctypes.POINTER(SqQWeight)
P_SIZE = ctypes.POINTER(c_size)

SIGNATURES = {
    "sq_qweight_sizes": (c_i32, [c_i32, c_i64, c_i64, c_i32, c_i32, P_SIZE, P_SIZE]),
    "sq_calibrate": (c_i32, [c_vp, c_i32, c_i64, c_i64, c_i64, P_SEG, c_vp, c_vp, c_vp]),
    "sq_quantize_weights": (c_i32, [c_vp, c_i32, c_i64, c_i64, c_i64, P_QW, c_vp]),
    "sq_linear_forward": (c_i32, [c_vp, c_i32, c_i64, c_i64, c_i64, P_QW, c_vp, c_vp, c_vp, c_vp,
                                  c_i32, c_i64, c_vp]),
    "sq_linear_forward_codes": (c_i32, [c_vp, c_vp, c_i64, c_i64, c_i64, P_QW, c_vp, c_vp, c_vp,
                                        c_vp, c_i32, c_i64, c_vp]),
    "sq_quantize_activations": (c_i32, [c_vp, c_i32, c_i64, c_i64, c_i64, P_SEG, c_vp, c_vp, c_vp,
                                        c_vp, c_i64, c_vp]),
    "sq_quantize_activations_combined": (c_i32, [c_vp, c_i32, c_i64, c_i64, c_i64, P_SEG, c_vp,
                                                 c_vp, c_vp, c_i64, c_vp]),
    "sq_calibrate_act": (c_i32, [c_vp, c_i32, c_i32, c_i64, c_i64, c_i64, P_SEG, c_vp, c_vp, c_vp]),
    "sq_quantize_activations_combined_act": (c_i32, [c_vp, c_i32, c_i32, c_i64, c_i64, c_i64, P_SEG,
                                                     c_vp, c_vp, c_vp, c_i64, c_vp]),
    "sq_linear_forward_combined": (c_i32, [c_vp, c_i64, c_i64, c_i64, P_QW, c_vp, c_vp, c_vp, c_vp,
                                           c_i32, c_i64, c_vp]),
    "sq_quantize_activations_single": (c_i32, [c_vp, c_i32, c_i64, c_i64, c_i64, P_SEG, c_vp,
                                               c_vp, c_vp, c_i64, c_vp]),
    "sq_linear_forward_single": (c_i32, [c_vp, c_i64, c_i64, c_i64, P_QW, c_vp, c_vp, c_vp, c_vp,
                                         c_i32, c_i64, c_vp]),
    "sq_linear_forward_codes_splitk": (c_i32, [c_vp, c_vp, c_i64, c_i64, c_i64, P_QW, c_vp, c_vp,
                                               c_vp, c_vp, c_i32, c_i64, c_vp, ctypes.c_size_t,
                                               c_vp]),
    "sq_splitk_workspace_size": (c_i32, [c_i64, c_i64, c_i64, ctypes.POINTER(ctypes.c_size_t)]),
    "sq_linear_forward_codes_splitk_static": (c_i32, [c_vp, c_vp, c_i64, c_i64, c_i64, P_QW, c_vp,
                                                      c_vp, c_vp, c_vp, c_i32, c_i64, c_vp]),
    "sq_linear_accumulators": (c_i32, [c_vp, c_i32, c_i64, c_i64, c_i64, P_QW, c_vp, c_vp, c_vp,
                                       c_vp]),
    "sq_calibrate_hadamard": (c_i32, [c_vp, c_i32, c_i64, c_i64, c_i64, P_SEG, c_vp, c_vp, c_vp]),
    "sq_quantize_activations_hadamard": (c_i32, [c_vp, c_i32, c_i64, c_i64, c_i64, P_SEG, c_vp,
                                                 c_vp, c_vp, c_vp, c_i64, c_vp]),
    "sq_rotate_weights_hadamard": (c_i32, [P_QW, c_vp, c_i64, c_vp]),
    "sq_linear_forward_codes_hadamard": (c_i32, [c_vp, c_vp, c_i64, c_i64, c_i64, P_QW, c_vp,
                                                 c_i64, c_vp, c_vp, c_vp, c_vp, c_i32, c_i64,
                                                 c_vp]),
    "sq_stream_status": (c_i32, [c_vp]),
    "sq_status_string": (ctypes.c_char_p, [c_i32]),
    "sq_last_cuda_error": (ctypes.c_char_p, []),
    "sq_set_wait_budget": (c_i32, [c_i64]),
    "sq_debug_starve_pipeline": (c_i32, [c_i32]),
}

_libs = {}
_active = None   # the development library while dev_library() is open


def _open(path: str):
    if path not in _libs:
        if not os.path.exists(path):
            raise ImportError(
                f"{path} is missing: build it with `python -m post_quantized_linear_b200.build`"
                " (there is no CPU fallback)")
        lib = ctypes.CDLL(path)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _libs[path] = lib
    return _libs[path]


def load():
    """The library the binding calls: ``libsegquant.so`` (built by
    ``post_quantized_linear_b200.build``), or the development build inside
    ``dev_library()``."""
    return _active if _active is not None else _open(LIB_PATH)


def load_dev():
    """The development build ``libsegquant_dev.so``."""
    return _open(DEV_LIB_PATH)


@contextlib.contextmanager
def dev_library():
    """Route the binding's calls to the development build for the duration
    (tests of the alternative kernels and of the wait hooks)."""
    global _active
    prev = _active
    _active = load_dev()
    try:
        yield _active
    finally:
        _active = prev


def status_string(code: int) -> str:
    return load().sq_status_string(int(code)).decode()


class SegQuantError(RuntimeError):
    def __init__(self, fn: str, code: int):
        self.code = int(code)
        msg = f"{fn} failed: {status_string(code)}"
        if self.code == SQ_ERR_CUDA:
            msg += f" ({load().sq_last_cuda_error().decode()})"
        super().__init__(msg)


def check(fn: str, code: int) -> None:
    if code != SQ_OK:
        raise SegQuantError(fn, code)


def segments(bounds) -> tuple:
    """Build an sq_segments struct; returns (struct, keep-alive array)."""
    arr = (ctypes.c_int32 * len(bounds))(*[int(b) for b in bounds])
    return SqSegments(len(bounds) - 1, ctypes.cast(arr, ctypes.POINTER(ctypes.c_int32))), arr
