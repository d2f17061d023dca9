"""B200 (sm_100a) DualScale / SegLinear quantized linear layer.

Python binding of the C ABI in ``include/segquant.h``: PyTorch supplies device
memory and the current CUDA stream; every step of the layer runs in the
library's CUDA kernels.  Function names follow the C entry points.

SegQuant ("SegQuant: A Semantics-Aware and Generalizable Quantization
Framework for Diffusion Models"): DualScale quantizes the non-negative and
negative parts of each activation with separate static scales and fuses the
two int8 products in one kernel's epilogue (Spanish technical summary 2.B;
Korean technical summary section 2); SegLinear gives each input segment its
own scales (Spanish technical summary 2.A).
"""
from __future__ import annotations

import ctypes
import dataclasses
from typing import Optional, Sequence, Tuple

import torch

from . import _lib
from ._lib import SegQuantError

__all__ = ["QuantizedWeight", "SegQuantError", "calibrate", "quantize_weights", "linear",
           "quantize_activations", "linear_from_codes", "quantize_activations_combined",
           "linear_from_combined", "quantize_activations_single", "linear_from_single",
           "splitk_workspace_size", "splitk_workspace", "linear_from_codes_splitk",
           "linear_accumulators", "stream_status", "qweight_sizes", "calibrate_hadamard",
           "quantize_activations_hadamard", "rotate_weights_hadamard",
           "linear_from_codes_hadamard", "calibrate_act", "quantize_activations_combined_act"]


def _dtype_code(t: torch.dtype) -> int:
    if t == torch.float32:
        return _lib.SQ_F32
    if t == torch.bfloat16:
        return _lib.SQ_BF16
    raise TypeError(f"unsupported dtype {t}: float32 or bfloat16")


# the current stream's raw handle without building a Stream object (a few
# microseconds per call at small M); the public call where it is missing
_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream(stream: Optional[torch.cuda.Stream]):
    """The given stream, else the current stream of the current device (the
    device the library launches on)."""
    if stream is not None:
        return ctypes.c_void_p(stream.cuda_stream)
    if _raw_stream is not None:
        return ctypes.c_void_p(_raw_stream(torch.cuda.current_device()))
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _check_2d(x: torch.Tensor, name: str):
    if x.dim() != 2 or x.stride(1) != 1:
        raise ValueError(f"{name} must be a 2-D tensor with unit column stride")
    if not x.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")


@dataclasses.dataclass
class QuantizedWeight:
    """Device codes/scales of a quantized [N, K] weight plus its segment bounds."""
    bits: int
    N: int
    K: int
    kseg: Tuple[int, ...]
    nseg: Tuple[int, ...]
    codes: torch.Tensor    # int8 [N, K] or uint8 [N, K/2]
    scales: torch.Tensor   # float32 [J, N] or float16 [K/128, N]

    @property
    def group(self) -> int:
        return 0 if self.bits == 8 else 128

    def c_struct(self):
        """The C view (sq_qweight) of this weight, rebuilt only when a field
        it is made of has changed."""
        key = (self.bits, self.N, self.K, tuple(self.kseg), tuple(self.nseg),
               self.codes.data_ptr(), self.scales.data_ptr())
        cached = self.__dict__.get("_c_struct")
        if cached is not None and cached[0] == key:
            return cached[1], cached[2]
        ks, ka = _lib.segments(self.kseg)
        ns, na = _lib.segments(self.nseg)
        qw = _lib.SqQWeight(self.bits, self.group, self.N, self.K, ks, ns,
                            ctypes.c_void_p(self.codes.data_ptr()),
                            ctypes.c_void_p(self.scales.data_ptr()))
        self.__dict__["_c_struct"] = (key, qw, (ka, na))
        return qw, (ka, na)


def qweight_sizes(bits: int, N: int, K: int, J: int) -> Tuple[int, int]:
    cb, sb = ctypes.c_size_t(), ctypes.c_size_t()
    _lib.check("sq_qweight_sizes", _lib.load().sq_qweight_sizes(
        bits, N, K, J, 0 if bits == 8 else 128, ctypes.byref(cb), ctypes.byref(sb)))
    return cb.value, sb.value


def calibrate(x: torch.Tensor, kseg: Sequence[int], s_pos: Optional[torch.Tensor] = None,
              s_neg: Optional[torch.Tensor] = None, stream=None):
    """Static DualScale scales of the calibration rows ``x`` [rows, K]: (s+, s-) fp32 [J]."""
    _check_2d(x, "x")
    J = len(kseg) - 1
    if s_pos is None:
        s_pos = torch.empty(J, dtype=torch.float32, device=x.device)
    if s_neg is None:
        s_neg = torch.empty(J, dtype=torch.float32, device=x.device)
    seg, keep = _lib.segments(kseg)
    _lib.check("sq_calibrate", _lib.load().sq_calibrate(
        _ptr(x), _dtype_code(x.dtype), x.shape[0], x.shape[1], x.stride(0), ctypes.byref(seg),
        _ptr(s_pos), _ptr(s_neg), _stream(stream)))
    return s_pos, s_neg


def quantize_weights(w: torch.Tensor, kseg: Sequence[int], nseg: Optional[Sequence[int]] = None,
                     bits: int = 8, out: Optional[QuantizedWeight] = None,
                     stream=None) -> QuantizedWeight:
    """Quantize an [N, K] weight: int8 per (channel, K segment) or int4 group 128."""
    _check_2d(w, "w")
    N, K = w.shape
    kseg = tuple(int(b) for b in kseg)
    nseg = tuple(int(b) for b in (nseg if nseg is not None else (0, N)))
    if out is None:
        cb, sb = qweight_sizes(bits, N, K, len(kseg) - 1)
        if bits == 8:
            codes = torch.empty((N, K), dtype=torch.int8, device=w.device)
            scales = torch.empty((len(kseg) - 1, N), dtype=torch.float32, device=w.device)
        else:
            codes = torch.empty((N, K // 2), dtype=torch.uint8, device=w.device)
            scales = torch.empty((K // 128, N), dtype=torch.float16, device=w.device)
        assert codes.numel() * codes.element_size() == cb
        assert scales.numel() * scales.element_size() == sb
        out = QuantizedWeight(bits, N, K, kseg, nseg, codes, scales)
    qw, keep = out.c_struct()
    _lib.check("sq_quantize_weights", _lib.load().sq_quantize_weights(
        _ptr(w), _dtype_code(w.dtype), N, K, w.stride(0), ctypes.byref(qw), _stream(stream)))
    return out


def linear(x: torch.Tensor, qw: QuantizedWeight, s_pos: torch.Tensor, s_neg: torch.Tensor,
           bias: Optional[torch.Tensor] = None, out_dtype: torch.dtype = torch.bfloat16,
           out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """The fused forward pass y = DualScale-quantized x times the quantized weight (+ bias)."""
    _check_2d(x, "x")
    M, K = x.shape
    if out is None:
        out = torch.empty((M, qw.N), dtype=out_dtype, device=x.device)
    _check_2d(out, "out")
    c, keep = qw.c_struct()
    _lib.check("sq_linear_forward", _lib.load().sq_linear_forward(
        _ptr(x), _dtype_code(x.dtype), M, K, x.stride(0), ctypes.byref(c), _ptr(s_pos),
        _ptr(s_neg), _ptr(bias), _ptr(out), _dtype_code(out.dtype), out.stride(0), _stream(stream)))
    return out


def linear_from_codes(q_pos: torch.Tensor, q_neg: torch.Tensor, qw: QuantizedWeight,
                      s_pos: torch.Tensor, s_neg: torch.Tensor, bias: Optional[torch.Tensor] = None,
                      out_dtype: torch.dtype = torch.bfloat16, out: Optional[torch.Tensor] = None,
                      stream=None) -> torch.Tensor:
    """Forward from pre-quantized DualScale codes (same result as ``linear``)."""
    _check_2d(q_pos, "q_pos")
    _check_2d(q_neg, "q_neg")
    M, K = q_pos.shape
    if q_neg.shape != q_pos.shape or q_neg.stride(0) != q_pos.stride(0):
        raise ValueError("q_pos and q_neg must have the same shape and row stride")
    if out is None:
        out = torch.empty((M, qw.N), dtype=out_dtype, device=q_pos.device)
    _check_2d(out, "out")
    c, keep = qw.c_struct()
    _lib.check("sq_linear_forward_codes", _lib.load().sq_linear_forward_codes(
        _ptr(q_pos), _ptr(q_neg), q_pos.stride(0), M, K, ctypes.byref(c), _ptr(s_pos), _ptr(s_neg),
        _ptr(bias), _ptr(out), _dtype_code(out.dtype), out.stride(0), _stream(stream)))
    return out


def quantize_activations(x: torch.Tensor, kseg: Sequence[int], s_pos: torch.Tensor,
                         s_neg: torch.Tensor, out=None, stream=None):
    """DualScale codes (q+, q-), int8 [M, K] each (row stride a multiple of 16)."""
    _check_2d(x, "x")
    M, K = x.shape
    if out is None:
        ldq = (K + 15) // 16 * 16
        qp = torch.empty((M, ldq), dtype=torch.int8, device=x.device)[:, :K]
        qn = torch.empty((M, ldq), dtype=torch.int8, device=x.device)[:, :K]
    else:
        qp, qn = out
        if qp.stride(0) != qn.stride(0):
            raise ValueError("q_pos and q_neg must share a row stride")
    seg, keep = _lib.segments(kseg)
    _lib.check("sq_quantize_activations", _lib.load().sq_quantize_activations(
        _ptr(x), _dtype_code(x.dtype), M, K, x.stride(0), ctypes.byref(seg), _ptr(s_pos),
        _ptr(s_neg), _ptr(qp), _ptr(qn), qp.stride(0), _stream(stream)))
    return qp, qn


def quantize_activations_combined(x: torch.Tensor, kseg: Sequence[int], s_pos: torch.Tensor,
                                  s_neg: torch.Tensor, out: Optional[torch.Tensor] = None,
                                  stream=None) -> torch.Tensor:
    """DualScale codes in one byte per activation: c = q+ + q-, int8 [M, K]
    (row stride a multiple of 16); q+ = max(c, 0), q- = min(c, 0)."""
    _check_2d(x, "x")
    M, K = x.shape
    if out is None:
        ldc = (K + 15) // 16 * 16
        out = torch.empty((M, ldc), dtype=torch.int8, device=x.device)[:, :K]
    seg, keep = _lib.segments(kseg)
    _lib.check("sq_quantize_activations_combined", _lib.load().sq_quantize_activations_combined(
        _ptr(x), _dtype_code(x.dtype), M, K, x.stride(0), ctypes.byref(seg), _ptr(s_pos),
        _ptr(s_neg), _ptr(out), out.stride(0), _stream(stream)))
    return out


def _act_code(act: str) -> int:
    if act == "silu":
        return _lib.SQ_ACT_SILU
    if act == "gelu":
        return _lib.SQ_ACT_GELU
    raise ValueError(f"unknown activation {act!r}: 'silu' or 'gelu'")


def calibrate_act(z: torch.Tensor, act: str, kseg: Sequence[int],
                  s_pos: Optional[torch.Tensor] = None, s_neg: Optional[torch.Tensor] = None,
                  stream=None):
    """Static DualScale scales (s+, s-) fp32 [J] of X = act(z) over the
    calibration rows of the pre-activation ``z`` [rows, K]; act: 'silu' or 'gelu'."""
    _check_2d(z, "z")
    J = len(kseg) - 1
    if s_pos is None:
        s_pos = torch.empty(J, dtype=torch.float32, device=z.device)
    if s_neg is None:
        s_neg = torch.empty(J, dtype=torch.float32, device=z.device)
    seg, keep = _lib.segments(kseg)
    _lib.check("sq_calibrate_act", _lib.load().sq_calibrate_act(
        _ptr(z), _dtype_code(z.dtype), _act_code(act), z.shape[0], z.shape[1], z.stride(0),
        ctypes.byref(seg), _ptr(s_pos), _ptr(s_neg), _stream(stream)))
    return s_pos, s_neg


def quantize_activations_combined_act(z: torch.Tensor, act: str, kseg: Sequence[int],
                                      s_pos: torch.Tensor, s_neg: torch.Tensor,
                                      out: Optional[torch.Tensor] = None,
                                      stream=None) -> torch.Tensor:
    """Combined DualScale codes of X = act(z) (X rounded once to bf16, never
    stored), int8 [M, K] with row stride a multiple of 16; act: 'silu' or 'gelu'."""
    _check_2d(z, "z")
    M, K = z.shape
    if out is None:
        ldc = (K + 15) // 16 * 16
        out = torch.empty((M, ldc), dtype=torch.int8, device=z.device)[:, :K]
    seg, keep = _lib.segments(kseg)
    _lib.check("sq_quantize_activations_combined_act",
               _lib.load().sq_quantize_activations_combined_act(
                   _ptr(z), _dtype_code(z.dtype), _act_code(act), M, K, z.stride(0),
                   ctypes.byref(seg), _ptr(s_pos), _ptr(s_neg), _ptr(out), out.stride(0),
                   _stream(stream)))
    return out


def linear_from_combined(c: torch.Tensor, qw: QuantizedWeight, s_pos: torch.Tensor,
                         s_neg: torch.Tensor, bias: Optional[torch.Tensor] = None,
                         out_dtype: torch.dtype = torch.bfloat16,
                         out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Forward from combined DualScale codes (same result as ``linear``); int8 weights."""
    _check_2d(c, "c")
    M, K = c.shape
    if out is None:
        out = torch.empty((M, qw.N), dtype=out_dtype, device=c.device)
    _check_2d(out, "out")
    cw, keep = qw.c_struct()
    _lib.check("sq_linear_forward_combined", _lib.load().sq_linear_forward_combined(
        _ptr(c), c.stride(0), M, K, ctypes.byref(cw), _ptr(s_pos), _ptr(s_neg), _ptr(bias),
        _ptr(out), _dtype_code(out.dtype), out.stride(0), _stream(stream)))
    return out


def quantize_activations_single(x: torch.Tensor, kseg: Sequence[int], s_pos: torch.Tensor,
                                s_neg: torch.Tensor, out: Optional[torch.Tensor] = None,
                                stream=None) -> torch.Tensor:
    """Single-scale baseline codes, int8 [M, K]: one symmetric scale per K
    segment, s = max(s_pos, s_neg) (= max|x| / 127 of the calibration rows)."""
    _check_2d(x, "x")
    M, K = x.shape
    if out is None:
        ldc = (K + 15) // 16 * 16
        out = torch.empty((M, ldc), dtype=torch.int8, device=x.device)[:, :K]
    seg, keep = _lib.segments(kseg)
    _lib.check("sq_quantize_activations_single", _lib.load().sq_quantize_activations_single(
        _ptr(x), _dtype_code(x.dtype), M, K, x.stride(0), ctypes.byref(seg), _ptr(s_pos),
        _ptr(s_neg), _ptr(out), out.stride(0), _stream(stream)))
    return out


def linear_from_single(c: torch.Tensor, qw: QuantizedWeight, s_pos: torch.Tensor,
                       s_neg: torch.Tensor, bias: Optional[torch.Tensor] = None,
                       out_dtype: torch.dtype = torch.bfloat16,
                       out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Single-scale baseline forward from ``quantize_activations_single`` codes (int8 weights)."""
    _check_2d(c, "c")
    M, K = c.shape
    if out is None:
        out = torch.empty((M, qw.N), dtype=out_dtype, device=c.device)
    _check_2d(out, "out")
    cw, keep = qw.c_struct()
    _lib.check("sq_linear_forward_single", _lib.load().sq_linear_forward_single(
        _ptr(c), c.stride(0), M, K, ctypes.byref(cw), _ptr(s_pos), _ptr(s_neg), _ptr(bias),
        _ptr(out), _dtype_code(out.dtype), out.stride(0), _stream(stream)))
    return out


def splitk_workspace_size(M: int, N: int, K: int) -> int:
    """Bytes of workspace ``linear_from_codes_splitk`` needs on the current device."""
    n = ctypes.c_size_t()
    _lib.check("sq_splitk_workspace_size",
               _lib.load().sq_splitk_workspace_size(M, N, K, ctypes.byref(n)))
    return n.value


def splitk_workspace(M: int, N: int, K: int, device=None) -> torch.Tensor:
    """A zeroed workspace for ``linear_from_codes_splitk`` (uint8, 256-byte aligned)."""
    return torch.zeros(splitk_workspace_size(M, N, K), dtype=torch.uint8, device=device)


def linear_from_codes_splitk(q_pos: torch.Tensor, q_neg: torch.Tensor, qw: QuantizedWeight,
                             s_pos: torch.Tensor, s_neg: torch.Tensor, workspace: torch.Tensor,
                             bias: Optional[torch.Tensor] = None,
                             out_dtype: torch.dtype = torch.bfloat16,
                             out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Small-M (M <= 128) forward from DualScale codes, K split across the GPU;
    bit-identical to ``linear_from_codes``.  ``workspace`` from ``splitk_workspace``
    (its counters return to zero after every completed call)."""
    _check_2d(q_pos, "q_pos")
    _check_2d(q_neg, "q_neg")
    M, K = q_pos.shape
    if q_neg.shape != q_pos.shape or q_neg.stride(0) != q_pos.stride(0):
        raise ValueError("q_pos and q_neg must have the same shape and row stride")
    if out is None:
        out = torch.empty((M, qw.N), dtype=out_dtype, device=q_pos.device)
    _check_2d(out, "out")
    c, keep = qw.c_struct()
    _lib.check("sq_linear_forward_codes_splitk", _lib.load().sq_linear_forward_codes_splitk(
        _ptr(q_pos), _ptr(q_neg), q_pos.stride(0), M, K, ctypes.byref(c), _ptr(s_pos), _ptr(s_neg),
        _ptr(bias), _ptr(out), _dtype_code(out.dtype), out.stride(0), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream)))
    return out


def num_units(qw: QuantizedWeight) -> int:
    return len(qw.kseg) - 1 if qw.bits == 8 else qw.K // 128


def linear_accumulators(x: torch.Tensor, qw: QuantizedWeight, s_pos: torch.Tensor,
                        s_neg: torch.Tensor, stream=None) -> torch.Tensor:
    """Raw int32 accumulators [U, 2, M, N] of the fused kernel (test surface)."""
    _check_2d(x, "x")
    M, K = x.shape
    acc = torch.empty((num_units(qw), 2, M, qw.N), dtype=torch.int32, device=x.device)
    c, keep = qw.c_struct()
    _lib.check("sq_linear_accumulators", _lib.load().sq_linear_accumulators(
        _ptr(x), _dtype_code(x.dtype), M, K, x.stride(0), ctypes.byref(c), _ptr(s_pos),
        _ptr(s_neg), _ptr(acc), _stream(stream)))
    return acc


def stream_status(stream=None) -> int:
    """Synchronize the stream and return (and clear) the device status word."""
    return int(_lib.load().sq_stream_status(_stream(stream)))


def set_wait_budget(cycles: int) -> None:
    """Test hook of the development library (inside ``_lib.dev_library()``):
    device-side pipeline wait budget in SM clock cycles (0 = default, ~1 s)."""
    _lib.check("sq_set_wait_budget", _lib.load().sq_set_wait_budget(int(cycles)))


def debug_starve_pipeline(enable: bool) -> None:
    """Test hook of the development library: GEMM launches issue no TMA
    copies, so their waits expire."""
    _lib.check("sq_debug_starve_pipeline", _lib.load().sq_debug_starve_pipeline(1 if enable else 0))


# ------------------------------------------------- block-Hadamard activations
# HQ-DM ("HQ-DM: Single Hadamard Transformation-Based Quantization-Aware
# Training for Low-Bit Diffusion Models", Spanish technical summary 2.1):
# activations times a block-diagonal Hadamard matrix (blocks of 16 along K)
# before quantization; int4 weights quantized untransformed; the forward is the
# integer product of the XH codes with the int4 codes rotated into the same
# basis, the block normalization 1/4 carried by the activation scales.

def calibrate_hadamard(x: torch.Tensor, kseg: Sequence[int], s_pos: Optional[torch.Tensor] = None,
                       s_neg: Optional[torch.Tensor] = None, stream=None):
    """DualScale scales (s+, s-) fp32 [J] of the transformed calibration rows XH."""
    _check_2d(x, "x")
    J = len(kseg) - 1
    if s_pos is None:
        s_pos = torch.empty(J, dtype=torch.float32, device=x.device)
    if s_neg is None:
        s_neg = torch.empty(J, dtype=torch.float32, device=x.device)
    seg, keep = _lib.segments(kseg)
    _lib.check("sq_calibrate_hadamard", _lib.load().sq_calibrate_hadamard(
        _ptr(x), _dtype_code(x.dtype), x.shape[0], x.shape[1], x.stride(0), ctypes.byref(seg),
        _ptr(s_pos), _ptr(s_neg), _stream(stream)))
    return s_pos, s_neg


def quantize_activations_hadamard(x: torch.Tensor, kseg: Sequence[int], s_pos: torch.Tensor,
                                  s_neg: torch.Tensor, out=None, stream=None):
    """DualScale codes (q+, q-) of XH, int8 [M, K] each (row stride a multiple of 16)."""
    _check_2d(x, "x")
    M, K = x.shape
    if out is None:
        ldq = (K + 15) // 16 * 16
        qp = torch.empty((M, ldq), dtype=torch.int8, device=x.device)[:, :K]
        qn = torch.empty((M, ldq), dtype=torch.int8, device=x.device)[:, :K]
    else:
        qp, qn = out
        if qp.stride(0) != qn.stride(0):
            raise ValueError("q_pos and q_neg must share a row stride")
    seg, keep = _lib.segments(kseg)
    _lib.check("sq_quantize_activations_hadamard", _lib.load().sq_quantize_activations_hadamard(
        _ptr(x), _dtype_code(x.dtype), M, K, x.stride(0), ctypes.byref(seg), _ptr(s_pos),
        _ptr(s_neg), _ptr(qp), _ptr(qn), qp.stride(0), _stream(stream)))
    return qp, qn


def rotate_weights_hadamard(qw: QuantizedWeight, out: Optional[torch.Tensor] = None,
                            stream=None) -> torch.Tensor:
    """The int4 codes of ``qw`` rotated into the transform's basis, int8 [N, K]."""
    if qw.bits != 4:
        raise ValueError("the Hadamard forward takes int4 weights")
    if out is None:
        out = torch.empty((qw.N, qw.K), dtype=torch.int8, device=qw.codes.device)
    _check_2d(out, "out")
    c, keep = qw.c_struct()
    _lib.check("sq_rotate_weights_hadamard", _lib.load().sq_rotate_weights_hadamard(
        ctypes.byref(c), _ptr(out), out.stride(0), _stream(stream)))
    return out


def linear_from_codes_hadamard(q_pos: torch.Tensor, q_neg: torch.Tensor, qw: QuantizedWeight,
                               w_rot: torch.Tensor, s_pos: torch.Tensor, s_neg: torch.Tensor,
                               bias: Optional[torch.Tensor] = None,
                               out_dtype: torch.dtype = torch.bfloat16,
                               out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Forward from the XH codes and the rotated int4 weight codes."""
    _check_2d(q_pos, "q_pos")
    _check_2d(q_neg, "q_neg")
    _check_2d(w_rot, "w_rot")
    M, K = q_pos.shape
    if q_neg.shape != q_pos.shape or q_neg.stride(0) != q_pos.stride(0):
        raise ValueError("q_pos and q_neg must have the same shape and row stride")
    if out is None:
        out = torch.empty((M, qw.N), dtype=out_dtype, device=q_pos.device)
    _check_2d(out, "out")
    c, keep = qw.c_struct()
    _lib.check("sq_linear_forward_codes_hadamard", _lib.load().sq_linear_forward_codes_hadamard(
        _ptr(q_pos), _ptr(q_neg), q_pos.stride(0), M, K, ctypes.byref(c), _ptr(w_rot),
        w_rot.stride(0), _ptr(s_pos), _ptr(s_neg), _ptr(bias), _ptr(out), _dtype_code(out.dtype),
        out.stride(0), _stream(stream)))
    return out
