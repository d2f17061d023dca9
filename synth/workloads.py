"""Seeded synthetic workloads for the DualScale / SegLinear quantized linear.

This module only draws inputs: random activations shaped like the diffusion
transformer layers the SegQuant summaries evaluate on (SD3.5 / FLUX.1 / DiT
MLP and attention projections), random weights and biases.  It holds none of
the quantization arithmetic, so both the CUDA path and the CPU oracle can take
their inputs from it.

Readings of the workload text (stated once, used everywhere):
  * N(mu, v): for the unit-normal pre-activations and the weight and bias
    draws (N(0,1), N(0,0.02), N(0,0.05), N(0,0.01)) the second parameter is
    the standard deviation (the usual initialization convention); the two
    perfect squares -- the timestep-feature segment N(0,25) and the outliers
    N(0,400) -- are read as variances, sigma = 5 and sigma = 20.  A literal
    standard-deviation reading of those two (sigma = 25, 400) would change the
    value spread only, not the work or the parity checks.
  * GELU is the exact (erf) GELU.
  * Activations are produced in fp32 by the activation function and then
    rounded once to the storage dtype (bf16 where the workload says bf16).
  * Draw order from one torch.Generator seeded with the case seed:
    X pre-activation -> W -> bias -> outlier positions -> outlier values.
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional, Tuple

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    M: int
    K: int
    N: int
    x_dtype: str                      # "f32" | "bf16"
    act: str                          # "silu" | "gelu"
    x_sigma: Tuple[Tuple[int, int, float], ...]   # (k0, k1, sigma) of the pre-activation
    w_sigma: Tuple[Tuple[int, int, float], ...]   # (n0, n1, sigma) of the weights
    bits: int                         # 8 | 4
    kseg: Tuple[int, ...]             # K-segment bounds (J+1 entries)
    nseg: Tuple[int, ...]             # N-segment bounds (metadata)
    bias_sigma: Optional[float]       # None = no bias
    out: str                          # "f32" | "bf16"
    calib_rows: Optional[int] = None  # calibrate on rows [0, calib_rows); None = all rows
    outlier_frac: float = 0.0
    outlier_sigma: float = 0.0
    seed: int = 0
    description: str = ""

    @property
    def exec_ops(self) -> int:
        """Executed int8 operations: two GEMMs (one per polarity), 2 ops per MAC."""
        return 4 * self.M * self.N * self.K

    def alg_bytes(self) -> int:
        """Algorithmic HBM bytes of one forward: X + weight codes + weight scales +
        activation scales + bias + Y."""
        xe = 4 if self.x_dtype == "f32" else 2
        ye = 4 if self.out == "f32" else 2
        J = len(self.kseg) - 1
        if self.bits == 8:
            wb = self.N * self.K + 4 * J * self.N
        else:
            wb = self.N * self.K // 2 + 2 * self.N * (self.K // 128)
        bb = 4 * self.N if self.bias_sigma is not None else 0
        return self.M * self.K * xe + wb + 8 * J + bb + self.M * self.N * ye


WORKLOADS = {
    "tiny_w8a8": Workload(
        name="tiny_w8a8", M=64, K=256, N=256, x_dtype="f32", act="silu",
        x_sigma=((0, 256, 1.0),), w_sigma=((0, 256, 0.02),), bits=8,
        kseg=(0, 256), nseg=(0, 256), bias_sigma=0.01, out="f32",
        description="tiny W8A8 DualScale linear, fp32 in/out, bias"),
    "dit_xl2_fc2_cfg": Workload(
        name="dit_xl2_fc2_cfg", M=8192, K=4608, N=1152, x_dtype="bf16", act="gelu",
        x_sigma=((0, 4608, 1.0),), w_sigma=((0, 1152, 0.02),), bits=8,
        kseg=(0, 4608), nseg=(0, 1152), bias_sigma=None, out="bf16", calib_rows=512,
        description="DiT-XL/2 MLP fc2, CFG-doubled batch 2x16x256 tokens, W8A8"),
    "seglinear_qkv": Workload(
        name="seglinear_qkv", M=8192, K=2304, N=3456, x_dtype="bf16", act="silu",
        x_sigma=((0, 1152, 1.0), (1152, 2304, 5.0)),
        w_sigma=((0, 1152, 0.02), (1152, 2304, 0.05), (2304, 3456, 0.02)), bits=8,
        kseg=(0, 1152, 2304), nseg=(0, 1152, 2304, 3456), bias_sigma=None, out="bf16",
        description="SegLinear: latent | timestep-embedding K segments, q/k/v N segments"),
    "mmdit_mlp_up": Workload(
        name="mmdit_mlp_up", M=16384, K=3072, N=12288, x_dtype="bf16", act="silu",
        x_sigma=((0, 3072, 1.0),), w_sigma=((0, 12288, 0.02),), bits=8,
        kseg=(0, 3072), nseg=(0, 12288), bias_sigma=None, out="bf16",
        outlier_frac=0.001, outlier_sigma=20.0,
        description="MMDiT MLP up-projection, 1024^2 image, CFG-doubled batch 2, 0.1% outliers"),
    "w4a8": Workload(
        name="w4a8", M=16384, K=3072, N=3072, x_dtype="bf16", act="silu",
        x_sigma=((0, 3072, 1.0),), w_sigma=((0, 3072, 0.02),), bits=4,
        kseg=(0, 3072), nseg=(0, 3072), bias_sigma=None, out="bf16",
        description="W4A8: int4 weights group 128 fp16 scales, int8 DualScale activations"),
}


def _act(z: torch.Tensor, act: str) -> torch.Tensor:
    if act == "silu":
        return torch.nn.functional.silu(z)
    if act == "gelu":
        return torch.nn.functional.gelu(z, approximate="none")
    if act == "none":
        return z
    raise ValueError(act)


def generate(wl: Workload, rows: Optional[Tuple[int, int]] = None):
    """Draw (x, w, bias) for a workload on the CPU.

    x: [M, K] torch.float32 or torch.bfloat16; w: [N, K] float32; bias: [N]
    float32 or None.  ``rows`` is accepted for API symmetry but the full
    matrix is always drawn so that every row is identical whatever the caller
    later slices."""
    g = torch.Generator(device="cpu")
    g.manual_seed(wl.seed)
    z = torch.randn(wl.M, wl.K, generator=g, dtype=torch.float32)
    for k0, k1, sig in wl.x_sigma:
        if sig != 1.0:
            z[:, k0:k1] *= sig
    x = _act(z, wl.act)
    del z
    w = torch.randn(wl.N, wl.K, generator=g, dtype=torch.float32)
    for n0, n1, sig in wl.w_sigma:
        w[n0:n1] *= sig
    bias = None
    if wl.bias_sigma is not None:
        bias = torch.randn(wl.N, generator=g, dtype=torch.float32) * wl.bias_sigma
    if wl.outlier_frac > 0:
        total = wl.M * wl.K
        count = int(round(wl.outlier_frac * total))
        pos = torch.randperm(total, generator=g)[:count]
        vals = torch.randn(count, generator=g, dtype=torch.float32) * wl.outlier_sigma
        x.view(-1)[pos] = vals
    if wl.x_dtype == "bf16":
        x = x.to(torch.bfloat16)
    return x, w, bias


def small_case(M: int, K: int, N: int, *, seed: int, x_dtype: str = "bf16", act: str = "silu",
               kseg: Optional[List[int]] = None, x_sigmas: Optional[List[float]] = None,
               bits: int = 8, bias: bool = True, out: str = "bf16") -> Workload:
    """A seeded ad-hoc workload used by the parity tests (ragged shapes, several
    segments, both weight formats)."""
    kseg = tuple(kseg or (0, K))
    J = len(kseg) - 1
    sig = x_sigmas or [1.0] * J
    return Workload(
        name=f"case_M{M}_K{K}_N{N}_s{seed}", M=M, K=K, N=N, x_dtype=x_dtype, act=act,
        x_sigma=tuple((kseg[j], kseg[j + 1], float(sig[j])) for j in range(J)),
        w_sigma=((0, N, 0.02),), bits=bits, kseg=kseg, nseg=(0, N),
        bias_sigma=0.01 if bias else None, out=out, seed=seed)


def to_numpy_x(x: torch.Tensor):
    """Host copy of x in the oracle's convention (fp32 values or bf16 bit patterns)."""
    if x.dtype == torch.bfloat16:
        return x.contiguous().view(torch.int16).numpy().view("uint16")
    return x.contiguous().numpy()


def calib_slice(wl: Workload, x: torch.Tensor) -> torch.Tensor:
    return x if wl.calib_rows is None else x[: wl.calib_rows]
