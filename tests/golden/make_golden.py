"""Writes the regression fixtures of this directory from the oracle alone.

Run from the repository root: ``python tests/golden/make_golden.py``.  Inputs
come from the seeded synthetic generator (synth/workloads.py); every stored
value is computed by ``oracle/`` (test infrastructure), never by the CUDA path.

Fixtures:
  * dualscale_w8_two_segments.txt -- SegQuant DualScale with SegLinear input
    segments ("SegQuant: A Semantics-Aware and Generalizable Quantization
    Framework for Diffusion Models", Spanish technical summary 2.A and 2.B):
    per-segment scales, codes, per-unit int32 accumulators and fp32 outputs;
  * hadamard_w4.txt -- the block-Hadamard variant with int4 weights ("HQ-DM:
    Single Hadamard Transformation-Based Quantization-Aware Training for
    Low-Bit Diffusion Models", Spanish technical summary 2.1): scales of XH,
    rotated weight codes, accumulators and fp32 outputs.
Floats are stored as the hexadecimal bit patterns of their fp32 values."""
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle as O                      # noqa: E402
from synth import workloads as W       # noqa: E402

CASES = {
    "dualscale_w8_two_segments": dict(M=4, K=256, N=16, seed=901, kseg=[0, 128, 256],
                                      x_sigmas=[1.0, 6.0], bits=8),
    "hadamard_w4": dict(M=3, K=256, N=16, seed=902, kseg=[0, 256], x_sigmas=None, bits=4),
}


def case_workload(name):
    p = dict(CASES[name])
    return W.small_case(p.pop("M"), p.pop("K"), p.pop("N"), seed=p.pop("seed"), kseg=p.pop("kseg"),
                        x_sigmas=p.pop("x_sigmas"), bits=p.pop("bits"), x_dtype="bf16", out="f32")


def compute(name):
    """The fixture's arrays, from the oracle."""
    wl = case_workload(name)
    x, w, b = W.generate(wl)
    xn, wn, bn = W.to_numpy_x(x), w.numpy(), b.numpy()
    if name == "hadamard_w4":
        sp, sn = O.calibrate_hadamard(xn, wl.kseg)
        packed, scales = O.quantize_weights_w4(wn)
        y, acc, (qp, qn), rot = O.linear_forward_hadamard(xn, wl.kseg, sp, sn, packed, scales, bn,
                                                          out="f32", return_acc=True)
        return dict(s_pos=sp, s_neg=sn, w_rot=rot, q_pos=qp, q_neg=qn, acc=acc, y=y)
    sp, sn = O.calibrate(xn, wl.kseg)
    wc, ws = O.quantize_weights_w8(wn, wl.kseg)
    y, acc, (qp, qn) = O.linear_forward(xn, wl.kseg, sp, sn, 8, wc, ws, bn, out="f32",
                                        return_acc=True)
    return dict(s_pos=sp, s_neg=sn, w_codes=wc, w_scales=ws, q_pos=qp, q_neg=qn, acc=acc, y=y)


def encode(arr) -> str:
    a = np.asarray(arr)
    if a.dtype == np.float32:
        body = " ".join(f"{v:08x}" for v in a.reshape(-1).view(np.uint32))
        kind = "f32hex"
    else:
        body = " ".join(str(int(v)) for v in a.reshape(-1))
        kind = "int"
    return f"{kind} {' '.join(str(d) for d in a.shape)} : {body}"


def decode(line: str):
    head, body = line.split(":", 1)
    parts = head.split()
    kind, shape = parts[0], tuple(int(d) for d in parts[1:])
    vals = body.split()
    if kind == "f32hex":
        return np.array([int(v, 16) for v in vals], np.uint32).view(np.float32).reshape(shape)
    return np.array([int(v) for v in vals], np.int64).reshape(shape)


def read(name):
    out = {}
    with open(os.path.join(HERE, name + ".txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            key, rest = line.split(" ", 1)
            out[key] = decode(rest.strip())
    return out


def main():
    for name in CASES:
        arrays = compute(name)
        with open(os.path.join(HERE, name + ".txt"), "w") as f:
            f.write(f"# {name}: written by tests/golden/make_golden.py from oracle/ only\n")
            f.write(f"# case {CASES[name]}, bf16 activations, fp32 output, bias on\n")
            for key, arr in arrays.items():
                f.write(f"{key} {encode(arr)}\n")


if __name__ == "__main__":
    main()
