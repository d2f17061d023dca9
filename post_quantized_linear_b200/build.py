"""Builds the sm_100a shared library ``libsegquant.so`` in-tree with nvcc.

Usage: ``python -m post_quantized_linear_b200.build [--force] [--verbose-ptxas]``.
"""
from __future__ import annotations

import argparse
import glob
import os
import shutil
import subprocess
import sys

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG_DIR)
CSRC = os.path.join(PKG_DIR, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB_PATH = os.path.join(PKG_DIR, "libsegquant.so")
# Development build: the same sources with SQ_DEV_BUILD (environment switches
# for the measured alternative kernels, live test hooks), for the tests.
DEV_LIB_PATH = os.path.join(PKG_DIR, "libsegquant_dev.so")

ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc_path() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else (shutil.which("nvcc") or "nvcc")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh")) +
                  glob.glob(os.path.join(INCLUDE, "*.h")))


def _build_one(path: str, defines, force: bool, ptxas_verbose: bool) -> str:
    newest = max(os.path.getmtime(p) for p in sources())
    if not force and os.path.exists(path) and os.path.getmtime(path) >= newest:
        return path
    tmp = path + f".tmp{os.getpid()}"
    cmd = [nvcc_path(), *ARCH_FLAGS, "-O3", "-lineinfo", "-std=c++17", "--shared",
           "-Xcompiler", "-fPIC", "-Xcompiler", "-O2", "-I", INCLUDE, "-I", CSRC, *defines,
           os.path.join(CSRC, "segquant.cu"), "-o", tmp]
    if ptxas_verbose:
        cmd[1:1] = ["-Xptxas", "-v"]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError(f"nvcc failed building {os.path.basename(path)}")
    if ptxas_verbose:
        sys.stdout.write(res.stdout + res.stderr)
    os.replace(tmp, path)
    return path


def build(force: bool = False, ptxas_verbose: bool = False, dev: bool = True) -> str:
    """Build libsegquant.so and (dev=True) libsegquant_dev.so, in parallel."""
    import concurrent.futures as cf
    jobs = [(LIB_PATH, [])] + ([(DEV_LIB_PATH, ["-DSQ_DEV_BUILD"])] if dev else [])
    with cf.ThreadPoolExecutor(max_workers=len(jobs)) as ex:
        futs = [ex.submit(_build_one, p, d, force, ptxas_verbose) for p, d in jobs]
        for f in futs:
            f.result()
    return LIB_PATH


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose-ptxas", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, ptxas_verbose=a.verbose_ptxas))
