"""Build the CUDA library libqspec.so in-tree for sm_100a.

Usage: python -m quantized_speculative_decoding_packed_b200.build [--verbose-ptxas]
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG_DIR)
CSRC = os.path.join(PKG_DIR, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG_DIR, "libqspec.so")
SOURCES = [os.path.join(CSRC, "qspec_api.cu")]
DEPENDS = SOURCES + [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cuh")] + [
    os.path.join(INCLUDE, "qspec.h")]


def nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(f) > t for f in DEPENDS)


def build(force: bool = False, verbose_ptxas: bool = False, trace: bool = False) -> str:
    """trace=True builds libqspec_trace.so, a debug variant with per-warp
    checkpoints and software alignment checks (never loaded by the package)."""
    out = LIB.replace("libqspec.so", "libqspec_trace.so") if trace else LIB
    if not force and not trace and not needs_build() and not verbose_ptxas:
        return LIB
    cmd = [nvcc(), "-std=c++17", "-O3", "-lineinfo", "--shared", "-Xcompiler", "-fPIC",
           "-gencode", "arch=compute_100a,code=sm_100a", "-I", INCLUDE, "-I", CSRC,
           "-o", out] + SOURCES
    if trace:
        cmd += ["-DQSPEC_TRACE", "-rdc=false"]
    if verbose_ptxas:
        cmd += ["-Xptxas", "-v"]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + res.stdout + res.stderr)
    if verbose_ptxas:
        sys.stdout.write(res.stdout + res.stderr)
    return out


if __name__ == "__main__":
    print(build(force=True, verbose_ptxas="--verbose-ptxas" in sys.argv, trace="--trace" in sys.argv))
