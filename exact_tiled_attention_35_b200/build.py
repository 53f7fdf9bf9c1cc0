"""Builds libfa.so in this package directory with nvcc for sm_100a.

Usage:  python -m exact_tiled_attention_35_b200.build   (or build() from Python)
"""

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libfa.so")
SOURCES = ["fa_lib.cu"]  # includes fa_api.cu, fa_simt.cu, fa_fwd_sm100.cu, fa_bwd_sm100.cu
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def sources():
    return [os.path.join(CSRC, s) for s in SOURCES if os.path.exists(os.path.join(CSRC, s))]


def up_to_date():
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    deps = sources() + [os.path.join(CSRC, f) for f in os.listdir(CSRC)]
    deps.append(os.path.join(os.path.dirname(HERE), "include", "fa.h"))
    return all(os.path.getmtime(p) <= t for p in deps if os.path.exists(p))


def build(force=False, verbose=False):
    if not force and up_to_date():
        return LIB
    cmd = [
        NVCC, "-shared", "-Xcompiler", "-fPIC",
        "-gencode", "arch=compute_100a,code=sm_100a",
        "-O3", "-lineinfo", "-std=c++17", "--expt-relaxed-constexpr",
        "-I", os.path.join(os.path.dirname(HERE), "include"),
        "-o", LIB + ".tmp",
    ] + sources()
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError("nvcc failed building libfa.so")
    if verbose:
        sys.stderr.write(r.stdout + r.stderr)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(LIB)
