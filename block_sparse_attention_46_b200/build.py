"""Builds liblf.so (the C-ABI library) in-tree with nvcc for sm_100a.

    python -m block_sparse_attention_46_b200.build [--verbose]

The library is a single translation unit (csrc/lf_api.cu includes the kernel headers),
linked against the CUDA runtime only; the tensor-map encoder is resolved at run time
through cudaGetDriverEntryPoint, so no link against libcuda is needed.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "liblf.so")
SOURCES = ["lf_api.cu"]
DEPS = ["lf_api.cu", "lf_common.cuh", "lf_select.cuh", "lf_attn.cuh", "lf_fused.cuh", "lf_fp8.cuh"]


def nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def flags(verbose: bool = False):
    f = ["-O3", "-std=c++17", "-lineinfo", "-gencode", "arch=compute_100a,code=sm_100a",
         "-Xcompiler", "-fPIC", "-shared", "-I", os.path.join(ROOT, "include"),
         "--expt-relaxed-constexpr"]
    if verbose:
        f += ["-Xptxas", "-v"]
    return f


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    srcs = [os.path.join(CSRC, s) for s in DEPS] + [os.path.join(ROOT, "include", "lf.h")]
    return any(os.path.getmtime(s) > t for s in srcs)


def build(verbose: bool = False, force: bool = False) -> str:
    if not force and not stale():
        return LIB
    cmd = [nvcc()] + flags(verbose) + [os.path.join(CSRC, s) for s in SOURCES] + \
          ["-o", LIB + ".tmp", "-cudart", "static"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + " ".join(cmd) + "\n" + r.stdout + r.stderr)
    if verbose:
        sys.stderr.write(r.stdout + r.stderr)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(verbose="--verbose" in sys.argv, force=True))
