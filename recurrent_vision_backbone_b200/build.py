"""Build the CUDA library in-tree: recurrent_vision_backbone_b200/libgtr_gla.so.

Compiles csrc/gtr_gla.cu for sm_100a only (nvcc cross-compiles without a GPU):
    python -m recurrent_vision_backbone_b200.build [--verbose]
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
SOURCES = [os.path.join(CSRC, "gtr_gla.cu")]
DEPS = SOURCES + [os.path.join(CSRC, n) for n in ("sm100_ptx.cuh", "gla_fwd_span.cuh", "gla_fwd_pipe.cuh", "swiglu_gate.cuh", "gla_bwd.cuh")]
DEPS += [os.path.join(ROOT, "include", n) for n in ("gtr_gla.h", "gtr_swiglu.h", "gtr_gla_bwd.h")]
LIB = os.path.join(HERE, "libgtr_gla.so")


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def nvcc_cmd(out: str = LIB, extra=()) -> list:
    return [nvcc_path(), "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3",
            "-std=c++17", "--shared", "-Xcompiler", "-fPIC", "-I", os.path.join(ROOT, "include"),
            *extra, *SOURCES, "-o", out, "-lcudart"]


def is_stale(out: str = LIB) -> bool:
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    return any(os.path.getmtime(d) > t for d in DEPS)


def build(force: bool = False, verbose: bool = False) -> str:
    if force or is_stale():
        extra = ["-Xptxas", "-v"] if verbose else []
        tmp = LIB + ".tmp"
        subprocess.run(nvcc_cmd(tmp, extra), check=True)
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True, verbose="--verbose" in sys.argv))
