"""Builds libmoe_decode.so in-tree for sm_100a with nvcc (no JIT cache)."""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libmoe_decode.so")
SOURCES = ["kernels.cu", "kernels_small.cu", "kernels_layer.cu", "kernels_router.cu", "kernels_large.cu",
           "kernels_tc.cu", "moe_decode.cu", "static_step.cu"]
HEADERS = ["common.cuh", "kernels.cuh", "gemv_mma.cuh", "topk.cuh", "rowdot.cuh", "mma.cuh"]

NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
              "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden", "--expt-relaxed-constexpr"]


def _stale(out: str, deps: list[str]) -> bool:
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    return any(os.path.getmtime(p) > t for p in deps)


def build(force: bool = False, verbose: bool = False, extra: list[str] | None = None) -> str:
    srcs = [os.path.join(CSRC, s) for s in SOURCES]
    deps = srcs + [os.path.join(CSRC, h) for h in HEADERS] + [os.path.join(ROOT, "include", "moe_decode.h")]
    if not (force or _stale(LIB, deps)):
        return LIB
    cmd = ["nvcc", *NVCC_FLAGS, *(extra or []), "-shared", "-o", LIB, *srcs]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.check_call(cmd)
    return LIB


if __name__ == "__main__":
    v = "-v" in sys.argv
    build(force=True, verbose=True, extra=["-Xptxas", "-v"] if v else None)
    print(LIB)
