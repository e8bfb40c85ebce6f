"""Build libsla.so (the C-ABI library) in-tree with nvcc for sm_100a."""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libsla.so")
SOURCES = ["api.cu", "route.cu", "route_noalloc.cu", "prepare.cu", "sparse_fwd.cu", "labels.cu", "backward.cu", "backward_tc.cu"]
HEADERS = ["sla_device.cuh", "sla_internal.h", "sla_kernels.h"]
NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
]


def _nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    deps.append(os.path.join(HERE, "..", "include", "sla.h"))
    return any(os.path.getmtime(p) > t for p in deps)


def build(verbose: bool = False, extra=None) -> str:
    cmd = [_nvcc(), *NVCC_FLAGS, *(extra or []), "-o", LIB + ".tmp",
           *[os.path.join(CSRC, f) for f in SOURCES], "-ldl", "-lpthread", "-lrt"]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True, cwd=CSRC)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    build(verbose=True, extra=sys.argv[1:])
    print(LIB)
