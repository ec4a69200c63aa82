"""Build libnq.so (the CUDA library behind include/nq.h) in-tree for sm_100a.

    python -m e8_lattice_vector_nq_b200.build [--force]

Flags: -gencode arch=compute_100a,code=sm_100a -O3 -lineinfo -fmad=false.
-fmad=false keeps every unfused multiply-add of the kernels rounded exactly
as written (each fused one is an explicit fmaf/__fmaf_rn).
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
SO = os.path.join(HERE, "libnq.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17", "-fmad=false",
    "-Xcompiler", "-fPIC", "-shared",
    "-Xptxas", "-v",
]


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def deps() -> list[str]:
    return sources() + sorted(glob.glob(os.path.join(CSRC, "*.h*"))) + [
        os.path.join(HERE, "..", "include", "nq.h")]


def build(force: bool = False, verbose: bool = False) -> str:
    stale = not os.path.exists(SO) or any(os.path.getmtime(d) > os.path.getmtime(SO) for d in deps())
    if not (force or stale):
        return SO
    tmp = SO + f".tmp{os.getpid()}"
    cmd = [NVCC, *NVCC_FLAGS, *sources(), "-o", tmp]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError("nvcc failed building libnq.so")
    with open(os.path.join(HERE, "libnq.ptxas.txt"), "w") as f:
        f.write(res.stderr)
    if verbose:
        sys.stderr.write(res.stderr)
    os.replace(tmp, SO)
    return SO


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
