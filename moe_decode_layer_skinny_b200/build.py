"""Build libkd.so (the sm_100a CUDA library) in-tree with nvcc."""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SO = os.path.join(HERE, "libkd.so")
NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17", "-lineinfo",
              "-Xcompiler", "-fPIC", "-shared"]


def sources() -> list[str]:
    return (sorted(glob.glob(os.path.join(HERE, "csrc", "*.cu"))) +
            sorted(glob.glob(os.path.join(HERE, "csrc", "*.cuh"))) +
            [os.path.join(ROOT, "include", "kd.h"), os.path.join(ROOT, "kdgen", "kd_gen.h")])


def stale() -> bool:
    if not os.path.exists(SO):
        return True
    t = os.path.getmtime(SO)
    return any(os.path.getmtime(s) > t for s in sources())


def build(force: bool = False, verbose: bool = False) -> str:
    if not (force or stale()):
        return SO
    nvcc = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
    cmd = [nvcc, *NVCC_FLAGS, "-o", SO, os.path.join(HERE, "csrc", "kd_layer.cu"),
           os.path.join(HERE, "csrc", "kd_static.cu")]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.check_call(cmd)
    return SO


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
