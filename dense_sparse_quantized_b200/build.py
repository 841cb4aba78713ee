"""Build step of libdsq.so (sm_100a) with nvcc, in-tree.

    python -m dense_sparse_quantized_b200.build [--debug]

Compiles every ``csrc/*.cu`` into ``libdsq.so`` beside this file.  No GPU is
needed: nvcc cross-compiles for sm_100a.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIBRARY = os.path.join(HERE, "libdsq.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
         "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden", "-shared",
         "--expt-relaxed-constexpr"]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def headers():
    return sorted(glob.glob(os.path.join(CSRC, "*.h")) +
                  glob.glob(os.path.join(HERE, "..", "include", "*.h")))


def stale() -> bool:
    if not os.path.exists(LIBRARY):
        return True
    t = os.path.getmtime(LIBRARY)
    return any(os.path.getmtime(f) > t for f in sources() + headers())


def build(debug: bool = False, verbose: bool = False) -> str:
    cmd = [NVCC] + FLAGS + (["-DDSQ_DEBUG"] if debug else []) + sources() + ["-o", LIBRARY]
    if verbose:
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    return LIBRARY


if __name__ == "__main__":
    build(debug="--debug" in sys.argv, verbose=True)
