"""Builds libsgq.so in-tree with nvcc for sm_100a (B200).

    python -m activation_sparse_quantized_b200.build [--force] [--verbose]

nvcc cross-compiles without a GPU. The library is linked against the static
CUDA runtime so that it does not depend on which libcudart the Python process
loaded first.
"""
from __future__ import annotations

import argparse
import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB_PATH = os.path.join(PKG, "libsgq.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-ftz=false", "-prec-div=true", "-prec-sqrt=true", "-Xcompiler", "-fPIC",
         "-Xcompiler", "-fvisibility=default", "-shared", "-cudart", "static"]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def headers():
    return sorted(glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))
                  + glob.glob(os.path.join(INCLUDE, "*.h")))


def nvcc():
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.isabs(cand) and os.path.exists(cand) or not os.path.isabs(cand)):
            return cand
    return "nvcc"


def is_stale(out: str = LIB_PATH) -> bool:
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    return any(os.path.getmtime(p) > t for p in sources() + headers() + [__file__])


def build(force: bool = False, verbose: bool = False, out: str = LIB_PATH) -> str:
    """Compile every .cu under csrc/ into one shared library (if stale)."""
    if not force and not is_stale(out):
        return out
    cmd = [nvcc(), *ARCH, *FLAGS, "-I", INCLUDE, *sources(), "-o", out + ".tmp"]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.run(cmd, check=True)
    os.replace(out + ".tmp", out)
    return out


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true", help="print ptxas register/smem usage")
    a = ap.parse_args(argv)
    print(build(force=a.force or a.verbose, verbose=a.verbose))


if __name__ == "__main__":
    sys.exit(main())
