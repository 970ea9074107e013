"""Builds libtq.so in-tree with nvcc for sm_100a (B200).

Usage: ``python embedding_vector_quantization_b200/build.py [--force] [-v]`` (a plain script:
it does not import the package, so a stale library is never loaded first).
The shared library lands next to this file so the Python binding (and any
copy of the repository) finds it without installation.
"""

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libtq.so")
SOURCES = ["tq_api.cu", "tq_noalloc.cu", "host_math.cpp"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _nvcc():
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def _newest_source_mtime():
    newest = 0.0
    for dirpath in (CSRC, os.path.join(ROOT, "include")):
        for name in os.listdir(dirpath):
            if name.endswith((".cu", ".cuh", ".cpp", ".h")):
                newest = max(newest, os.path.getmtime(os.path.join(dirpath, name)))
    return newest


def build(force: bool = False, verbose: bool = False) -> str:
    """Compiles libtq.so if missing or older than any source; returns its path."""
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= _newest_source_mtime():
        return LIB
    cmd = [_nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
           "-Xcompiler", "-O3", "--expt-relaxed-constexpr",
           "-I", os.path.join(ROOT, "include"), "-I", CSRC,
           *[os.path.join(CSRC, s) for s in SOURCES], "-o", LIB + ".tmp"]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(LIB)
