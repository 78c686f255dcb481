"""Build the C-ABI shared library (libhq.so) in-tree with nvcc for sm_100a.

    python -m quantized_gemm_bit_b200.build [--force]

The library is rebuilt when any source under csrc/ or include/ is newer
than the .so.  Only nvcc and the host compiler are needed (no GPU).
"""

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libhq.so")
SOURCES = ["hq_api.cu", "w4a16.cu", "w4a16_small.cu", "w4a16_reg.cu", "w4a16_static.cu", "blockscaled.cu", "quant.cu", "moe.cu", "hq_pack.cpp"]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = [
    "-O3", "-std=c++17", "-shared", "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
    "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
    "--expt-relaxed-constexpr", "-I", os.path.join(ROOT, "include"),
]


def _inputs():
    files = [os.path.join(CSRC, f) for f in os.listdir(CSRC)]
    files.append(os.path.join(ROOT, "include", "hq.h"))
    return files


def needs_build():
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(f) > t for f in _inputs())


def build(force=False, verbose=False, extra=()):
    if not force and not needs_build():
        return LIB
    tmp = LIB + ".tmp"
    cmd = [NVCC] + FLAGS + list(extra) + ["-o", tmp] + [os.path.join(CSRC, s) for s in SOURCES] + ["-lpthread"]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True,
          extra=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else ())
    print(LIB)
