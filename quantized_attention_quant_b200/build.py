"""Builds libsage_b200.so (the C-ABI library) in-tree with nvcc for sm_100a.

    python -m quantized_attention_quant_b200.build [--verbose]

The CUDA runtime is linked statically and libcuda is reached through the
runtime's driver entry points, so the library loads on a machine without a
GPU driver (for symbol checks) and on the B200 machine alike.
"""

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libsage_b200.so")
SOURCES = ["api.cu", "quant.cu", "attn_i8f8.cu", "attn_i8f8_persist.cu", "attn_fp4.cu"]
# the microbenchmarks of include/sage_ubench.h (bench.py --ubench)
UBENCH_LIB = os.path.join(HERE, "libsage_ubench.so")
UBENCH_SOURCES = ["ubench.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-cudart", "static",
         "--expt-relaxed-constexpr"]


def nvcc():
    for c in [os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")]:
        if c and os.path.exists(c):
            return c
    raise RuntimeError("nvcc not found")


def _link(lib, sources, header, verbose, force):
    srcs = [os.path.join(CSRC, s) for s in sources]
    deps = srcs + [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))]
    deps.append(os.path.join(os.path.dirname(HERE), "include", header))
    if (not force and os.path.exists(lib)
            and os.path.getmtime(lib) >= max(os.path.getmtime(d) for d in deps)):
        return lib
    objdir = os.path.join(HERE, "_build")
    os.makedirs(objdir, exist_ok=True)
    objs = []
    for s in srcs:
        o = os.path.join(objdir, os.path.basename(s) + ".o")
        cmd = [nvcc()] + ARCH + FLAGS + (["-Xptxas", "-v"] if verbose else []) + ["-c", s, "-o", o]
        subprocess.run(cmd, check=True)
        objs.append(o)
    tmp = lib + ".tmp"
    subprocess.run([nvcc()] + ARCH + ["-shared", "-cudart", "static", "-o", tmp] + objs, check=True)
    os.replace(tmp, lib)
    return lib


def build(verbose=False, force=False):
    """Both libraries: the attention path (libsage_b200.so) and its
    microbenchmarks (libsage_ubench.so).  Returns the attention library."""
    _link(UBENCH_LIB, UBENCH_SOURCES, "sage_ubench.h", verbose, force)
    return _link(LIB, SOURCES, "sage.h", verbose, force)


if __name__ == "__main__":
    print(build(verbose="--verbose" in sys.argv, force=True))
