"""Build step of the CUDA library: nvcc for sm_100a into ``libsharq.so``.

Run ``python -m sparse_activation_quantization_b200.build`` (or call
``build()``).  The shared library is written next to this file (in-tree), so
it travels with the source tree.  No fast-math flags: the quantizer's float32
steps must round exactly as IEEE single precision.
"""
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libsharq.so")
SOURCES = ["api.cu", "prep.cu", "pack_weight.cu", "gemm.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC"]


def nvcc():
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _stale(objs):
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in os.listdir(CSRC)]
    deps.append(os.path.join(HERE, "peak", "fp4_peak.cu"))
    deps.append(os.path.join(HERE, "..", "include", "sharq.h"))
    deps.append(os.path.abspath(__file__))
    return any(os.path.getmtime(d) > t for d in deps if os.path.exists(d))


def build(force=False, verbose=False, extra=()):
    """Compile every source for sm_100a and link libsharq.so; returns its path."""
    if not force and not _stale(None):
        return LIB
    out_dir = os.path.join(HERE, "_build")
    os.makedirs(out_dir, exist_ok=True)
    objs = []
    for src in SOURCES:
        obj = os.path.join(out_dir, src.replace(".cu", ".o"))
        cmd = [nvcc(), *ARCH, *FLAGS, *extra, "-c", os.path.join(CSRC, src), "-o", obj]
        if verbose:
            print(" ".join(cmd), file=sys.stderr)
        subprocess.run(cmd, check=True)
        objs.append(obj)
    tmp = LIB + ".tmp"
    cmd = [nvcc(), *ARCH, "-shared", "-cudart", "static", "-o", tmp, *objs]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    # the FP4 peak microbenchmark (roofline denominators), a separate library
    peak_src = os.path.join(HERE, "peak", "fp4_peak.cu")
    peak_lib = os.path.join(HERE, "peak", "libsharq_peak.so")
    subprocess.run([nvcc(), *ARCH, *FLAGS, "-shared", "-cudart", "static", peak_src, "-o", peak_lib + ".tmp"],
                   check=True)
    os.replace(peak_lib + ".tmp", peak_lib)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True,
                extra=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else ()))
