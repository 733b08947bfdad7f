"""Build step of the CUDA library: nvcc for sm_100a into ``libsharq.so``.

Run ``python -m sparse_activation_quantization_b200.build`` (or call
``build()``).  The shared library is written next to this file (in-tree), so
it travels with the source tree.  No fast-math flags: the quantizer's float32
steps must round exactly as IEEE single precision.
"""
import hashlib
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


STAMP = LIB + ".sha256"
PEAK_SRC = os.path.join(HERE, "peak", "fp4_peak.cu")
PEAK_LIB = os.path.join(HERE, "peak", "libsharq_peak.so")


def source_hash(extra=()):
    """sha256 over every input of the build: the CUDA sources and headers,
    the public header, the peak microbenchmark, this file and the compiler
    flags.  A library whose recorded hash differs is rebuilt, whatever the
    files' times say (a prebuilt library copied in beside newer sources is
    never reused)."""
    h = hashlib.sha256()
    deps = sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cu", ".cuh", ".h")))
    deps += [PEAK_SRC, os.path.join(HERE, "..", "include", "sharq.h"), os.path.abspath(__file__)]
    for d in deps:
        h.update(os.path.basename(d).encode())
        with open(d, "rb") as f:
            h.update(f.read())
    h.update(" ".join([*ARCH, *FLAGS, *extra]).encode())
    return h.hexdigest()


def _stale(digest):
    if not (os.path.exists(LIB) and os.path.exists(PEAK_LIB) and os.path.exists(STAMP)):
        return True
    with open(STAMP) as f:
        return f.read().strip() != digest


def build(force=False, verbose=False, extra=()):
    """Compile every source for sm_100a and link libsharq.so; returns its path.
    Skipped when the library was built from exactly these sources and flags."""
    digest = source_hash(extra)
    if not force and not _stale(digest):
        return LIB
    out_dir = os.path.join(HERE, "_build")
    os.makedirs(out_dir, exist_ok=True)
    objs, procs = [], []
    for src in SOURCES:  # the translation units compile side by side
        obj = os.path.join(out_dir, src.replace(".cu", ".o"))
        cmd = [nvcc(), *ARCH, *FLAGS, *extra, "-c", os.path.join(CSRC, src), "-o", obj]
        if verbose:
            print(" ".join(cmd), file=sys.stderr)
        procs.append((cmd, subprocess.Popen(cmd)))
        objs.append(obj)
    failed = [cmd for cmd, p in procs if p.wait() != 0]
    if failed:
        raise subprocess.CalledProcessError(1, failed[0])
    tmp = LIB + ".tmp"
    cmd = [nvcc(), *ARCH, "-shared", "-cudart", "static", "-o", tmp, *objs]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    # the FP4 peak microbenchmark (roofline denominators), a separate library
    subprocess.run([nvcc(), *ARCH, *FLAGS, "-shared", "-cudart", "static", PEAK_SRC, "-o", PEAK_LIB + ".tmp"],
                   check=True)
    os.replace(PEAK_LIB + ".tmp", PEAK_LIB)
    with open(STAMP + ".tmp", "w") as f:
        f.write(digest + "\n")
    os.replace(STAMP + ".tmp", STAMP)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True,
                extra=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else ()))
