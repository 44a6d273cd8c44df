"""Builds libeffort.so in-tree with nvcc for sm_100a (B200).

Run as ``python -m dynamic_approximate_gemv_b200.build``; ``__graft_entry__``
calls :func:`build`.  Device code is compiled without fast-math and with
denormals kept, so the selection products round exactly as the C ABI states.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libeffort.so")
LIB_DEBUG = os.path.join(HERE, "libeffort_debug.so")
SOURCES = ["api.cu", "prep.cu", "effort.cu", "dense.cu", "noalloc.cu"]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-shared", "-Xcompiler", "-fPIC", "-Xcompiler", "-ffp-contract=off",
    "-ftz=false", "-prec-div=true", "-prec-sqrt=true",
    "-Xptxas", "-v",
]


def needs_build():
    if not (os.path.exists(LIB) and os.path.exists(LIB_DEBUG)):
        return True
    t = min(os.path.getmtime(LIB), os.path.getmtime(LIB_DEBUG))
    deps = [os.path.join(CSRC, f) for f in os.listdir(CSRC)] + [
        os.path.join(HERE, "..", "include", "effort.h"), __file__]
    return any(os.path.getmtime(p) > t for p in deps if os.path.exists(p))


def _compile(out, extra):
    cmd = [NVCC] + FLAGS + extra + ["-I" + os.path.join(HERE, "..", "include"), "-o", out + ".tmp"] + [
        os.path.join(CSRC, s) for s in SOURCES]
    res = subprocess.run(cmd, capture_output=True, text=True)
    log = res.stdout + res.stderr
    with open(os.path.join(HERE, "build.log"), "a") as f:
        f.write(" ".join(cmd) + "\n" + log)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + log[-8000:])
    os.replace(out + ".tmp", out)
    return log


def build(force=False, verbose=False):
    """Compile the CUDA sources into libeffort.so (release) and
    libeffort_debug.so (-DEFFORT_DEBUG: kernels bounds-check the indices they
    take from data and report violations through the status word) next to
    this file."""
    if not force and not needs_build():
        return LIB
    with open(os.path.join(HERE, "build.log"), "w"):
        pass
    log = _compile(LIB, [])
    log += _compile(LIB_DEBUG, ["-DEFFORT_DEBUG"])
    if verbose:
        print(log)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True)
