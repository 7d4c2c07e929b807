"""Build libcoli.so (sm_100a) in-tree with nvcc."""
import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libcoli.so")
# the bounds-checked build: index checks record status 4 in the call's status word instead of trapping
LIB_BOUNDS = os.path.join(PKG, "libcoli_bounds.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "--expt-relaxed-constexpr",
]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h"))


def build(force=False, verbose=False, extra=(), bounds=False):
    """Build libcoli.so, or with bounds=True the bounds-checked libcoli_bounds.so."""
    out = LIB_BOUNDS if bounds else LIB
    if not force and os.path.exists(out) and os.path.getmtime(out) >= max(os.path.getmtime(p) for p in _deps()):
        return out
    nvcc = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    flags = [*NVCC_FLAGS, *extra] + (["-DCOLI_DEBUG_BOUNDS"] if bounds else [])
    cmd = [nvcc, *flags, "-I", INCLUDE, "-I", CSRC, "-shared", "-o", out + ".tmp", *sources()]
    if verbose:
        print(" ".join(cmd))
    subprocess.check_call(cmd)
    os.replace(out + ".tmp", out)
    return out


if __name__ == "__main__":
    extra = ["-Xptxas", "-v"] if "-v" in sys.argv else []
    print(build(force=True, verbose=True, extra=extra, bounds="--bounds" in sys.argv))
