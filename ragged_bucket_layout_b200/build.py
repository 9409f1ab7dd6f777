"""Build libdbuf.so in-tree with nvcc for sm_100a (no GPU needed to build)."""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libdbuf.so")
SOURCES = [os.path.join(CSRC, f) for f in ("dbuf.cu", "rowwise.cu", "muon.cu", "planner.cpp")]
HEADERS = [os.path.join(CSRC, f) for f in sorted(os.listdir(CSRC)) if f.endswith((".h", ".cuh"))] + [
    os.path.join(ROOT, "include", "dbuf.h")]

NVCC_FLAGS = [
    "-O3", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo",
    # IEEE division and square root, no contraction of a*b+c into one FMA:
    # the step's arithmetic is rounded operation by operation.
    "-prec-div=true", "-prec-sqrt=true", "-fmad=false",
    "-I", os.path.join(ROOT, "include"), "-I", CSRC,
]


def nvcc():
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def stale():
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(f) > t for f in SOURCES + HEADERS)


def build(force=False, verbose=False):
    """Compile csrc/*.cu|cpp into ragged_bucket_layout_b200/libdbuf.so."""
    if not force and not stale():
        return LIB
    cmd = [nvcc(), *NVCC_FLAGS, *(["-Xptxas", "-v"] if verbose else []), "-o", LIB, *SOURCES, "-lcudart", "-lcublas"]
    subprocess.check_call(cmd)
    return LIB


if __name__ == "__main__":
    build(force=True, verbose="-v" in sys.argv)
    print(LIB)
