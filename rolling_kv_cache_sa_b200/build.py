"""Builds rolling_kv_cache_sa_b200/libsa.so (sm_100a) from csrc/*.cu with nvcc."""
import glob
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libsa.so")
# the debug build: every computed buffer index is range-checked in the kernels
DEBUG_LIB = os.path.join(HERE, "libsa_debug.so")

NVCC_FLAGS = ["-O3", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
              "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
              "-Xptxas", "-v", "--expt-relaxed-constexpr"]


def sources():
    return sorted(glob.glob(os.path.join(HERE, "csrc", "*.cu")))


def deps():
    return sources() + sorted(glob.glob(os.path.join(HERE, "csrc", "*.h"))) + \
        sorted(glob.glob(os.path.join(HERE, "csrc", "*.cuh"))) + \
        [os.path.join(ROOT, "include", "sa.h")]


def is_stale() -> bool:
    for lib in (LIB, DEBUG_LIB):
        if not os.path.exists(lib):
            return True
        t = os.path.getmtime(lib)
        if any(os.path.getmtime(s) > t for s in deps()):
            return True
    return False


def build(verbose: bool = False) -> str:
    """Builds libsa.so and the debug build libsa_debug.so (-DSA_DEBUG_BOUNDS)
    side by side; returns the path of libsa.so."""
    cmds = [["nvcc", *NVCC_FLAGS, *sources(), "-o", LIB, "-lcuda", "-ldl"],
            ["nvcc", *NVCC_FLAGS, "-DSA_DEBUG_BOUNDS", *sources(), "-o", DEBUG_LIB, "-lcuda",
             "-ldl"]]
    if verbose:
        for c in cmds:
            print(" ".join(c))
    procs = [subprocess.Popen(c, stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True)
             for c in cmds]
    outs = [pr.communicate() for pr in procs]
    log = os.path.join(HERE, "build.log")
    with open(log, "w") as f:
        for (o, e) in outs:
            f.write(o + e)
    for pr, (o, e) in zip(procs, outs):
        if pr.returncode != 0:
            raise RuntimeError("nvcc failed:\n" + e[-6000:])
    return LIB


if __name__ == "__main__":
    print(build(verbose=True))
