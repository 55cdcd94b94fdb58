"""Compiles inputgen.cu into inputgen/libsa_inputgen.so (host + sm_100a device fill)."""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))


def build(verbose: bool = False) -> str:
    out = os.path.join(HERE, "libsa_inputgen.so")
    src = os.path.join(HERE, "inputgen.cu")
    cmd = ["nvcc", "-O3", "-std=c++17", "-shared", "-Xcompiler", "-fPIC,-fopenmp",
           "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-fmad=false",
           src, "-o", out, "-lgomp"]
    if verbose:
        print(" ".join(cmd))
    subprocess.check_call(cmd)
    return out


if __name__ == "__main__":
    print(build(verbose=True))
