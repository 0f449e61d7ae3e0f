"""Build synth/libsynth.so, the device twin of the input generator."""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "csrc", "synth.cu")
LIB = os.path.join(HERE, "libsynth.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def build(verbose: bool = False) -> str:
    if os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    cmd = [NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-O3",
           "-std=c++17", "-Xcompiler", "-fPIC", "-shared", SRC, "-o", LIB]
    if verbose:
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    return LIB


if __name__ == "__main__":
    print(build(verbose=True))
