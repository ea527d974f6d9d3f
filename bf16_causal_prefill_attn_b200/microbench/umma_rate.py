"""Build (nvcc, sm_100a, in-tree) and run the tcgen05.mma issue-rate microbenchmark
(umma_rate.cu); prints its JSON lines.  Needs a B200."""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "umma_rate.cu")
EXE = os.path.join(HERE, "umma_rate")


def build():
    if not os.path.exists(EXE) or os.path.getmtime(EXE) < os.path.getmtime(SRC):
        subprocess.check_call(["nvcc", "-O3", "-std=c++17", "-gencode",
                               "arch=compute_100a,code=sm_100a", "-lineinfo", SRC, "-o", EXE])
    return EXE


if __name__ == "__main__":
    exe = build()
    if "--build-only" not in sys.argv:
        sys.exit(subprocess.call([exe]))
