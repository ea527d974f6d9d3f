"""Build libattn_b200.so in-tree with nvcc for sm_100a (no JIT, no torch extension)."""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libattn_b200.so")
HEADER = os.path.join(ROOT, "include", "attn.h")


def sources():
    """Every file the library is compiled from: all of csrc/ and the public header."""
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC)
                  if f.endswith((".cu", ".cuh", ".h")))


def nvcc_cmd(out=LIB, extra=()):
    return ["nvcc", "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a",
            "-lineinfo", "-Xcompiler", "-fPIC", "-shared", *extra,
            os.path.join(CSRC, "api.cu"), "-o", out]


def up_to_date():
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    deps = sources() + [HEADER, __file__]
    return all(os.path.getmtime(d) <= t for d in deps)


def build(force=False, verbose=False):
    """Compile the library unless it is up to date.  Returns its path."""
    if not force and up_to_date():
        return LIB
    tmp = LIB + ".tmp"
    extra = ("-Xptxas", "-v") if verbose else ()
    subprocess.check_call(nvcc_cmd(tmp, extra))
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    import sys
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
