"""Compile the CPU oracle (plain C) into ``oracle/_build/liboracle.so``.

Test infrastructure: the oracle is built here so that the test suite, the smoke
check and the benchmark's CPU-baseline leg can load it with ctypes.
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "bitnet_oracle.c")
HDR = os.path.join(HERE, "bitnet_oracle.h")
OUT_DIR = os.path.join(HERE, "_build")
LIB = os.path.join(OUT_DIR, "liboracle.so")

# -ffp-contract=off: no multiply may be fused into an add (the quantiser's
# x*inv is one rounded fp32 product); -fno-fast-math keeps IEEE semantics.
CFLAGS = ["-std=c11", "-O2", "-Wall", "-Wextra", "-ffp-contract=off",
          "-fno-fast-math", "-fno-tree-vectorize", "-shared", "-fPIC"]


def build(force: bool = False) -> str:
    os.makedirs(OUT_DIR, exist_ok=True)
    stale = force or not os.path.exists(LIB) or any(
        os.path.getmtime(p) > os.path.getmtime(LIB) for p in (SRC, HDR, __file__))
    if stale:
        tmp = LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, SRC, "-lm"])
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True))
