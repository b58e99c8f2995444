"""Compile the CPU oracle into ``oracle/liblpar_oracle.so`` (test infrastructure).

Plain gcc, no contraction of a*b+c into fused multiply-adds and no fast-math,
so every binary32 operation in the oracle rounds once, to nearest even.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "lpar_oracle.c")
LIB = os.path.join(HERE, "liblpar_oracle.so")

CFLAGS = ["-std=c11", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
          "-Wall", "-Wextra", "-Werror"]


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    lib_mtime = os.path.getmtime(LIB)
    return any(os.path.getmtime(os.path.join(HERE, f)) > lib_mtime
               for f in ("lpar_oracle.c", "lpar_oracle.h"))


def build(force: bool = False) -> str:
    if force or needs_build():
        tmp = LIB + ".tmp.%d" % os.getpid()
        subprocess.run(["gcc", *CFLAGS, SRC, "-o", tmp, "-lm"], check=True)
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
