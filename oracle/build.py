"""Build the CPU oracle (test infrastructure) into oracle/libtg_oracle.so.

Plain C11, gcc -O2, no -ffast-math, no OpenMP: the oracle is single-threaded
and follows IEEE fp64 arithmetic so that its results are reproducible.
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "tg_oracle.c")
HDR = os.path.join(HERE, "tg_oracle.h")
LIB = os.path.join(HERE, "libtg_oracle.so")


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(p) > t for p in (SRC, HDR, __file__))


def build(force: bool = False) -> str:
    if force or needs_build():
        tmp = LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-std=c11", "-O2", "-fno-fast-math", "-ffp-contract=off",
               "-fPIC", "-shared", "-Wall", "-Wextra", "-o", tmp, SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True))
