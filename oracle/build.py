"""Build the CPU oracle (test infrastructure) into oracle/liboracle.so.

Flags keep float arithmetic IEEE-754: -ffp-contract=off (no fused
multiply-add), no -ffast-math, SSE arithmetic (the x86-64 default).
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "fp8blk_oracle.cpp")
OUT = os.path.join(HERE, "liboracle.so")


def build(force: bool = False) -> str:
    if not force and os.path.exists(OUT) and os.path.getmtime(OUT) >= os.path.getmtime(SRC):
        return OUT
    cxx = os.environ.get("CXX", "g++")
    tmp = OUT + f".tmp{os.getpid()}"
    cmd = [cxx, "-O2", "-std=c++17", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
           "-pthread", SRC, "-o", tmp]
    subprocess.run(cmd, check=True)
    os.replace(tmp, OUT)
    return OUT


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
