"""Compile the CPU oracle (test infrastructure) into oracle/libhhr_oracle.so."""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "hhr_oracle.cpp")
LIB = os.path.join(HERE, "libhhr_oracle.so")

# Plain optimisation only: no -ffast-math, no -ffp-contract=fast, so every sum
# keeps the order written in the source and products are rounded separately.
CXXFLAGS = ["-O2", "-std=c++17", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math"]


def up_to_date() -> bool:
    return os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC)


def build(force: bool = False) -> str:
    if force or not up_to_date():
        cmd = [os.environ.get("CXX", "g++"), *CXXFLAGS, SRC, "-o", LIB + ".tmp"]
        subprocess.run(cmd, check=True)
        os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
