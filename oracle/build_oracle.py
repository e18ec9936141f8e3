"""Compile the C++ oracle (moe_oracle_ref.cpp) into liboracle_ref.so next to it.

    python -m oracle.build_oracle

Test infrastructure: the tests, the smoke check and the benchmark's CPU legs
load it; nothing on the product path does.  Plain g++, single-threaded code,
no fast-math and no FMA contraction, so every fp32 division and fp64 sum is
the IEEE operation the source spells out.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "moe_oracle_ref.cpp")
LIB = os.path.join(HERE, "liboracle_ref.so")
CXX = os.environ.get("CXX", "g++")
FLAGS = ["-O3", "-std=c++17", "-shared", "-fPIC", "-fno-fast-math", "-ffp-contract=off"]


def build(force: bool = False) -> str:
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= os.path.getmtime(SRC)):
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    r = subprocess.run([CXX, *FLAGS, SRC, "-o", tmp], capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"g++ failed on {SRC}:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
