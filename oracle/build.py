"""Build the CPU oracle library (test infrastructure) with plain g++.

The flags keep every fp32 operation a single IEEE-754 round-to-nearest-even operation:
no fused multiply-add contraction and no fast-math.  Run ``python oracle/build.py``.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "nvfp4kv_oracle.cpp")
LIB = os.path.join(HERE, "liboracle_nvfp4kv.so")


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/liboracle_nvfp4kv.so`` (skipped when up to date)."""
    deps = [SRC, os.path.join(HERE, "nvfp4kv_oracle.h")]
    if not force and os.path.exists(LIB) and all(
            os.path.getmtime(LIB) >= os.path.getmtime(p) for p in deps):
        return LIB
    cmd = ["g++", "-std=c++17", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC",
           "-shared", "-Wall", "-Wextra", "-o", LIB, SRC]
    subprocess.run(cmd, check=True)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
