"""Builds the CPU oracle (test infrastructure) into oracle/liboracle.so.

Plain g++, IEEE arithmetic only: -ffp-contract=off so no multiply-add is fused,
and no -ffast-math.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "kvq_oracle.cpp")
LIB = os.path.join(HERE, "liboracle.so")


def compile_to(src: str, lib: str) -> str:
    """Compiles the oracle's C++ source `src` (this directory's, or a test's
    copy of it) into the shared library `lib`; returns `lib`."""
    cmd = ["g++", "-O2", "-std=c++17", "-ffp-contract=off", "-fno-fast-math", "-Wall",
           "-shared", "-fPIC", "-pthread", src, "-o", lib + ".tmp"]
    subprocess.check_call(cmd)
    os.replace(lib + ".tmp", lib)
    return lib


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    return compile_to(SRC, LIB)


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
