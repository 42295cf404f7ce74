"""Build the CPU oracle (liboracle.so) with gcc.

Test infrastructure: the oracle is compiled with -ffp-contract=off so that the
noise specification's binary32 operations are never fused, and with OpenMP so
that token loops can spread over the host cores (results do not depend on the
thread count: every token is computed by one thread, in a fixed order).
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SOURCES = ["noise.c", "estimator.c", "head.c", "suffix.c", "attention.c"]
LIB = os.path.join(HERE, "liboracle.so")


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = SOURCES + ["oracle.h", "build.py"]
    return any(os.path.getmtime(os.path.join(HERE, s)) > t for s in deps)


def compile_sources(src_dir: str, out: str) -> str:
    """Compile the oracle's sources found in src_dir into the shared library out."""
    cmd = ["gcc", "-O2", "-std=gnu11", "-fPIC", "-shared", "-fopenmp",
           "-ffp-contract=off", "-fno-fast-math", "-Wall", "-Wextra",
           "-o", out + ".tmp"] + [os.path.join(src_dir, s) for s in SOURCES] + ["-lm"]
    subprocess.run(cmd, check=True)
    os.replace(out + ".tmp", out)
    return out


def build(force: bool = False) -> str:
    if force or _stale():
        compile_sources(HERE, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
