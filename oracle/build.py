"""Builds the C++ oracle (liboracle.so) in-tree -- TEST INFRASTRUCTURE ONLY.

    python oracle/build.py            # incremental
    python oracle/build.py --force    # rebuild

Flags: -O2 -ffp-contract=off -fno-fast-math, so every binary32 / binary64
operation of the oracle rounds once as IEEE 754 states it (no fused
multiply-add, no reassociation).
"""

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
LIB = os.path.join(HERE, "liboracle.so")
SOURCES = ["blocks.cc", "turbo.cc", "attention.cc"]
HEADERS = ["oracle.h", "oracle_internal.h"]
FLAGS = ["-O2", "-std=c++17", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared", "-pthread",
         "-Wall", "-Wextra"]


def _stale():
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = SOURCES + HEADERS + [os.path.basename(__file__)]
    return any(os.path.getmtime(os.path.join(HERE, f)) > t for f in deps)


def build(force=False):
    """Compile the oracle's sources into oracle/liboracle.so; returns its path."""
    if force or _stale():
        tmp = LIB + f".tmp{os.getpid()}"
        cmd = ["g++", *FLAGS, "-o", tmp, *[os.path.join(HERE, f) for f in SOURCES]]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"oracle build failed:\n{r.stdout}\n{r.stderr}")
        os.replace(tmp, LIB)   # atomic: a concurrent loader never sees a partial file
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
