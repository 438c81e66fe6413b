"""Compile the fp64 CPU oracle (pkv_oracle.c) into oracle/_build/libpkv_oracle.so.

Test infrastructure: the oracle is what the CUDA library is checked against.
Plain -O2 with IEEE semantics (no -ffast-math), so that gcc does not
re-associate the oracle's sums.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "pkv_oracle.c")
OUT_DIR = os.path.join(HERE, "_build")
LIB = os.path.join(OUT_DIR, "libpkv_oracle.so")


def compile_source(src: str, lib: str) -> str:
    """Compile one oracle source file into a shared library at ``lib``."""
    os.makedirs(os.path.dirname(lib), exist_ok=True)
    tmp = lib + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-D_GNU_SOURCE", "-fPIC", "-shared",
           "-fno-fast-math", "-ffp-contract=off", "-Wall", "-Wextra",
           "-o", tmp, src, "-lm", "-lpthread"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


def build(force: bool = False) -> str:
    """Build the oracle library if it is missing or older than its source."""
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= os.path.getmtime(SRC)):
        return LIB
    return compile_source(SRC, LIB)


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
