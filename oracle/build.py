"""Build the fp64 attention oracle (``oracle.c``) into ``liboracle.so``.

Test infrastructure only.  Plain C, ``-O2`` without ``-ffast-math`` (so the
compiler keeps IEEE double semantics and the written summation order),
OpenMP across independent rows.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "oracle.c")
LIB = os.path.join(HERE, "liboracle.so")


def compile_oracle(src: str = SRC, out: str = LIB, extra_flags: list[str] | None = None) -> str:
    """Compile ``src`` into the shared library ``out`` and return its path."""
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-Wall", "-Wextra",
           "-fno-fast-math", src, "-o", out, "-lm"]
    if extra_flags:
        cmd[1:1] = list(extra_flags)
    subprocess.run(cmd, check=True)
    return out


def ensure_built() -> str:
    """Build ``liboracle.so`` if it is missing or older than its source."""
    if not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        compile_oracle()
    return LIB


if __name__ == "__main__":
    print(compile_oracle())
    sys.exit(0)
