"""Compile the CPU oracle (test infrastructure) into ``oracle/liboracle.so``.

Plain gcc, fp64, no fast-math and no FMA contraction, so each operation in
the C source is one correctly rounded IEEE operation.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "qknr_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")

CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
          "-fno-fast-math", "-Wall", "-Wextra"]


def build(src: str = SRC, out: str = LIB, quiet: bool = True) -> str:
    """Compile ``src`` to the shared object ``out``; returns ``out``."""
    cmd = ["gcc", *CFLAGS, src, "-o", out, "-lm"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"oracle build failed:\n{' '.join(cmd)}\n{r.stderr}")
    if not quiet and r.stderr:
        sys.stderr.write(r.stderr)
    return out


def needs_build(src: str = SRC, out: str = LIB) -> bool:
    return (not os.path.exists(out)) or os.path.getmtime(out) < os.path.getmtime(src)


if __name__ == "__main__":
    print(build(quiet=False))
