"""Build the CUDA library ``libqknr.so`` in-tree, for sm_100a only.

    python -m qk_rmsnorm_rope_norm_b200.build [--verbose]

nvcc cross-compiles without a GPU. The CUDA runtime is linked statically, so
the shared object needs only the driver (libcuda) at run time.
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libqknr.so")
SOURCES = [os.path.join(CSRC, "qknr_api.cu"), os.path.join(CSRC, "qknr_layerwise.cu")]
DEPS = SOURCES + [os.path.join(CSRC, "qknr_kernels.cuh"),
                  os.path.join(CSRC, "qknr_pipe.cuh"),
                  os.path.join(INCLUDE, "qknr.h")]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "-shared", "-cudart", "static",
]


def nvcc() -> str:
    for c in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if c and (os.path.sep not in c or os.path.exists(c)):
            return c
    return "nvcc"


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(p) > t for p in DEPS)


def build(verbose: bool = False, force: bool = False) -> str:
    """Compile every source to an object (in parallel), then link the
    shared library."""
    if not force and not needs_build():
        return LIB
    import tempfile
    flags = [f for f in NVCC_FLAGS if f != "-shared"]
    with tempfile.TemporaryDirectory() as tmp:
        objs, procs = [], []
        for src in SOURCES:
            obj = os.path.join(tmp, os.path.basename(src) + ".o")
            cmd = [nvcc(), *flags, "-I", INCLUDE, "-I", CSRC, "-c", src, "-o", obj]
            if verbose:
                cmd.insert(1, "-Xptxas=-v")
            objs.append(obj)
            procs.append((cmd, subprocess.Popen(cmd, stdout=subprocess.PIPE,
                                                stderr=subprocess.STDOUT, text=True)))
        out = []
        for cmd, p in procs:
            text, _ = p.communicate()
            out.append(text)
            if p.returncode != 0:
                raise RuntimeError("nvcc failed:\n" + " ".join(cmd) + "\n" + text)
        cmd = [nvcc(), *NVCC_FLAGS, *objs, "-o", LIB]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError("nvcc link failed:\n" + " ".join(cmd) + "\n" + r.stdout + r.stderr)
    if verbose:
        sys.stderr.write("".join(out))
    return LIB


if __name__ == "__main__":
    print(build(verbose="--verbose" in sys.argv, force=True))
