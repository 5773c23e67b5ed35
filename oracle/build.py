"""Compile the fp64 attention oracle into ``oracle/liboracle.so``.

Test infrastructure only: the oracle is a checker for the CUDA library, never part of
its path.  Built with plain ``-O2`` (no ``-march=native``) so the same shared object runs
on any x86-64 host it is copied to, and with ``-ffp-contract=off`` so no fused
multiply-add changes the rounding of the written-out definition.

``build_native()`` compiles the same source with ``-O3 -march=native`` for the host it
runs on, for timing the oracle as a CPU baseline.  It keeps ``-ffp-contract=off`` and,
like the portable build, allows no reassociation (no ``-ffast-math``), so both builds
compute bit-identical results; the object is named after the host's CPU model, since
code for one CPU may not run on another.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "attention_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")


def build(force: bool = False, verbose: bool = False) -> str:
    """Build the shared object if it is missing or older than its source; return its path."""
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= os.path.getmtime(SRC)):
        return LIB
    cmd = ["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-fPIC",
           "-shared", "-std=c11", "-Wall", "-Wextra", "-o", LIB + ".tmp", SRC, "-lm"]
    if verbose:
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


NATIVE_FLAGS = ["-O3", "-march=native", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-fPIC",
                "-shared", "-std=c11", "-Wall", "-Wextra"]


def cpu_model() -> str:
    """The host CPU's model name (from /proc/cpuinfo), or "unknown"."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def build_native(verbose: bool = False) -> str:
    """Build (once per CPU model and source version) the -O3 -march=native timing variant;
    return its path."""
    import hashlib
    with open(SRC, "rb") as f:
        tag = hashlib.sha256(f.read() + cpu_model().encode() + " ".join(NATIVE_FLAGS).encode()).hexdigest()[:16]
    out_dir = os.path.join(HERE, "_native")
    os.makedirs(out_dir, exist_ok=True)
    lib = os.path.join(out_dir, f"liboracle-{tag}.so")
    if os.path.exists(lib):
        return lib
    cmd = ["gcc", *NATIVE_FLAGS, "-o", lib + ".tmp", SRC, "-lm"]
    if verbose:
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    os.replace(lib + ".tmp", lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
