"""Compile the CPU oracle (plain C) into oracle/libep_oracle.so.

TEST INFRASTRUCTURE ONLY: the oracle is what the CUDA library is checked
against.  Flags keep the arithmetic plain IEEE: no contraction of a*b+c into
fma (only the explicit fmaf calls fuse), no fast-math.  -mfma only lets the
compiler use the CPU's fused multiply-add instruction for those fmaf calls,
which is correctly rounded like the library routine it replaces.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "ep_oracle.c")
LIB = os.path.join(HERE, "libep_oracle.so")


def _cpu_has_fma() -> bool:
    try:
        with open("/proc/cpuinfo") as f:
            return " fma " in f.read()
    except OSError:
        return False


def build(force: bool = False) -> str:
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= os.path.getmtime(SRC)):
        return LIB
    flags = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
             "-fexcess-precision=standard", "-fPIC", "-shared"]
    if _cpu_has_fma():
        flags.append("-mfma")
    tmp = LIB + f".tmp{os.getpid()}"
    subprocess.run(["gcc", *flags, SRC, "-o", tmp, "-lm"], check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
