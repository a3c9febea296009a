"""Builds the CPU oracle (test infrastructure) with gcc: ``oracle/libmoe_oracle.so``.

-O1 -ffp-contract=off keeps every floating-point operation in moe_oracle.c a single IEEE
binary32/binary64 operation (no fused multiply-add, no reassociation).
"""
from __future__ import annotations

import os
import subprocess
import sys

_HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(_HERE, "moe_oracle.c")
LIB = os.path.join(_HERE, "libmoe_oracle.so")


def build(force: bool = False) -> str:
    override = os.environ.get("MOE_ORACLE_LIB")  # tests: a separately built (e.g. mutated) oracle
    if override:
        return override
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", "-std=c11", "-O1", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
           "-Wall", "-Wextra", "-o", tmp, SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


def build_from(src: str, out: str) -> str:
    """Compile another copy of the oracle source with the same flags (used by the tests that
    plant mistakes in the oracle to show that its pins catch them)."""
    subprocess.run(["gcc", "-std=c11", "-O1", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared", "-w",
                    "-o", out, src, "-lm"], check=True)
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
