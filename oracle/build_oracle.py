"""Compile the fp64 CPU oracle (``ssm_oracle.c``) into a shared library.

Test infrastructure: the oracle is never linked into the product library.
Plain ``gcc -O2`` without fast-math, so every operation is IEEE double in
source order.  ``mutant`` builds a copy with one deliberate mistake planted
(see ``SSM_ORACLE_MUTANT`` in the C source) for the tests that show the pins
catch such mistakes.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "ssm_oracle.c")


def lib_path(mutant: int = 0) -> str:
    if mutant == 0:
        return os.path.join(HERE, "libssm_oracle.so")
    return os.path.join(HERE, "_mutants", f"libssm_oracle_m{mutant}.so")


def build(mutant: int = 0, force: bool = False) -> str:
    out = lib_path(mutant)
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(SRC):
        return out
    os.makedirs(os.path.dirname(out), exist_ok=True)
    tmp = out + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fno-fast-math", "-ffp-contract=off", "-fopenmp",
           "-fPIC", "-shared", f"-DSSM_ORACLE_MUTANT={mutant}", SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    print(build(int(sys.argv[1]) if len(sys.argv) > 1 else 0, force=True))
