"""Compile the CPU oracle (plain C, gcc) into oracle/liboracle.so.

Test infrastructure: building the checker is not using it. Run as
``python oracle/build.py`` or through ``__graft_entry__.build()``.
"""

from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "skiparse_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")


def build(force: bool = False, verbose: bool = False, mutant: int = 0) -> str:
    """The oracle library; with mutant = k > 0, a copy with planted mistake k (see the
    mutation hooks at the top of skiparse_oracle.c), for the oracle's own tests only."""
    lib = LIB if mutant == 0 else os.path.join(HERE, f"liboracle_mutant{mutant}.so")
    deps = [SRC, os.path.join(HERE, "skiparse_oracle.h")]
    if not force and os.path.exists(lib):
        if os.path.getmtime(lib) >= max(os.path.getmtime(p) for p in deps):
            return lib
    tmp = lib + f".tmp{os.getpid()}"
    cmd = ["gcc", "-std=c11", "-O2", "-fPIC", "-shared", "-Wall", "-Wextra",
           "-fno-fast-math", "-ffp-contract=off", f"-DORACLE_MUTANT={mutant}", SRC, "-o", tmp,
           "-lm", "-lpthread"]
    if verbose:
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
