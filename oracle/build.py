"""Compile the C oracle with gcc.

TEST INFRASTRUCTURE ONLY: the oracle checks the CUDA library; the library never
uses it.  ``build()`` writes ``oracle/libpa_oracle.so``; ``build_mutant(n, dir)``
writes a copy with planted mistake ``n`` for the tests that check the pins catch it.
"""
from __future__ import annotations

import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(HERE, "pa_oracle.c")
LIBRARY = os.path.join(HERE, "libpa_oracle.so")


def _compile(out: str, defines: tuple[str, ...] = ()) -> str:
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread", "-Wall", "-Wextra",
           *[f"-D{d}" for d in defines], "-o", out, SOURCE, "-lm"]
    subprocess.run(cmd, check=True)
    return out


def build(force: bool = False) -> str:
    """Build the default (unmutated) oracle library in-tree and return its path."""
    if force or not os.path.exists(LIBRARY) or os.path.getmtime(LIBRARY) < os.path.getmtime(SOURCE):
        tmp = LIBRARY + f".tmp{os.getpid()}"
        _compile(tmp)
        os.replace(tmp, LIBRARY)
    return LIBRARY


def build_mutant(mutant: int, out_dir: str) -> str:
    """Build the oracle with planted mistake ``mutant`` into ``out_dir``."""
    return _compile(os.path.join(out_dir, f"libpa_oracle_m{mutant}.so"), (f"PA_ORACLE_MUTANT={mutant}",))


if __name__ == "__main__":
    print(build(force=True))
