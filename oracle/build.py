"""Compile the plain-C oracle into ``oracle/libsbl_oracle.so`` (test infrastructure).

Flags: ``-O2 -ffp-contract=off -fno-fast-math`` so that every fp32/fp64
operation in ``sbl_oracle.c`` is a single IEEE round-to-nearest-even step.
"""
from __future__ import annotations

import os
import subprocess
import sys

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sbl_oracle.c")
_LIB = os.path.join(_HERE, "libsbl_oracle.so")

CFLAGS = ["-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared", "-Wall"]


def library_path() -> str:
    return _LIB


def build_oracle(force: bool = False) -> str:
    """Build the oracle library if it is missing or older than its source."""
    stale = (not os.path.exists(_LIB)) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC)
    if force or stale:
        tmp = _LIB + f".{os.getpid()}.tmp"
        cmd = ["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


if __name__ == "__main__":
    print(build_oracle(force="--force" in sys.argv))
