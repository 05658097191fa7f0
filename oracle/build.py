"""Compile the C oracle into ``oracle/libgdn_oracle.so`` (gcc, -O2, no fast-math).

Test infrastructure only.  ``build(src=..., out=..., defines=...)`` is also used
by the planted-mistake tests to compile altered copies of the source into a
temporary directory.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "gdn_oracle.c")
LIB = os.path.join(HERE, "libgdn_oracle.so")


def build(src: str = SRC, out: str = LIB, force: bool = False) -> str:
    """Build the shared library if it is missing or older than its source."""
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(src):
        return out
    # -ffp-contract=off: keep every multiply and add as written (no FMA fusion),
    # so the oracle's rounding follows its source line by line.
    cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fPIC", "-shared", "-pthread",
           src, "-o", out, "-lm"]
    subprocess.run(cmd, check=True)
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
