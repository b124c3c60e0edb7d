"""Compile the fp64 CPU oracle (``gdn2_ref.c``) into ``liboracle_gdn2.so``.

Test infrastructure: only the tests, the smoke check and the benchmark's CPU
baseline load the result.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "gdn2_ref.c")
LIB = os.path.join(HERE, "liboracle_gdn2.so")


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    # -ffp-contract=off keeps every multiply and add separately rounded (no FMA
    # contraction), so the oracle is plain IEEE fp64 arithmetic.
    cmd = ["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-shared", "-fPIC",
           "-pthread", SRC, "-o", LIB + ".tmp", "-lm"]
    subprocess.check_call(cmd)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
