"""Build the CPU oracle shared library (plain C, gcc).

Test infrastructure: see the header of rsq_oracle.c.  No fast-math and no
floating-point contraction, so every binary32 operation in the C source is one
IEEE operation.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "rsq_oracle.c")
LIB = os.path.join(HERE, "librsq_oracle.so")


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    tmp = LIB + ".tmp.%d" % os.getpid()
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math",
           "-Wall", "-Wextra", "-Werror", SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


SAN_LIB = os.path.join(HERE, "librsq_oracle_san.so")


def build_sanitized() -> str:
    """The same library under AddressSanitizer and UndefinedBehaviorSanitizer
    (for the sanitizer test; load it with RSQ_ORACLE_LIB and libasan preloaded)."""
    if os.path.exists(SAN_LIB) and os.path.getmtime(SAN_LIB) >= os.path.getmtime(SRC):
        return SAN_LIB
    tmp = SAN_LIB + ".tmp.%d" % os.getpid()
    cmd = ["gcc", "-O1", "-g", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math",
           "-fsanitize=address,undefined,float-cast-overflow", "-fno-sanitize-recover=all", "-fno-omit-frame-pointer",
           SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, SAN_LIB)
    return SAN_LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
