"""Build the CPU oracle (plain C) into ``oracle/liboracle.so``.

Test infrastructure only: the product library never links or loads it.
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "gq_oracle.c")
HDR = os.path.join(HERE, "gq_oracle.h")
LIB = os.path.join(HERE, "liboracle.so")

# -ffp-contract=off: no fused multiply-add, every binary32/binary64 operation rounds on its own.
CFLAGS = ["-O2", "-std=gnu11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared", "-Wall", "-Wno-maybe-uninitialized"]


def build(force: bool = False) -> str:
    """Compile the oracle if the shared object is missing or older than its sources."""
    stale = force or not os.path.exists(LIB) or any(
        os.path.getmtime(p) > os.path.getmtime(LIB) for p in (SRC, HDR))
    if stale:
        tmp = LIB + ".tmp"
        subprocess.run(["gcc", *CFLAGS, "-o", tmp, SRC, "-lm"], check=True)
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True))
