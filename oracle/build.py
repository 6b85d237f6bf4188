"""Compile the fp64 CPU oracle (oracle.c) into oracle/liboracle.so.

Test infrastructure: the oracle is loaded only by tests/, the package's
smoke() check and bench.py's CPU-baseline / reference leg.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SO = os.path.join(HERE, "liboracle.so")


def build(force: bool = False) -> str:
    src = os.path.join(HERE, "oracle.c")
    hdr = os.path.join(HERE, "oracle.h")
    if (not force and os.path.exists(SO)
            and os.path.getmtime(SO) >= max(os.path.getmtime(src), os.path.getmtime(hdr))):
        return SO
    tmp = SO + ".tmp%d" % os.getpid()
    # IEEE semantics: no -ffast-math, no FMA contraction (plain C evaluation order).
    cmd = ["gcc", "-std=c99", "-O2", "-ffp-contract=off", "-fPIC", "-shared",
           "-Wall", "-o", tmp, src, "-lm", "-lpthread"]
    subprocess.check_call(cmd)
    os.replace(tmp, SO)
    return SO


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
