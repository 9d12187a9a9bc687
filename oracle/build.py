"""Build liboracle.so (test infrastructure) in-tree: plain g++, -O2, no FP
contraction, no fast-math, so every fp64 sum runs in index order."""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))


def build(force: bool = False) -> str:
    src = os.path.join(HERE, "oracle_core.cpp")
    out = os.path.join(HERE, "liboracle.so")
    if not force and os.path.exists(out) and os.path.getmtime(out) >= max(os.path.getmtime(src),
                                                                          os.path.getmtime(__file__)):
        return out
    cmd = ["g++", "-std=c++17", "-O2", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math",
           "-pthread", src, "-o", out]
    print(" ".join(cmd), flush=True)
    subprocess.check_call(cmd)
    return out


if __name__ == "__main__":
    build(force="--force" in sys.argv)
