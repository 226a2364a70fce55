"""Compile the C++ oracle into oracle/liboracle_kvq.so (g++, OpenMP, IEEE fp).

No fast-math and no FMA contraction: the oracle's fp32 quantizer relies on
each subtract and divide being rounded once, nearest-even.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SO = os.path.join(HERE, "liboracle_kvq.so")


def build(force: bool = False) -> str:
    src = os.path.join(HERE, "kvq_oracle.cpp")
    hdr = os.path.join(HERE, "kvq_oracle.h")
    if not force and os.path.exists(SO) and os.path.getmtime(SO) >= max(os.path.getmtime(src), os.path.getmtime(hdr)):
        return SO
    cmd = ["g++", "-std=c++17", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-fPIC", "-shared",
           "-Wall", "-o", SO, src]
    subprocess.check_call(cmd)
    return SO


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
