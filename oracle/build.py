"""Build the CPU oracle (liboracle.so) with g++.

TEST INFRASTRUCTURE ONLY: the oracle is loaded by the test suite, the smoke
check and the benchmark's CPU-baseline leg, never by the CUDA library.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SOURCES = ["philox.cpp", "topk_softmax.cpp", "pair_select.cpp", "verify_greedy.cpp",
           "verify_sample.cpp", "verify_sample_trunc.cpp", "dynconv2.cpp"]
HEADERS = ["oracle.h", "oracle_util.h"]
LIB = os.path.join(HERE, "liboracle.so")


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(os.path.join(HERE, f)) > t for f in SOURCES + HEADERS)


def build(force: bool = False) -> str:
    if force or needs_build():
        tmp = LIB + ".tmp.%d" % os.getpid()
        cmd = ["g++", "-std=c++17", "-O2", "-fPIC", "-shared", "-fno-fast-math",
               "-ffp-contract=off", "-Wall", "-Wextra", "-o", tmp] + \
              [os.path.join(HERE, f) for f in SOURCES]
        subprocess.run(cmd, check=True)
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
