"""Compile the fp64 oracle (oracle.c) into liboracle.so beside it.

Test infrastructure: built by __graft_entry__.build() so the checker exists,
loaded only by the tests, the smoke check and the benchmark's CPU baseline."""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
LIB = os.path.join(HERE, "liboracle.so")


def build(force=False):
    srcs = [os.path.join(HERE, "oracle.c"), os.path.join(HERE, "oracle.h")]
    if not force and os.path.exists(LIB) and all(os.path.getmtime(LIB) >= os.path.getmtime(s) for s in srcs):
        return LIB
    subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fopenmp", "-shared", "-fPIC", "-Wall",
                           "-o", LIB, srcs[0], "-lm"])
    return LIB


if __name__ == "__main__":
    print(build(force=True))
