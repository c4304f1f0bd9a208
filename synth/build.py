"""Compile the seeded input generator (synth.c) into libsynth.so beside it."""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
LIB = os.path.join(HERE, "libsynth.so")


def build(force=False):
    src = os.path.join(HERE, "synth.c")
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(src):
        return LIB
    subprocess.check_call(["gcc", "-O3", "-march=x86-64-v2", "-fno-math-errno", "-ffp-contract=off", "-fopenmp", "-shared", "-fPIC", "-Wall", "-o", LIB, src, "-lm"])
    return LIB


if __name__ == "__main__":
    print(build(force=True))
