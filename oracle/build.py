"""Build liboracle.so (TEST INFRASTRUCTURE: the fp64 CPU reference).

Only tests, the smoke check and the benchmark's CPU-baseline leg load it.
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
LIB = os.path.join(HERE, "libmsk_oracle.so")
SOURCES = ["msk_oracle.c", "msk_oracle.h", "../synth/msk_source.h"]


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB):
        t = os.path.getmtime(LIB)
        if all(os.path.getmtime(os.path.join(HERE, s)) <= t for s in SOURCES + ["build.py"]):
            return LIB
    tmp = LIB + ".tmp"
    subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-std=c11", "-Wall",
                           os.path.join(HERE, "msk_oracle.c"), "-o", tmp, "-lm", "-lpthread"])
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True))
