"""Build libmsk_synth.so: the seeded input generator (host C + device fills).

The host part is compiled with -ffp-contract=off so its float steps round
exactly like the device fill kernels (which use __f*_rn intrinsics).
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
LIB = os.path.join(HERE, "libmsk_synth.so")
SOURCES = ["msk_synth.h", "msk_source.h", "synth_host.c", "synth_dev.cu"]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = "-gencode=arch=compute_100a,code=sm_100a"


def _stale(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(os.path.join(HERE, d)) > t for d in deps)


def build(force: bool = False) -> str:
    if not force and not _stale(LIB, SOURCES + ["build.py"]):
        return LIB
    bdir = os.path.join(HERE, "_build")
    os.makedirs(bdir, exist_ok=True)
    ho = os.path.join(bdir, "synth_host.o")
    do = os.path.join(bdir, "synth_dev.o")
    subprocess.check_call(["gcc", "-O2", "-fPIC", "-ffp-contract=off", "-msse2", "-std=c11",
                           "-Wall", "-c", os.path.join(HERE, "synth_host.c"), "-o", ho])
    subprocess.check_call([NVCC, ARCH, "-O2", "-std=c++17", "-Xcompiler", "-fPIC,-ffp-contract=off",
                           "-c", os.path.join(HERE, "synth_dev.cu"), "-o", do])
    tmp = LIB + ".tmp"
    subprocess.check_call([NVCC, ARCH, "-shared", "--cudart", "shared", "-o", tmp, ho, do,
                           "-lpthread", "-lm"])
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True))
