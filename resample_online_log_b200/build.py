"""Builds libsmcsd.so (the C-ABI library) in-tree with nvcc for sm_100a."""

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SOURCES = ["abi.cu", "smc.cu", "verify.cu", "resample.cu", "pagetable.cu", "topk.cu",
           "bandit.cu", "ngram.cu", "draft.cu"]
LIB = os.path.join(HERE, "libsmcsd.so")
TESTING_LIB = os.path.join(HERE, "libsmcsd_testing.so")
FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
         "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden"]


def build(verbose=False, jobs=None):
    inc = os.path.join(ROOT, "include")
    csrc = os.path.join(HERE, "csrc")
    objdir = os.path.join(HERE, "_build")
    os.makedirs(objdir, exist_ok=True)
    procs = []
    objs = []
    for src in SOURCES:
        obj = os.path.join(objdir, src.replace(".cu", ".o"))
        objs.append(obj)
        cmd = ["nvcc", *FLAGS, "-I", inc, "-c", os.path.join(csrc, src), "-o", obj]
        if verbose:
            print(" ".join(cmd))
        procs.append(subprocess.Popen(cmd))
    for p in procs:
        if p.wait() != 0:
            raise RuntimeError("nvcc failed")
    # Static CUDA runtime with its symbols kept local: the library carries its own
    # runtime and never binds to another copy already loaded in the process.
    cmd = ["nvcc", "-shared", "-gencode", "arch=compute_100a,code=sm_100a", "--cudart", "static",
           "-Xlinker", "--exclude-libs,ALL", "-o", LIB, *objs]
    if verbose:
        print(" ".join(cmd))
    subprocess.check_call(cmd)
    # Test-only library: the device generator on chosen counters (tests pin it).
    tobj = os.path.join(objdir, "testing.o")
    subprocess.check_call(["nvcc", *FLAGS, "-I", inc, "-c", os.path.join(csrc, "testing.cu"),
                           "-o", tobj])
    subprocess.check_call(["nvcc", "-shared", "-gencode", "arch=compute_100a,code=sm_100a",
                           "--cudart", "static", "-Xlinker", "--exclude-libs,ALL", "-o",
                           TESTING_LIB, tobj])
    return LIB


if __name__ == "__main__":
    print(build(verbose="-v" in sys.argv))
