"""Build the CPU oracle (``oracle.c``) into ``liboracle.so`` next to it.

Test infrastructure only: the oracle checks the CUDA library; nothing on the
product path loads it.
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "oracle.c")
LIB = os.path.join(HERE, "liboracle.so")
# the same source with its output-row loops split over threads (OpenMP); used
# only for the multi-threaded CPU baseline
LIB_THREADS = os.path.join(HERE, "liboracle_omp.so")


def build(force: bool = False, threads: bool = False) -> str:
    """Compile the oracle with gcc (plain C11, -O2, no fast-math) if stale;
    threads=True builds the OpenMP variant."""
    lib = LIB_THREADS if threads else LIB
    stale = (not os.path.exists(lib)) or os.path.getmtime(lib) < os.path.getmtime(SRC)
    if force or stale:
        tmp = lib + ".tmp.%d" % os.getpid()
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
               "-ffp-contract=off"] + (["-fopenmp"] if threads else []) + ["-o", tmp, SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force=True))
    print(build(force=True, threads=True))
