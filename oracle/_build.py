"""Compile the C oracle into oracle/libkvq_oracle.so (test infrastructure),
and the all-core baseline build into oracle/libkvq_oracle_omp.so (the same
kvq_oracle.c plus baseline_omp.c, with OpenMP; used only by the benchmark's
CPU-baseline leg)."""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "kvq_oracle.c")
OMP_SRC = os.path.join(HERE, "baseline_omp.c")
LIB = os.path.join(HERE, "libkvq_oracle.so")
OMP_LIB = os.path.join(HERE, "libkvq_oracle_omp.so")
FLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math"]


def _fresh(lib, srcs):
    return os.path.exists(lib) and all(os.path.getmtime(lib) >= os.path.getmtime(s)
                                       for s in srcs)


def _compile(lib, srcs, extra):
    tmp = lib + ".tmp.%d" % os.getpid()
    subprocess.run(["gcc", *FLAGS, *extra, "-o", tmp, *srcs, "-lm"], check=True)
    os.replace(tmp, lib)


def build(force: bool = False) -> str:
    if force or not _fresh(LIB, [SRC]):
        _compile(LIB, [SRC], [])
    return LIB


def build_omp(force: bool = False) -> str:
    srcs = [SRC, OMP_SRC]
    if force or not _fresh(OMP_LIB, srcs):
        _compile(OMP_LIB, srcs, ["-fopenmp"])
    return OMP_LIB


if __name__ == "__main__":
    print(build(force=True))
    print(build_omp(force=True))
