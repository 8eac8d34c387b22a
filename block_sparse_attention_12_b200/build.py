"""Builds libabattn.so, the self-test library libabattn_selftest.so and the
gather and MMA-rate microbenchmarks (libabattn_gatherbench.so,
libabattn_mmabench.so), in-tree with nvcc for sm_100a (B200)."""
from __future__ import annotations

import glob
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libabattn.so")
SELFTEST_SRC = os.path.join(HERE, "selftest", "wait_selftest.cu")
SELFTEST_LIB = os.path.join(HERE, "libabattn_selftest.so")
GATHERBENCH_SRC = os.path.join(HERE, "microbench", "gather_bench.cu")
GATHERBENCH_LIB = os.path.join(HERE, "libabattn_gatherbench.so")
MMABENCH_SRC = os.path.join(HERE, "microbench", "mma_bench.cu")
MMABENCH_LIB = os.path.join(HERE, "libabattn_mmabench.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "-I", os.path.join(ROOT, "include"),
]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))
                  + [os.path.join(ROOT, "include", "abattn.h")])


def selftest_sources():
    return [SELFTEST_SRC, os.path.join(CSRC, "common.cuh"), os.path.join(ROOT, "include", "abattn.h"),
            os.path.join(ROOT, "include", "abattn_selftest.h")]


def stale(lib: str = LIB, srcs=None) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(s) > t for s in (sources() if srcs is None else srcs))


def _nvcc(src: str, lib: str, verbose: bool, extra=()) -> None:
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [NVCC, *FLAGS, *extra, "-o", tmp, src]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.check_call(cmd)
    os.replace(tmp, lib)


def build_selftest(force: bool = False, verbose: bool = False) -> str:
    if force or stale(SELFTEST_LIB, selftest_sources()):
        # hidden symbols: its copy of the device error word never binds to
        # libabattn.so's, however the two libraries are loaded
        _nvcc(SELFTEST_SRC, SELFTEST_LIB, verbose, ["-Xcompiler", "-fvisibility=hidden"])
    return SELFTEST_LIB


def build_gatherbench(force: bool = False, verbose: bool = False) -> str:
    """The gather microbenchmark of the benchmark's --gather-bench mode."""
    if force or stale(GATHERBENCH_LIB, [GATHERBENCH_SRC]):
        _nvcc(GATHERBENCH_SRC, GATHERBENCH_LIB, verbose)
    return GATHERBENCH_LIB


def build_mmabench(force: bool = False, verbose: bool = False) -> str:
    """The tensor-core rate microbenchmark of the benchmark's --mma-bench mode."""
    if force or stale(MMABENCH_LIB, [MMABENCH_SRC, os.path.join(CSRC, "common.cuh")]):
        _nvcc(MMABENCH_SRC, MMABENCH_LIB, verbose)
    return MMABENCH_LIB


def build(force: bool = False, verbose: bool = False) -> str:
    """Builds the libraries (each only when stale); returns libabattn.so."""
    if force or stale():
        _nvcc(os.path.join(CSRC, "abattn.cu"), LIB, verbose)
    build_selftest(force, verbose)
    build_gatherbench(force, verbose)
    build_mmabench(force, verbose)
    return LIB


if __name__ == "__main__":
    print(build(force=True, verbose=True))
