"""Build librra.so in-tree with nvcc for sm_100a (B200).

    python -m ragged_varlen_attention_rra_b200.build [--verbose-ptxas]

The CUDA runtime is linked statically and the driver's tensor-map encoder is fetched at run
time, so the library loads on machines without a GPU driver (it only fails once a call needs
the device).
"""
from __future__ import annotations

import argparse
import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "librra.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-O2", "-shared", "-cudart", "static",
         "--expt-relaxed-constexpr"]


# the exponential-unit microbenchmark bench.py uses for the attention kernel's exp bound
MB_SRC = os.path.join(HERE, "microbench", "ex2_rate.cu")
MB_LIB = os.path.join(HERE, "libmicrobench.so")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def headers():
    return sorted(glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) +
                  [os.path.join(HERE, "..", "include", "rra.h")])


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(f) <= t for f in sources() + headers())


def build_microbench(force: bool = False) -> str:
    if not force and os.path.exists(MB_LIB) and os.path.getmtime(MB_SRC) <= os.path.getmtime(MB_LIB):
        return MB_LIB
    tmp = MB_LIB + f".tmp{os.getpid()}"
    subprocess.run([NVCC, *ARCH_FLAGS, *FLAGS, MB_SRC, "-o", tmp], check=True)
    os.replace(tmp, MB_LIB)
    return MB_LIB


def build(force: bool = False, verbose_ptxas: bool = False, extra=()) -> str:
    build_microbench(force)
    if not force and not verbose_ptxas and up_to_date():
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [NVCC, *ARCH_FLAGS, *FLAGS, *extra]
    if verbose_ptxas:
        cmd += ["-Xptxas", "-v"]
    cmd += [*sources(), "-o", tmp]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--verbose-ptxas", action="store_true")
    ap.add_argument("--force", action="store_true")
    args = ap.parse_args(argv)
    print(build(force=args.force, verbose_ptxas=args.verbose_ptxas))


if __name__ == "__main__":
    sys.exit(main())
