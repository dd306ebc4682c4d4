"""Build libfa.so in-tree with nvcc for sm_100a.

    python -m tiled_attention_18_b200.build [--force] [--verbose-ptxas]

The library holds the C ABI of include/fa.h (host code in csrc/fa_api.cpp)
and the sm_100a kernels (csrc/fa_fwd_sm100.cu forward for D = 64/128,
csrc/fa_fwd_d256_sm100.cu forward for D = 256,
csrc/fa_fwd_short_sm100.cu forward for key sets of at most 128 keys, csrc/fa_bwd_sm100.cu backward,
with the shared device helpers of csrc/sm100_helpers.cuh).  It links the CUDA runtime
statically and reaches cuTensorMapEncodeTiled through the runtime's driver
entry-point query, so it needs no libcuda at link time.
"""
from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libfa.so")
SOURCES = [os.path.join(CSRC, "fa_fwd_sm100.cu"), os.path.join(CSRC, "fa_fwd_d256_sm100.cu"),
           os.path.join(CSRC, "fa_fwd_short_sm100.cu"), os.path.join(CSRC, "fa_bwd_sm100.cu"), os.path.join(CSRC, "fa_merge_sm100.cu"),
           os.path.join(CSRC, "fa_api.cpp")]
HEADERS = [os.path.join(CSRC, "fa_internal.h"), os.path.join(CSRC, "sm100_helpers.cuh"),
           os.path.join(INCLUDE, "fa.h")]

ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(p) > t for p in SOURCES + HEADERS + [os.path.abspath(__file__)])


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    if not force and not _stale():
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [nvcc(), *ARCH_FLAGS, "-O3", "-lineinfo", "-std=c++17", "--expt-relaxed-constexpr",
           "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden", "-shared",
           "-I", INCLUDE, "-I", CSRC, "-cudart", "static", "-o", tmp, *SOURCES]
    if verbose_ptxas:
        cmd.insert(1, "-Xptxas")
        cmd.insert(2, "-v")
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


def main(argv=None) -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose-ptxas", action="store_true")
    args = ap.parse_args(argv)
    print(build(force=args.force or args.verbose_ptxas, verbose_ptxas=args.verbose_ptxas))
    return 0


if __name__ == "__main__":
    sys.exit(main())
