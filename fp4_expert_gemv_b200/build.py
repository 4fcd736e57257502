"""Build the CUDA libraries in-tree with nvcc for sm_100a.

  fp4_expert_gemv_b200/libfe_moe.so   the layer (C ABI of include/fe_moe.h)
  synth/libfe_synth.so                the seeded weight generator used by tests and the benchmark

Run ``python fp4_expert_gemv_b200/build.py`` (or ``__graft_entry__.build()``); the package
itself cannot be imported before the library exists.
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-shared", "--expt-relaxed-constexpr"]

LIB_MOE = os.path.join(PKG, "libfe_moe.so")
LIB_SYNTH = os.path.join(ROOT, "synth", "libfe_synth.so")


def _sources_moe():
    return ([os.path.join(CSRC, f) for f in sorted(os.listdir(CSRC)) if f.endswith((".cu", ".cpp", ".cuh"))]
            + [os.path.join(ROOT, "include", "fe_moe.h")])


def _stale(out, deps):
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    return any(os.path.getmtime(d) > t for d in deps)


def _run(cmd):
    print(" ".join(cmd), flush=True)
    subprocess.check_call(cmd)


def build(force: bool = False, verbose_ptxas: bool = False) -> None:
    extra = ["-Xptxas", "-v"] if verbose_ptxas else []
    deps = _sources_moe()
    if force or _stale(LIB_MOE, deps):
        tmp = LIB_MOE + f".{os.getpid()}.tmp"
        _run([NVCC, *ARCH, *COMMON, *extra, "-I", os.path.join(ROOT, "include"), "-o", tmp,
              os.path.join(CSRC, "fe_moe.cu"), os.path.join(CSRC, "pack_host.cpp")])
        os.replace(tmp, LIB_MOE)
    src = os.path.join(ROOT, "synth", "synth.cu")
    if force or _stale(LIB_SYNTH, [src]):
        tmp = LIB_SYNTH + f".{os.getpid()}.tmp"
        _run([NVCC, *ARCH, *COMMON, "-o", tmp, src])
        os.replace(tmp, LIB_SYNTH)


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose_ptxas="-v" in sys.argv)
