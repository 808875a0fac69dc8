"""Builds the CUDA library libimq.so in-tree for sm_100a (B200).

    python -m bit_integer_gemm_b200.build [--force] [--verbose] [--debug]

Every translation unit is compiled with nvcc for ``sm_100a`` only (tcgen05 / TMA code does not exist
on other architectures) and linked with the static CUDA runtime, so the library depends on nothing but
the driver.  --debug builds libimq_debug.so with IMQ_DEBUG defined: every plan is followed by a kernel
that checks each index the unpack and GEMM kernels read against the plan's sizes (IMQ_ERR_BOUNDS in the
status word on a violation); the binding loads it when IMQ_LIB=debug is set in the environment.
"""
from __future__ import annotations

import argparse
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libimq.so")
LIB_DEBUG = os.path.join(PKG, "libimq_debug.so")
SOURCES = ["api.cu", "rtn.cu", "plan.cu", "unpack.cu", "gemm.cu"]
HEADERS = ["common.cuh", "internal.h"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
         "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def _stale(target: str, deps) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    bdir = os.path.join(BUILD, "debug") if debug else BUILD
    lib = LIB_DEBUG if debug else LIB
    os.makedirs(bdir, exist_ok=True)
    headers = [os.path.join(CSRC, h) for h in HEADERS] + [os.path.join(INCLUDE, "imq.h")]
    nvcc = _nvcc()
    objs, procs = [], []
    for src in SOURCES:
        s = os.path.join(CSRC, src)
        o = os.path.join(bdir, src.replace(".cu", ".o"))
        objs.append(o)
        if force or _stale(o, [s] + headers):
            cmd = [nvcc] + ARCH + FLAGS + (["-DIMQ_DEBUG"] if debug else []) + \
                (["-Xptxas", "-v"] if verbose else []) + ["-c", s, "-o", o]
            procs.append((src, subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT,
                                                text=True)))
    failed = []
    for src, p in procs:
        out, _ = p.communicate()
        if out and (verbose or p.returncode):
            sys.stderr.write(f"--- {src}\n{out}")
        if p.returncode:
            failed.append(src)
    if failed:
        raise RuntimeError(f"nvcc failed for {failed}")
    if force or _stale(lib, objs):
        tmp = lib + f".tmp{os.getpid()}"
        subprocess.run([nvcc] + ARCH + ["-shared", "-o", tmp] + objs, check=True)
        os.replace(tmp, lib)
    return lib


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--debug", action="store_true", help="build libimq_debug.so (IMQ_DEBUG index checks)")
    a = ap.parse_args()
    print(build(a.force, a.verbose, a.debug))


if __name__ == "__main__":
    main()
