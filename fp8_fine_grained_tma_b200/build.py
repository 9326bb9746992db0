"""Build libfg8.so in-tree with nvcc for sm_100a.

    python -m fp8_fine_grained_tma_b200.build [--force] [--jobs N] [--verbose]

Each GEMM block width (16..256 in steps of 16) is one object compiled from
csrc/gemm_inst.cu with -DFG8_BN=<width>, and each decode token-tile width
(32..256 in steps of 32) one object from csrc/decode_inst.cu with
-DFG8_MT=<width>, all in parallel; the host code is csrc/fg8_host.cu.  The CUDA runtime is linked statically, so the library
needs only the NVIDIA driver at run time.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libfg8.so")
BLOCK_NS = list(range(16, 257, 16))
DECODE_MTS = list(range(32, 257, 32))
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden", "-I", INCLUDE,
         "-I", CSRC]


def nvcc() -> str:
    cand = os.environ.get("NVCC") or shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    return cand


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*")) + [os.path.join(INCLUDE, "fg8.h")])


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(s) <= t for s in _sources())


def _run(cmd, verbose):
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("command failed:\n" + " ".join(cmd) + "\n" + r.stdout + r.stderr)
    if verbose and (r.stdout or r.stderr):
        print(r.stdout + r.stderr, end="")
    return r


def build(force: bool = False, jobs: int = 0, verbose: bool = False) -> str:
    if not force and up_to_date():
        return LIB
    os.makedirs(BUILD, exist_ok=True)
    cmds = []
    objs = []
    ptxas = ["-Xptxas", "-v"] if verbose else []
    for bn in BLOCK_NS:
        o = os.path.join(BUILD, f"gemm_bn_{bn}.o")
        objs.append(o)
        cmds.append([nvcc(), *ARCH, *FLAGS, *ptxas, f"-DFG8_BN={bn}", "-c",
                     os.path.join(CSRC, "gemm_inst.cu"), "-o", o])
    for mt in DECODE_MTS:
        o = os.path.join(BUILD, f"decode_mt_{mt}.o")
        objs.append(o)
        cmds.append([nvcc(), *ARCH, *FLAGS, *ptxas, f"-DFG8_MT={mt}", "-c",
                     os.path.join(CSRC, "decode_inst.cu"), "-o", o])
    for src in ["fg8_host.cu", "quant.cu", "jit.cu"]:
        o = os.path.join(BUILD, src.replace(".cu", ".o"))
        objs.append(o)
        cmds.append([nvcc(), *ARCH, *FLAGS, *ptxas, "-c", os.path.join(CSRC, src), "-o", o])
    jobs = jobs or max(1, min(len(cmds), os.cpu_count() or 1))
    with cf.ThreadPoolExecutor(jobs) as ex:
        list(ex.map(lambda c: _run(c, verbose), cmds))
    tmp = LIB + f".tmp{os.getpid()}"
    _run([nvcc(), *ARCH, "-shared", "-o", tmp, *objs, "-ldl"], verbose)
    os.replace(tmp, LIB)
    return LIB


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--jobs", type=int, default=0)
    ap.add_argument("--verbose", action="store_true")
    a = ap.parse_args(argv)
    print(build(a.force, a.jobs, a.verbose))


if __name__ == "__main__":
    sys.exit(main())
