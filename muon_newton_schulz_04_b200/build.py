"""Builds libmuon_b200.so in-tree with nvcc for sm_100a.

    python -m muon_newton_schulz_04_b200.build          # incremental
    python -m muon_newton_schulz_04_b200.build --force  # rebuild everything

Objects go to muon_newton_schulz_04_b200/_build/, the shared library next to
this file.  The CUDA runtime is linked statically and the driver is reached at
run time through cudaGetDriverEntryPoint, so the library loads on a machine
without a GPU (its entry points then report MUON_ERR_CUDA).
"""
from __future__ import annotations

import argparse
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libmuon_b200.so")
SOURCES = ["api.cu", "elementwise.cu", "gemm_tc.cu", "gemm_simt.cu", "plan.cpp", "noalloc.cu"]
HEADERS = ["kernels.cuh", "ptx.cuh", "plan.h"]

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
# extra nvcc flags for experiments with compile-time constants (e.g. -DMUON_S2_STAGES=7)
EXTRA = os.environ.get("MUON_NVCC_EXTRA", "").split()
NVCC_FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-O3", "-Xptxas", "-v",
              "--expt-relaxed-constexpr", f"-I{os.path.join(ROOT, 'include')}"]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    return "nvcc"


def _newest_dep() -> float:
    deps = [os.path.join(CSRC, h) for h in HEADERS] + [os.path.join(ROOT, "include", "muon.h"), __file__]
    return max(os.path.getmtime(p) for p in deps if os.path.exists(p))


def build(force: bool = False, verbose: bool = False) -> str:
    os.makedirs(BUILD, exist_ok=True)
    nvcc = _nvcc()
    dep_t = _newest_dep()
    jobs = []
    objs = []
    for src in SOURCES:
        sp = os.path.join(CSRC, src)
        op = os.path.join(BUILD, src + ".o")
        objs.append(op)
        if force or not os.path.exists(op) or os.path.getmtime(op) < max(os.path.getmtime(sp), dep_t):
            jobs.append([nvcc, *ARCH, *NVCC_FLAGS, *EXTRA, "-x", "cu" if src.endswith(".cu") else "c++", "-c", sp, "-o", op])

    def run(cmd):
        r = subprocess.run(cmd, capture_output=True, text=True)
        return cmd, r

    with ThreadPoolExecutor(max_workers=len(jobs) or 1) as ex:
        results = list(ex.map(run, jobs))
    for cmd, r in results:
        if r.returncode != 0:
            sys.stderr.write(r.stdout + r.stderr)
            raise RuntimeError(f"nvcc failed: {' '.join(cmd)}")
        if verbose:
            sys.stderr.write(r.stderr)
    if jobs or not os.path.exists(LIB):
        cmd = [nvcc, *ARCH, "-shared", "-o", LIB, *objs, "-cudart", "static", "-Xcompiler", "-fPIC"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            sys.stderr.write(r.stdout + r.stderr)
            raise RuntimeError("link failed")
    return LIB


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("-v", "--verbose", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose))


if __name__ == "__main__":
    main()
