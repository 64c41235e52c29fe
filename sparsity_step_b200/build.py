"""Compile the CUDA library ``libbitlinear.so`` (sm_100a) in-tree with nvcc.

Usage: ``python -m sparsity_step_b200.build [--force] [--verbose]``.
"""
from __future__ import annotations

import argparse
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libbitlinear.so")
MAIN = os.path.join(CSRC, "bitlinear_api.cu")
# measurement-only tensor-pipe probe (not part of the BitLinear ABI)
PROBE_LIB = os.path.join(PKG, "libblprobe.so")
PROBE_SRC = os.path.join(CSRC, "probe_mma_peak.cu")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-shared", "-Xcompiler", "-fPIC",
    "--expt-relaxed-constexpr",
]


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))) + [
        os.path.join(ROOT, "include", "bitlinear.h")]


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(s) <= t for s in sources())


def _nvcc(out: str, src: str, verbose: bool, extra: list[str] | None) -> None:
    cmd = [nvcc_path(), *NVCC_FLAGS, *(extra or []), "-o", out + ".tmp", src]
    if verbose:
        print(" ".join(cmd), flush=True)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed ({res.returncode}):\n{res.stdout}\n{res.stderr}")
    if verbose and (res.stdout or res.stderr):
        print(res.stdout, res.stderr, sep="\n")
    os.replace(out + ".tmp", out)


def build(force: bool = False, verbose: bool = False, extra: list[str] | None = None) -> str:
    if force or not up_to_date(LIB):
        _nvcc(LIB, MAIN, verbose, extra)
    if force or not up_to_date(PROBE_LIB):
        _nvcc(PROBE_LIB, PROBE_SRC, verbose, extra)
    return LIB


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--ptxas-v", action="store_true", help="print register / shared-memory usage")
    a = ap.parse_args(argv)
    extra = ["-Xptxas", "-v"] if a.ptxas_v else None
    print(build(force=a.force or a.ptxas_v, verbose=a.verbose or a.ptxas_v, extra=extra))
    return 0


if __name__ == "__main__":
    sys.exit(main())
