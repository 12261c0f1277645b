"""Build step of the CUDA library: nvcc, sm_100a, in-tree liblatentmoe.so.

Two targets from the same sources:
  liblatentmoe.so         the library (what every caller loads);
  liblatentmoe_checks.so  the checking build (LMOE_CHECKS=1): device-side bounds
                          checks on every index a kernel reads from memory (tile
                          records, permutation and slot indices, flag and z lists)
                          that record LMOE_ERR_INVALID_ARG and skip the access.
"""
from __future__ import annotations

import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
SO = os.path.join(HERE, "liblatentmoe.so")
SO_CHECKS = os.path.join(HERE, "liblatentmoe_checks.so")
SOURCES = ["api.cu", "router.cu", "permute.cu", "gemm_tc.cu", "gemm_nvfp4.cu", "gemm_simt.cu", "nvfp4.cu", "zcheck.cu"]
HEADERS = ["lmoe_internal.h", "handle.h", "ptx.cuh", "gemm_common.cuh"]
FLAGS = ["-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-Xcompiler", "-fPIC",
         "-shared", "--expt-relaxed-constexpr", "-Xptxas", "-v"]


def _stale(target) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    deps.append(os.path.join(HERE, "..", "include", "latentmoe.h"))
    deps.append(os.path.abspath(__file__))
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, checks: bool = False) -> str:
    target = SO_CHECKS if checks else SO
    if not force and not _stale(target):
        return target
    extra = ["-DLMOE_CHECKS=1"] if checks else []
    cmd = ["nvcc", *FLAGS, *extra, *[os.path.join(CSRC, f) for f in SOURCES], "-o", target + ".tmp"]
    r = subprocess.run(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT, text=True)
    if r.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + r.stdout)
    os.replace(target + ".tmp", target)
    if verbose:
        print(r.stdout)
    if not checks:
        with open(os.path.join(HERE, "ptxas_info.txt"), "w") as f:
            f.write(r.stdout)
    return target


def build_all(force: bool = False) -> None:
    build(force=force)
    build(force=force, checks=True)


if __name__ == "__main__":
    build_all(force=True)
