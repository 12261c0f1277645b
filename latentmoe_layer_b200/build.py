"""Build step of the CUDA library: nvcc, sm_100a, in-tree liblatentmoe.so."""
from __future__ import annotations

import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
SO = os.path.join(HERE, "liblatentmoe.so")
SOURCES = ["api.cu", "router.cu", "permute.cu", "gemm_tc.cu", "gemm_nvfp4.cu", "gemm_simt.cu", "nvfp4.cu", "zcheck.cu"]
HEADERS = ["lmoe_internal.h", "handle.h", "ptx.cuh", "gemm_common.cuh"]
FLAGS = ["-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-Xcompiler", "-fPIC",
         "-shared", "--expt-relaxed-constexpr", "-Xptxas", "-v"]


def _stale() -> bool:
    if not os.path.exists(SO):
        return True
    t = os.path.getmtime(SO)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    deps.append(os.path.join(HERE, "..", "include", "latentmoe.h"))
    deps.append(os.path.abspath(__file__))
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not _stale():
        return SO
    cmd = ["nvcc", *FLAGS, *[os.path.join(CSRC, f) for f in SOURCES], "-o", SO + ".tmp"]
    r = subprocess.run(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT, text=True)
    if r.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + r.stdout)
    os.replace(SO + ".tmp", SO)
    if verbose:
        print(r.stdout)
    with open(os.path.join(HERE, "ptxas_info.txt"), "w") as f:
        f.write(r.stdout)
    return SO


if __name__ == "__main__":
    build(force=True, verbose=True)
