"""Seeded synthetic inputs for the LatentMoE layer (host and device).

The generator is defined in synth.h and implemented twice: synth.c (host,
used by the oracle side) and synth_cuda.cu (device, used to fill multi-GB
weight sets directly in HBM). This package holds none of the layer's
arithmetic; it is shared by the tests, the oracle side and the benchmark.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

from .workloads import (LayerShape, WORKLOADS, TINY, NANO_DECODE, ULTRA_DECODE, ULTRA_PREFILL, ULTRA_SKEW,
                        tensor_specs, W_SIGMA, BIAS_LO, BIAS_HI, TID_X, TID_ROUTER)

_HERE = os.path.dirname(os.path.abspath(__file__))
_CPU_SO = os.path.join(_HERE, "libsynth.so")
_GPU_SO = os.path.join(_HERE, "libsynth_cuda.so")
_cpu = None
_gpu = None

BF16_ONE = 0x3F80
BF16_THREE = 0x4040


def _run(cmd):
    r = subprocess.run(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT, text=True)
    if r.returncode != 0:
        raise RuntimeError("build failed: %s\n%s" % (" ".join(cmd), r.stdout))


def _stale(target, sources):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(s) > t for s in sources)


def build(force: bool = False, cuda: bool = True):
    """Compile libsynth.so (gcc, OpenMP) and libsynth_cuda.so (nvcc, sm_100a)."""
    src_c = [os.path.join(_HERE, "synth.c"), os.path.join(_HERE, "synth.h")]
    if force or _stale(_CPU_SO, src_c):
        _run(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off", "-std=c11",
              src_c[0], "-o", _CPU_SO, "-lm"])
    if cuda:
        src_cu = [os.path.join(_HERE, "synth_cuda.cu")]
        if force or _stale(_GPU_SO, src_cu):
            _run(["nvcc", "-O2", "-shared", "-Xcompiler", "-fPIC", "--fmad=false",
                  "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", src_cu[0], "-o", _GPU_SO])


def _cpu_lib():
    global _cpu
    if _cpu is None:
        if not os.path.exists(_CPU_SO):
            build(cuda=False)
        lib = ctypes.CDLL(_CPU_SO)
        u64, i64, dbl, vp = ctypes.c_uint64, ctypes.c_int64, ctypes.c_double, ctypes.c_void_p
        lib.synth_normal_f64.argtypes = [u64, u64, u64]
        lib.synth_normal_f64.restype = dbl
        lib.synth_uniform_f64.argtypes = [u64, u64, u64, dbl, dbl]
        lib.synth_uniform_f64.restype = dbl
        lib.synth_fill_normal_bf16.argtypes = [vp, i64, u64, u64, dbl, i64]
        lib.synth_fill_normal_f32.argtypes = [vp, i64, u64, u64, dbl, i64]
        lib.synth_fill_uniform_f32.argtypes = [vp, i64, u64, u64, dbl, dbl, i64]
        _cpu = lib
    return _cpu


def _gpu_lib():
    global _gpu
    if _gpu is None:
        if not os.path.exists(_GPU_SO):
            build()
        lib = ctypes.CDLL(_GPU_SO)
        u64, i64, dbl, vp = ctypes.c_uint64, ctypes.c_int64, ctypes.c_double, ctypes.c_void_p
        lib.synth_cuda_fill_normal_bf16.argtypes = [vp, i64, u64, u64, dbl, i64, vp]
        lib.synth_cuda_fill_normal_f32.argtypes = [vp, i64, u64, u64, dbl, i64, vp]
        lib.synth_cuda_fill_uniform_f32.argtypes = [vp, i64, u64, u64, dbl, dbl, i64, vp]
        for f in (lib.synth_cuda_fill_normal_bf16, lib.synth_cuda_fill_normal_f32, lib.synth_cuda_fill_uniform_f32):
            f.restype = ctypes.c_int
        _gpu = lib
    return _gpu


# ---------------------------------------------------------------- host side
def normal_bf16(n, seed, tid, sigma, offset=0) -> np.ndarray:
    out = np.empty(n, dtype=np.uint16)
    _cpu_lib().synth_fill_normal_bf16(out.ctypes.data, n, seed, tid, sigma, offset)
    return out


def normal_f32(n, seed, tid, sigma, offset=0) -> np.ndarray:
    out = np.empty(n, dtype=np.float32)
    _cpu_lib().synth_fill_normal_f32(out.ctypes.data, n, seed, tid, sigma, offset)
    return out


def uniform_f32(n, seed, tid, lo, hi, offset=0) -> np.ndarray:
    out = np.empty(n, dtype=np.float32)
    _cpu_lib().synth_fill_uniform_f32(out.ctypes.data, n, seed, tid, lo, hi, offset)
    return out


def host_tensor(w: LayerShape, key: str, seed: int = 0, rows=None) -> np.ndarray:
    """One input tensor on the host (bf16 as uint16 bits). rows=(r0, r1) slices the leading dim."""
    for k, tid, shape, kind in tensor_specs(w):
        if k != key:
            continue
        inner = int(np.prod(shape[1:])) if len(shape) > 1 else 1
        r0, r1 = (0, shape[0]) if rows is None else rows
        n = (r1 - r0) * inner
        off = r0 * inner
        oshape = (r1 - r0,) + tuple(shape[1:])
        if kind == "b":
            a = uniform_f32(n, seed, tid, BIAS_LO, BIAS_HI, off)
        elif kind == "x" and w.x_f32:
            a = normal_f32(n, seed, tid, 1.0, off)
        elif kind == "x":
            a = normal_bf16(n, seed, tid, 1.0, off)
        else:
            a = normal_bf16(n, seed, tid, W_SIGMA, off)
        a = a.reshape(oshape)
        if w.skew_hot and key == "x":
            a[:, 0] = 1.0 if w.x_f32 else BF16_ONE
        if w.skew_hot and key == "router_w":
            assert w.skew_offset == 3.0, "skew offset must be representable; 3.0 is"
            lo, hi = max(r0, 0), min(r1, w.skew_hot)
            if hi > lo:
                a[lo - r0:hi - r0, 0] = BF16_THREE
        return a
    raise KeyError(key)


def element(w: LayerShape, key: str, flat: int, seed: int = 0):
    """Stored value of one element (uint16 bits for bf16, float for fp32), overrides included."""
    for k, tid, shape, kind in tensor_specs(w):
        if k != key:
            continue
        inner = int(np.prod(shape[1:])) if len(shape) > 1 else 1
        r, c = divmod(int(flat), inner)
        if w.skew_hot and key == "x" and c == 0:
            return 1.0 if w.x_f32 else BF16_ONE
        if w.skew_hot and key == "router_w" and c == 0 and r < w.skew_hot:
            return BF16_THREE
        if kind == "b":
            return float(uniform_f32(1, seed, tid, BIAS_LO, BIAS_HI, flat)[0])
        if kind == "x" and w.x_f32:
            return float(normal_f32(1, seed, tid, 1.0, flat)[0])
        return int(normal_bf16(1, seed, tid, 1.0 if kind == "x" else W_SIGMA, flat)[0])
    raise KeyError(key)


def host_inputs(w: LayerShape, seed: int = 0) -> dict:
    return {k: host_tensor(w, k, seed) for k, _, _, _ in tensor_specs(w)}


# -------------------------------------------------------------- device side
def device_inputs(w: LayerShape, seed: int = 0, device="cuda") -> dict:
    """Allocate and fill every input of the layer directly in HBM."""
    import torch
    lib = _gpu_lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)
    out = {}
    for k, tid, shape, kind in tensor_specs(w):
        n = int(np.prod(shape))
        if kind == "b":
            t = torch.empty(shape, dtype=torch.float32, device=device)
            rc = lib.synth_cuda_fill_uniform_f32(t.data_ptr(), n, seed, tid, BIAS_LO, BIAS_HI, 0, stream)
        elif kind == "x" and w.x_f32:
            t = torch.empty(shape, dtype=torch.float32, device=device)
            rc = lib.synth_cuda_fill_normal_f32(t.data_ptr(), n, seed, tid, 1.0, 0, stream)
        else:
            t = torch.empty(shape, dtype=torch.bfloat16, device=device)
            sigma = 1.0 if kind == "x" else W_SIGMA
            rc = lib.synth_cuda_fill_normal_bf16(t.data_ptr(), n, seed, tid, sigma, 0, stream)
        if rc != 0:
            raise RuntimeError("device generator failed with cudaError %d" % rc)
        out[k] = t
    if w.skew_hot:
        out["x"][:, 0] = 1.0
        out["router_w"][: w.skew_hot, 0] = 3.0
    return out


def bf16_bits_to_f32(a: np.ndarray) -> np.ndarray:
    return (a.astype(np.uint32) << 16).view(np.float32)


__all__ = ["LayerShape", "WORKLOADS", "TINY", "NANO_DECODE", "ULTRA_DECODE", "ULTRA_PREFILL", "ULTRA_SKEW",
           "tensor_specs", "host_tensor", "host_inputs", "device_inputs", "build", "normal_bf16", "normal_f32",
           "uniform_f32", "bf16_bits_to_f32", "element", "TID_X", "TID_ROUTER"]
