"""fp64 CPU oracle of the LatentMoE layer forward -- TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. It shares no code with the CUDA
library (``latentmoe_layer_b200``); the only common dependency is the seeded
input generator in ``synth``. The arithmetic lives in ``oracle.c`` (plain
loops, fp64, OpenMP over tokens); this module only marshals arguments.

What each function computes and which passage it follows is stated in
``oracle.h``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "liboracle.so")
_lib = None


class LmoCfg(ctypes.Structure):
    _fields_ = [("H", ctypes.c_int), ("L", ctypes.c_int), ("E", ctypes.c_int), ("k", ctypes.c_int),
                ("G", ctypes.c_int), ("Gk", ctypes.c_int), ("I", ctypes.c_int), ("Is", ctypes.c_int),
                ("s", ctypes.c_double), ("x_f32", ctypes.c_int), ("fp32_mode", ctypes.c_int)]


class LmoWeights(ctypes.Structure):
    _fields_ = [("router_w", ctypes.c_void_p), ("e_bias", ctypes.c_void_p), ("fc1_w", ctypes.c_void_p),
                ("fc2_w", ctypes.c_void_p), ("up_w", ctypes.c_void_p), ("down_w", ctypes.c_void_p),
                ("shared_up_w", ctypes.c_void_p), ("shared_down_w", ctypes.c_void_p),
                ("up_gs", ctypes.c_void_p), ("down_gs", ctypes.c_void_p)]


def build(force: bool = False):
    srcs = [os.path.join(_HERE, "oracle.c"), os.path.join(_HERE, "oracle.h")]
    if not force and os.path.exists(_SO) and all(os.path.getmtime(s) <= os.path.getmtime(_SO) for s in srcs):
        return
    cmd = ["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off", "-std=c11", srcs[0], "-o", _SO, "-lm"]
    r = subprocess.run(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT, text=True)
    if r.returncode != 0:
        raise RuntimeError("oracle build failed:\n" + r.stdout)


def _get():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_SO)
        vp, i64 = ctypes.c_void_p, ctypes.c_int64
        lib.lmo_round_bf16.argtypes = [ctypes.c_double]
        lib.lmo_round_bf16.restype = ctypes.c_double
        lib.lmo_select.argtypes = [vp, vp, vp]
        lib.lmo_logits.argtypes = [vp, vp, vp, i64, vp]
        lib.lmo_route.argtypes = [vp, vp, vp, vp, i64, vp, vp]
        lib.lmo_latent.argtypes = [vp, vp, vp, i64, vp]
        lib.lmo_latent.restype = ctypes.c_int
        lib.lmo_forward.argtypes = [vp, vp, vp, i64, vp, vp, vp]
        lib.lmo_update_bias.argtypes = [ctypes.c_int, vp, vp, ctypes.c_double, vp, vp]
        lib.lmo_rmsnorm.argtypes = [ctypes.c_int, vp, vp, ctypes.c_double, i64, vp]
        lib.lmo_rmsnorm.restype = ctypes.c_int
        lib.lmo_forward_block.argtypes = [vp, vp, vp, ctypes.c_double, vp, i64, vp, vp, vp]
        lib.lmo_forward_block.restype = ctypes.c_int
        lib.lmo_update_bias.restype = ctypes.c_int
        lib.lmo_e2m1_value.argtypes = [ctypes.c_int]
        lib.lmo_e2m1_value.restype = ctypes.c_double
        lib.lmo_e4m3_value.argtypes = [ctypes.c_int]
        lib.lmo_e4m3_value.restype = ctypes.c_double
        lib.lmo_e2m1_encode.argtypes = [ctypes.c_float]
        lib.lmo_e2m1_encode.restype = ctypes.c_int
        lib.lmo_e4m3_encode.argtypes = [ctypes.c_float]
        lib.lmo_e4m3_encode.restype = ctypes.c_int
        lib.lmo_nvfp4_quantize.argtypes = [vp, i64, ctypes.c_int, ctypes.c_int, vp, vp, vp]
        lib.lmo_nvfp4_quantize.restype = ctypes.c_int
        lib.lmo_nvfp4_dequant.argtypes = [vp, vp, i64, ctypes.c_int, ctypes.c_int, vp]
        lib.lmo_nvfp4_dequant.restype = ctypes.c_int
        for f in (lib.lmo_select, lib.lmo_logits, lib.lmo_route, lib.lmo_forward):
            f.restype = ctypes.c_int
        _lib = lib
    return _lib


def make_cfg(shape, fp32_mode=False, x_f32=None) -> LmoCfg:
    """shape: any object with H, L, E, k, G, Gk, I, Is, s (and x_f32)."""
    xf = shape.x_f32 if x_f32 is None else x_f32
    return LmoCfg(shape.H, shape.L, shape.E, shape.k, shape.G, shape.Gk, shape.I, shape.Is, float(shape.s),
                  int(bool(xf)), int(bool(fp32_mode)))


def _c(a, dtype):
    a = np.ascontiguousarray(a)
    assert a.dtype == dtype, (a.dtype, dtype)
    return a


def _xarr(cfg: LmoCfg, x):
    return _c(x, np.float32 if cfg.x_f32 else np.uint16)


def round_bf16(v: float) -> float:
    return _get().lmo_round_bf16(float(v))


def select(cfg: LmoCfg, c) -> np.ndarray:
    c = _c(np.asarray(c, dtype=np.float64), np.float64)
    sel = np.zeros(cfg.k, dtype=np.int32)
    rc = _get().lmo_select(ctypes.byref(cfg), c.ctypes.data, sel.ctypes.data)
    if rc != 0:
        raise ValueError("invalid selection configuration")
    return sel


def logits(cfg: LmoCfg, x, router_w) -> np.ndarray:
    x = _xarr(cfg, x)
    rw = _c(router_w, np.uint16)
    n = x.shape[0]
    out = np.zeros((n, cfg.E), dtype=np.float64)
    _get().lmo_logits(ctypes.byref(cfg), x.ctypes.data, rw.ctypes.data, n, out.ctypes.data)
    return out


def latent(cfg: LmoCfg, x, fc1_w) -> np.ndarray:
    """fc1_latent_proj of the rows of x before its bf16 rounding (fp64 [n, L])."""
    x = _xarr(cfg, x)
    w = _c(fc1_w, np.uint16)
    n = x.shape[0]
    out = np.zeros((n, cfg.L), dtype=np.float64)
    _get().lmo_latent(ctypes.byref(cfg), x.ctypes.data, w.ctypes.data, n, out.ctypes.data)
    return out


def route(cfg: LmoCfg, x, router_w, e_bias):
    x = _xarr(cfg, x)
    rw = _c(router_w, np.uint16)
    b = _c(e_bias, np.float32)
    n = x.shape[0]
    idx = np.zeros((n, cfg.k), dtype=np.int32)
    w = np.zeros((n, cfg.k), dtype=np.float64)
    rc = _get().lmo_route(ctypes.byref(cfg), x.ctypes.data, rw.ctypes.data, b.ctypes.data, n, idx.ctypes.data,
                          w.ctypes.data)
    if rc != 0:
        raise ValueError("routing failed (invalid configuration)")
    return idx, w


def _weights(cfg: LmoCfg, wts: dict, keep: list):
    def ptr(a, dt):
        a = _c(a, dt)
        keep.append(a)
        return a.ctypes.data

    def expert_ptrs(arr):
        ps = (ctypes.c_void_p * cfg.E)()
        for e in range(cfg.E):
            a = arr[e]
            ps[e] = None if a is None else ptr(a, np.uint16)
        keep.append(ps)
        return ctypes.cast(ps, ctypes.c_void_p).value

    def opt_scales(key):
        g = wts.get(key)
        return None if g is None else ptr(np.asarray(g, dtype=np.float32), np.float32)

    return LmoWeights(ptr(wts["router_w"], np.uint16), ptr(wts["e_bias"], np.float32), ptr(wts["fc1_w"], np.uint16),
                      ptr(wts["fc2_w"], np.uint16), expert_ptrs(wts["up_w"]), expert_ptrs(wts["down_w"]),
                      ptr(wts["shared_up_w"], np.uint16), ptr(wts["shared_down_w"], np.uint16),
                      opt_scales("up_gs"), opt_scales("down_gs"))


def forward(cfg: LmoCfg, x, wts: dict):
    """Full layer on the rows of x. wts: router_w, e_bias, fc1_w, fc2_w, up_w, down_w,
    shared_up_w, shared_down_w (bf16 as uint16). up_w/down_w are [E, ...] arrays or
    lists of per-expert arrays (None where not needed). Optional up_gs / down_gs
    ([E] fp32): per-expert matrix scales of NVFP4 experts (up_w/down_w then hold
    the dequantised code * block-scale values, see nvfp4_dequant)."""
    x = _xarr(cfg, x)
    n = x.shape[0]
    keep = []
    W = _weights(cfg, wts, keep)
    idx = np.zeros((n, cfg.k), dtype=np.int32)
    w = np.zeros((n, cfg.k), dtype=np.float64)
    y = np.zeros((n, cfg.H), dtype=np.float64)
    rc = _get().lmo_forward(ctypes.byref(cfg), x.ctypes.data, ctypes.byref(W), n, idx.ctypes.data, w.ctypes.data,
                            y.ctypes.data)
    if rc != 0:
        raise ValueError("oracle forward failed (invalid configuration or missing expert weights)")
    return y, idx, w


def rmsnorm(x, gamma, eps):
    x = _c(x, np.uint16)
    g = _c(gamma, np.uint16)
    out = np.zeros_like(x)
    _get().lmo_rmsnorm(x.shape[1], x.ctypes.data, g.ctypes.data, float(eps), x.shape[0], out.ctypes.data)
    return out


def forward_block(cfg: LmoCfg, x, gamma, eps, wts: dict):
    """y = x + layer(rmsnorm(x)) (x bf16)."""
    x = _c(x, np.uint16)
    g = _c(gamma, np.uint16)
    n = x.shape[0]
    keep = []
    W = _weights(cfg, wts, keep)
    idx = np.zeros((n, cfg.k), dtype=np.int32)
    w = np.zeros((n, cfg.k), dtype=np.float64)
    y = np.zeros((n, cfg.H), dtype=np.float64)
    rc = _get().lmo_forward_block(ctypes.byref(cfg), x.ctypes.data, g.ctypes.data, float(eps), ctypes.byref(W), n,
                                  idx.ctypes.data, w.ctypes.data, y.ctypes.data)
    if rc != 0:
        raise ValueError("oracle block forward failed")
    return y, idx, w


def update_bias(counts, bias, eta):
    """Returns (new bias fp32 [E], MaxVio)."""
    counts = _c(np.asarray(counts, dtype=np.int32), np.int32)
    bias = _c(np.asarray(bias, dtype=np.float32), np.float32)
    out = np.zeros_like(bias)
    mv = ctypes.c_double()
    _get().lmo_update_bias(len(bias), counts.ctypes.data, bias.ctypes.data, float(eta), out.ctypes.data,
                           ctypes.byref(mv))
    return out, mv.value


# ---------------------------------------------------------------- NVFP4
def e2m1_value(code: int) -> float:
    return _get().lmo_e2m1_value(int(code))


def e4m3_value(byte: int) -> float:
    return _get().lmo_e4m3_value(int(byte))


def e2m1_encode(q: float) -> int:
    return _get().lmo_e2m1_encode(float(q))


def e4m3_encode(u: float) -> int:
    return _get().lmo_e4m3_encode(float(u))


def nvfp4_quantize(w):
    """w: [n_mat, R, K] bf16 bits (uint16). Returns (codes uint8 [n_mat*R*K/2],
    sf uint8 [n_mat*R*K/16], g float32 [n_mat]) in the tiled layout of oracle.h."""
    w = _c(w, np.uint16)
    n_mat, R, K = w.shape
    codes = np.zeros(n_mat * R * K // 2, dtype=np.uint8)
    sf = np.zeros(n_mat * R * K // 16, dtype=np.uint8)
    g = np.zeros(n_mat, dtype=np.float32)
    rc = _get().lmo_nvfp4_quantize(w.ctypes.data, n_mat, R, K, codes.ctypes.data, sf.ctypes.data, g.ctypes.data)
    if rc != 0:
        raise ValueError("NVFP4 quantisation needs R % 128 == 0 and K % 64 == 0")
    return codes, sf, g


def nvfp4_dequant(codes, sf, n_mat, R, K):
    """bf16 bits [n_mat, R, K] of code_value * block scale (the matrix scale g not applied)."""
    codes = _c(codes, np.uint8)
    sf = _c(sf, np.uint8)
    out = np.zeros((n_mat, R, K), dtype=np.uint16)
    rc = _get().lmo_nvfp4_dequant(codes.ctypes.data, sf.ctypes.data, n_mat, R, K, out.ctypes.data)
    if rc != 0:
        raise ValueError("NVFP4 dequantisation: bad shape or inexact product")
    return out
