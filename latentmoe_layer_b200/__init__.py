"""Python binding of the B200 LatentMoE layer library (liblatentmoe.so).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels. PyTorch provides device memory and the current stream. The entry
points keep the C names (include/latentmoe.h); ``LatentMoE`` is a small
convenience wrapper that owns a handle and a workspace.

Importing this package does not load the library; the first call does, and it
raises ``RuntimeError`` if liblatentmoe.so has not been built (there is no
fallback implementation). With ``LATENTMOE_CHECKS=1`` in the environment the
checking build (liblatentmoe_checks.so: device-side bounds checks that report
LMOE_ERR_INVALID_ARG instead of touching memory out of range) is loaded instead;
``LATENTMOE_LIB=<path>`` loads that build of the library.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.environ.get("LATENTMOE_LIB") or os.path.join(
    _HERE, "liblatentmoe_checks.so" if os.environ.get("LATENTMOE_CHECKS") == "1" else "liblatentmoe.so")

LMOE_OK, LMOE_ERR_INVALID_ARG, LMOE_ERR_UNSUPPORTED, LMOE_ERR_WORKSPACE, LMOE_ERR_CUDA, LMOE_ERR_TIMEOUT, \
    LMOE_ERR_INTERNAL = range(7)
LMOE_BF16, LMOE_FP32 = 0, 1
LMOE_MODE_BF16, LMOE_MODE_FP32 = 0, 1
LMOE_EXPERTS_BF16, LMOE_EXPERTS_NVFP4 = 0, 1
OPT_GEMM_PATH, OPT_ROUTER_FP64_ALL, OPT_FLAG_DELTA, OPT_SPIN_LIMIT, OPT_Z_RECHECK_DELTA, OPT_ACT_RECHECK_TAU = range(6)
GEMM_AUTO, GEMM_PREFILL, GEMM_DECODE, GEMM_SIMT, GEMM_PREFILL_PAIR = range(5)

EXPORTS = ["latentmoe_create", "latentmoe_workspace_size", "latentmoe_route", "latentmoe_forward",
           "latentmoe_destroy", "latentmoe_status_string", "latentmoe_set_option", "latentmoe_read_stats",
           "latentmoe_selftest_bounded_wait", "latentmoe_set_profile_events", "latentmoe_route_noalloc", "latentmoe_update_bias", "latentmoe_forward_block",
           "latentmoe_quantize_nvfp4", "latentmoe_ep_front", "latentmoe_ep_workspace_size", "latentmoe_ep_experts",
           "latentmoe_ep_back", "latentmoe_workspace_layout"]


class lmoe_config(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int), ("latent", ctypes.c_int), ("num_experts", ctypes.c_int),
                ("top_k", ctypes.c_int), ("n_group", ctypes.c_int), ("topk_group", ctypes.c_int),
                ("expert_inter", ctypes.c_int), ("shared_inter", ctypes.c_int), ("max_tokens", ctypes.c_int),
                ("routed_scaling_factor", ctypes.c_float), ("x_dtype", ctypes.c_int), ("mode", ctypes.c_int),
                ("expert_format", ctypes.c_int), ("local_experts", ctypes.c_int), ("expert_base", ctypes.c_int)]


class lmoe_weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("router_w", "e_bias", "fc1_w", "fc2_w", "up_w", "down_w",
                                                "shared_up_w", "shared_down_w", "up_sf", "down_sf", "up_gs",
                                                "down_gs")]


class lmoe_stats(ctypes.Structure):
    _fields_ = [("flagged_tokens", ctypes.c_int), ("distinct_experts", ctypes.c_int),
                ("max_expert_tokens", ctypes.c_int), ("device_error", ctypes.c_int),
                ("kernel_launches", ctypes.c_int), ("cuda_error", ctypes.c_int), ("z_rechecked", ctypes.c_int),
                ("ae_rechecked", ctypes.c_int), ("as_rechecked", ctypes.c_int)]


class lmoe_ws_layout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in ("logits_f32", "z_f32", "z", "flag_list", "perm", "slot", "total",
                                              "offsets", "act_e", "act_s")]


class LmoeError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__("%s: %s (status %d)" % (where, status_string(status), status))


_lib = None


def load():
    """Load liblatentmoe.so (raises if it is missing: there is no fallback)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError("liblatentmoe.so is not built (run `python -c 'import __graft_entry__ as g; g.build()'`); "
                           "the LatentMoE layer has no non-CUDA implementation")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    lib.latentmoe_create.argtypes = [ctypes.POINTER(lmoe_config), ctypes.POINTER(lmoe_weights), ctypes.POINTER(vp)]
    lib.latentmoe_workspace_size.argtypes = [vp, i32, ctypes.POINTER(sz)]
    lib.latentmoe_route.argtypes = [vp, vp, i32, vp, vp, vp, vp, sz, vp]
    lib.latentmoe_forward.argtypes = [vp, vp, i32, vp, vp, sz, vp, vp, vp, vp]
    lib.latentmoe_destroy.argtypes = [vp]
    lib.latentmoe_destroy.restype = None
    lib.latentmoe_status_string.argtypes = [i32]
    lib.latentmoe_status_string.restype = ctypes.c_char_p
    lib.latentmoe_set_option.argtypes = [vp, i32, ctypes.c_longlong]
    lib.latentmoe_read_stats.argtypes = [vp, vp, ctypes.POINTER(lmoe_stats)]
    lib.latentmoe_selftest_bounded_wait.argtypes = [vp]
    lib.latentmoe_set_profile_events.argtypes = [vp, vp, i32]
    lib.latentmoe_route_noalloc.argtypes = [vp, vp, i32, vp, vp, vp, vp]
    lib.latentmoe_update_bias.argtypes = [vp, vp, vp, ctypes.c_float, vp, vp, vp]
    lib.latentmoe_forward_block.argtypes = [vp, vp, i32, vp, ctypes.c_float, vp, vp, sz, vp, vp, vp, vp]
    lib.latentmoe_quantize_nvfp4.argtypes = [vp, ctypes.c_longlong, i32, i32, vp, vp, vp, vp]
    lib.latentmoe_ep_front.argtypes = [vp, vp, i32, vp, vp, vp, vp, sz, vp]
    lib.latentmoe_ep_workspace_size.argtypes = [vp, i32, i32, ctypes.POINTER(sz)]
    lib.latentmoe_ep_experts.argtypes = [vp, vp, vp, vp, i32, i32, vp, vp, sz, vp]
    lib.latentmoe_ep_back.argtypes = [vp, vp, i32, vp, vp, sz, vp]
    lib.latentmoe_workspace_layout.argtypes = [vp, i32, ctypes.POINTER(lmoe_ws_layout)]
    for f in ("latentmoe_create", "latentmoe_workspace_size", "latentmoe_route", "latentmoe_forward",
              "latentmoe_set_option", "latentmoe_read_stats", "latentmoe_selftest_bounded_wait",
              "latentmoe_set_profile_events", "latentmoe_route_noalloc", "latentmoe_update_bias",
              "latentmoe_forward_block", "latentmoe_quantize_nvfp4", "latentmoe_ep_front",
              "latentmoe_ep_workspace_size", "latentmoe_ep_experts", "latentmoe_ep_back",
              "latentmoe_workspace_layout"):
        getattr(lib, f).restype = i32
    _lib = lib
    return lib


def status_string(s: int) -> str:
    return load().latentmoe_status_string(int(s)).decode()


def _p(t):
    return None if t is None else t.data_ptr()


# ---------------------------------------------------------------- C entry points
def latentmoe_create(cfg: lmoe_config, w: lmoe_weights):
    h = ctypes.c_void_p()
    s = load().latentmoe_create(ctypes.byref(cfg), ctypes.byref(w), ctypes.byref(h))
    return s, h


def latentmoe_workspace_size(h, T: int):
    n = ctypes.c_size_t()
    s = load().latentmoe_workspace_size(h, T, ctypes.byref(n))
    return s, n.value


def latentmoe_route(h, x, T, idx, w, counts, ws, ws_bytes, stream):
    return load().latentmoe_route(h, x, T, idx, w, counts, ws, ws_bytes, stream)


def latentmoe_forward(h, x, T, y, ws, ws_bytes, stream, idx=None, w=None, counts=None):
    return load().latentmoe_forward(h, x, T, y, ws, ws_bytes, stream, idx, w, counts)


def latentmoe_forward_block(h, x, T, norm_w, norm_eps, y, ws, ws_bytes, stream, idx=None, w=None, counts=None):
    return load().latentmoe_forward_block(h, x, T, norm_w, norm_eps, y, ws, ws_bytes, stream, idx, w, counts)


def latentmoe_destroy(h):
    load().latentmoe_destroy(h)


def latentmoe_set_option(h, opt: int, value: int) -> int:
    return load().latentmoe_set_option(h, opt, value)


def latentmoe_read_stats(h, ws):
    st = lmoe_stats()
    s = load().latentmoe_read_stats(h, ws, ctypes.byref(st))
    return s, st


def latentmoe_set_profile_events(h, events, n: int) -> int:
    return load().latentmoe_set_profile_events(h, events, n)


def latentmoe_route_noalloc(h, x, T, idx, w, counts, stream) -> int:
    """Routing with the library's static scratch (no workspace, no allocation)."""
    return load().latentmoe_route_noalloc(h, x, T, idx, w, counts, stream)


def latentmoe_update_bias(h, counts, bias_in, eta, bias_out, maxvio, stream) -> int:
    return load().latentmoe_update_bias(h, counts, bias_in, eta, bias_out, maxvio, stream)


def latentmoe_quantize_nvfp4(w, n_mat, R, K, codes, sf, gs, stream) -> int:
    return load().latentmoe_quantize_nvfp4(w, n_mat, R, K, codes, sf, gs, stream)


def quantize_nvfp4(w):
    """NVFP4 of a bf16 CUDA tensor [n_mat, R, K] on the current stream. Returns
    (codes uint8 [n_mat*R*K/2], sf uint8 [n_mat*R*K/16], gs float32 [n_mat]) in
    the library's tiled layout (include/latentmoe.h)."""
    import torch
    n_mat, R, K = w.shape
    assert w.is_cuda and w.dtype == torch.bfloat16 and w.is_contiguous()
    codes = torch.empty(n_mat * R * K // 2, dtype=torch.uint8, device=w.device)
    sf = torch.empty(n_mat * R * K // 16, dtype=torch.uint8, device=w.device)
    gs = torch.empty(n_mat, dtype=torch.float32, device=w.device)
    s = latentmoe_quantize_nvfp4(_p(w), n_mat, R, K, _p(codes), _p(sf), _p(gs),
                                 ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    if s != LMOE_OK:
        raise LmoeError(s, "latentmoe_quantize_nvfp4")
    return codes, sf, gs


def latentmoe_workspace_layout(h, T: int):
    out = lmoe_ws_layout()
    s = load().latentmoe_workspace_layout(h, T, ctypes.byref(out))
    return s, out


def latentmoe_selftest_bounded_wait(h) -> int:
    return load().latentmoe_selftest_bounded_wait(h)


# ---------------------------------------------------------------- convenience wrapper
class LatentMoE:
    """A handle plus a workspace, driven with torch tensors.

    shape: an object with H, L, E, k, G, Gk, I, Is, s (e.g. synth.LayerShape).
    weights: dict of CUDA tensors router_w, e_bias, fc1_w, fc2_w, up_w, down_w,
    shared_up_w, shared_down_w (bf16, e_bias fp32). The tensors are borrowed.
    expert_format LMOE_EXPERTS_NVFP4: up_w / down_w are the E2M1 code arrays of
    quantize_nvfp4 and weights also holds up_sf, down_sf, up_gs, down_gs.
    """

    def __init__(self, shape, weights: dict, max_tokens: int, x_f32: bool = False, mode: int = LMOE_MODE_BF16,
                 expert_format: int = LMOE_EXPERTS_BF16, local_experts: int = 0, expert_base: int = 0):
        import torch
        self.torch = torch
        self.shape = shape
        self.weights = weights
        cfg = lmoe_config(shape.H, shape.L, shape.E, shape.k, shape.G, shape.Gk, shape.I, shape.Is, max_tokens,
                          float(shape.s), LMOE_FP32 if x_f32 else LMOE_BF16, mode, expert_format, local_experts,
                          expert_base)
        w = lmoe_weights(*[_p(weights.get(n)) for n in ("router_w", "e_bias", "fc1_w", "fc2_w", "up_w", "down_w",
                                                         "shared_up_w", "shared_down_w", "up_sf", "down_sf",
                                                         "up_gs", "down_gs")])
        s, h = latentmoe_create(cfg, w)
        if s != LMOE_OK:
            raise LmoeError(s, "latentmoe_create")
        self.h = h
        self.cfg = cfg
        self.x_f32 = x_f32
        self.mode = mode
        self._ws = None
        self._ws_T = -1
        self._ep_ws = None

    def workspace(self, T: int):
        s, n = latentmoe_workspace_size(self.h, T)
        if s != LMOE_OK:
            raise LmoeError(s, "latentmoe_workspace_size")
        if self._ws is None or self._ws.numel() < n:
            self._ws = self.torch.empty(max(n, 256), dtype=self.torch.uint8, device="cuda")
        return self._ws, n

    def set_option(self, opt: int, value: int):
        s = latentmoe_set_option(self.h, opt, value)
        if s != LMOE_OK:
            raise LmoeError(s, "latentmoe_set_option")

    def _stream(self):
        return ctypes.c_void_p(self.torch.cuda.current_stream().cuda_stream)

    def forward(self, x, y=None, idx=None, w=None, counts=None):
        torch = self.torch
        T = x.shape[0]
        if y is None:
            y = torch.empty((T, self.shape.H), dtype=torch.float32, device=x.device)
        ws, n = self.workspace(T)
        s = latentmoe_forward(self.h, _p(x), T, _p(y), _p(ws), ws.numel(), self._stream(), _p(idx), _p(w), _p(counts))
        if s != LMOE_OK:
            raise LmoeError(s, "latentmoe_forward")
        return y

    def forward_block(self, x, norm_w, norm_eps=1e-5, y=None, idx=None, w=None, counts=None):
        """y = x + layer(rmsnorm(x) * norm_w) (x bf16)."""
        torch = self.torch
        T = x.shape[0]
        if y is None:
            y = torch.empty((T, self.shape.H), dtype=torch.float32, device=x.device)
        ws, n = self.workspace(T)
        s = latentmoe_forward_block(self.h, _p(x), T, _p(norm_w), float(norm_eps), _p(y), _p(ws), ws.numel(),
                                    self._stream(), _p(idx), _p(w), _p(counts))
        if s != LMOE_OK:
            raise LmoeError(s, "latentmoe_forward_block")
        return y

    # ---- expert parallelism (the three stages around the all-to-all exchange)
    def ep_front(self, x, send_rows, send_w, counts):
        """Routing, fc1 + shared up, and the rows of z in expert order (send_rows
        [T*k, L] bf16, send_w [T*k] fp32, counts [E] int32). Keeps the workspace
        state that ep_back needs."""
        T = x.shape[0]
        ws, n = self.workspace(T)
        s = load().latentmoe_ep_front(self.h, _p(x), T, _p(send_rows), _p(send_w), _p(counts), _p(ws), ws.numel(),
                                      self._stream())
        if s != LMOE_OK:
            raise LmoeError(s, "latentmoe_ep_front")

    def ep_experts(self, recv_rows, recv_w, recv_counts, n_src, recv_o):
        """This handle's experts on received rows (source-major, expert order within a source)."""
        n_rows = recv_rows.shape[0]
        nbytes = ctypes.c_size_t()
        s = load().latentmoe_ep_workspace_size(self.h, n_rows, n_src, ctypes.byref(nbytes))
        if s != LMOE_OK:
            raise LmoeError(s, "latentmoe_ep_workspace_size")
        if self._ep_ws is None or self._ep_ws.numel() < nbytes.value:
            self._ep_ws = self.torch.empty(max(nbytes.value, 256), dtype=self.torch.uint8, device="cuda")
        s = load().latentmoe_ep_experts(self.h, _p(recv_rows), _p(recv_w), _p(recv_counts), n_src, n_rows,
                                        _p(recv_o), _p(self._ep_ws), self._ep_ws.numel(), self._stream())
        if s != LMOE_OK:
            raise LmoeError(s, "latentmoe_ep_experts")

    def ep_back(self, send_o, y):
        """Combine the returned rows (send order) and the output GEMM into y [T, H] fp32."""
        T = y.shape[0]
        ws, n = self.workspace(T)
        s = load().latentmoe_ep_back(self.h, _p(send_o), T, _p(y), _p(ws), ws.numel(), self._stream())
        if s != LMOE_OK:
            raise LmoeError(s, "latentmoe_ep_back")

    def route(self, x, idx=None, w=None, counts=None):
        torch = self.torch
        T = x.shape[0]
        k, E = self.shape.k, self.shape.E
        idx = torch.empty((T, k), dtype=torch.int32, device=x.device) if idx is None else idx
        w = torch.empty((T, k), dtype=torch.float32, device=x.device) if w is None else w
        counts = torch.empty((E,), dtype=torch.int32, device=x.device) if counts is None else counts
        ws, n = self.workspace(T)
        s = latentmoe_route(self.h, _p(x), T, _p(idx), _p(w), _p(counts), _p(ws), ws.numel(), self._stream())
        if s != LMOE_OK:
            raise LmoeError(s, "latentmoe_route")
        return idx, w, counts

    def update_bias(self, counts, eta: float, maxvio=None):
        """In-place load-balancing step on this layer's e_bias tensor."""
        b = self.weights["e_bias"]
        s = latentmoe_update_bias(self.h, _p(counts), _p(b), float(eta), _p(b), _p(maxvio), self._stream())
        if s != LMOE_OK:
            raise LmoeError(s, "latentmoe_update_bias")

    def layout(self, T: int):
        s, out = latentmoe_workspace_layout(self.h, T)
        if s != LMOE_OK:
            raise LmoeError(s, "latentmoe_workspace_layout")
        return out

    def ws_view(self, offset: int, shape, dtype):
        """A tensor view of the workspace at a byte offset (diagnostics)."""
        n = 1
        for d in shape:
            n *= d
        nbytes = n * self.torch.empty((), dtype=dtype).element_size()
        return self._ws[offset:offset + nbytes].view(dtype).view(*shape)

    def stats(self):
        s, st = latentmoe_read_stats(self.h, _p(self._ws))
        if s != LMOE_OK:
            raise LmoeError(s, "latentmoe_read_stats")
        return st

    def close(self):
        if getattr(self, "h", None):
            latentmoe_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
