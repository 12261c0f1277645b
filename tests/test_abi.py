"""The C ABI: exported symbols, argument validation and error paths."""
import ctypes
import os
import re
import subprocess

import pytest

import latentmoe_layer_b200 as lm
import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    syms = set()
    inc = os.path.join(ROOT, "include")
    for f in os.listdir(inc):
        if f.endswith(".h"):
            txt = open(os.path.join(inc, f)).read()
            syms |= set(re.findall(r"\b(latentmoe_\w+)\s*\(", txt))
    return syms


@pytest.fixture(scope="module")
def lib():
    from latentmoe_layer_b200 import build
    build.build()
    return lm.load()


def test_library_exports_every_declared_symbol(lib):
    syms = declared_symbols()
    assert len(syms) >= 9
    out = subprocess.run(["nm", "-D", "--defined-only", lm.LIB_PATH], stdout=subprocess.PIPE, text=True).stdout
    exported = set(re.findall(r"\bT (latentmoe_\w+)", out))
    assert syms <= exported, syms - exported
    for s in syms:
        assert hasattr(lib, s)
    assert set(lm.EXPORTS) <= syms


def good_cfg(**kw):
    w = synth.TINY
    c = dict(hidden=w.H, latent=w.L, num_experts=w.E, top_k=w.k, n_group=w.G, topk_group=w.Gk,
             expert_inter=w.I, shared_inter=w.Is, max_tokens=64, routed_scaling_factor=5.0, x_dtype=1, mode=0)
    c.update(kw)
    return lm.lmoe_config(**c)


def fake_weights(addr=0x10000, nvfp4_addr=None):
    extra = addr if nvfp4_addr is None else nvfp4_addr
    return lm.lmoe_weights(*([addr] * 8 + [extra] * 4))


@pytest.mark.parametrize("kw,status", [
    (dict(hidden=100), lm.LMOE_ERR_INVALID_ARG),          # not a multiple of 64
    (dict(latent=0), lm.LMOE_ERR_INVALID_ARG),
    (dict(top_k=0), lm.LMOE_ERR_INVALID_ARG),
    (dict(top_k=17), lm.LMOE_ERR_INVALID_ARG),            # k > E
    (dict(n_group=3), lm.LMOE_ERR_INVALID_ARG),           # E % G != 0
    (dict(n_group=4, topk_group=5), lm.LMOE_ERR_INVALID_ARG),
    (dict(n_group=4, topk_group=1, top_k=5), lm.LMOE_ERR_INVALID_ARG),  # k > kept experts
    (dict(max_tokens=0), lm.LMOE_ERR_INVALID_ARG),
    (dict(mode=7), lm.LMOE_ERR_INVALID_ARG),
    (dict(x_dtype=3), lm.LMOE_ERR_INVALID_ARG),
    (dict(routed_scaling_factor=float("nan")), lm.LMOE_ERR_INVALID_ARG),
    (dict(num_experts=2048, top_k=2), lm.LMOE_ERR_UNSUPPORTED),
    (dict(num_experts=64, n_group=64, topk_group=1, top_k=1), lm.LMOE_ERR_UNSUPPORTED),
    (dict(num_experts=16, top_k=65), lm.LMOE_ERR_INVALID_ARG),
])
def test_invalid_configs_rejected_before_any_cuda_call(lib, kw, status):
    s, h = lm.latentmoe_create(good_cfg(**kw), fake_weights())
    assert s == status and not h.value


@pytest.mark.parametrize("kw,status", [
    (dict(expert_format=7), lm.LMOE_ERR_INVALID_ARG),
    (dict(expert_format=lm.LMOE_EXPERTS_NVFP4, latent=128, mode=lm.LMOE_MODE_FP32), lm.LMOE_ERR_UNSUPPORTED),
    (dict(expert_format=lm.LMOE_EXPERTS_NVFP4), lm.LMOE_ERR_UNSUPPORTED),                # L = 64: not 128 rows
    (dict(expert_format=lm.LMOE_EXPERTS_NVFP4, latent=128, expert_inter=192), lm.LMOE_ERR_UNSUPPORTED),
])
def test_nvfp4_configs_rejected_before_any_cuda_call(lib, kw, status):
    s, h = lm.latentmoe_create(good_cfg(**kw), fake_weights())
    assert s == status and not h.value


@pytest.mark.parametrize("kw,status", [
    (dict(local_experts=-1), lm.LMOE_ERR_INVALID_ARG),
    (dict(local_experts=17), lm.LMOE_ERR_INVALID_ARG),             # more than E
    (dict(local_experts=8, expert_base=9), lm.LMOE_ERR_INVALID_ARG),  # block past E
    (dict(expert_base=-8), lm.LMOE_ERR_INVALID_ARG),
])
def test_expert_shard_configs_rejected_before_any_cuda_call(lib, kw, status):
    s, h = lm.latentmoe_create(good_cfg(**kw), fake_weights())
    assert s == status and not h.value


def test_expert_parallel_entry_points_reject_null_handles(lib):
    n = ctypes.c_size_t()
    assert lib.latentmoe_ep_workspace_size(None, 4, 1, ctypes.byref(n)) == lm.LMOE_ERR_INVALID_ARG
    assert lib.latentmoe_ep_front(None, None, 1, None, None, None, None, 0, None) == lm.LMOE_ERR_INVALID_ARG
    assert lib.latentmoe_ep_experts(None, None, None, None, 1, 1, None, None, 0, None) == lm.LMOE_ERR_INVALID_ARG
    assert lib.latentmoe_ep_back(None, None, 1, None, None, 0, None) == lm.LMOE_ERR_INVALID_ARG


def test_nvfp4_weights_need_scales(lib):
    cfg = good_cfg(expert_format=lm.LMOE_EXPERTS_NVFP4, latent=128)
    for bad in (0, 0x10008):
        s, h = lm.latentmoe_create(cfg, fake_weights(nvfp4_addr=bad))
        assert s == lm.LMOE_ERR_INVALID_ARG and not h.value


def test_quantize_nvfp4_argument_checks(lib):
    q, st = lm.latentmoe_quantize_nvfp4, None
    assert q(0x10000, 0, 128, 64, 0x10000, 0x10000, 0x10000, st) == lm.LMOE_OK          # nothing to do
    assert q(None, 1, 128, 64, 0x10000, 0x10000, 0x10000, st) == lm.LMOE_ERR_INVALID_ARG
    assert q(0x10008, 1, 128, 64, 0x10000, 0x10000, 0x10000, st) == lm.LMOE_ERR_INVALID_ARG
    assert q(0x10000, 1, 128, 64, 0x10000, 0x10000, 0x10002, st) == lm.LMOE_ERR_INVALID_ARG
    assert q(0x10000, -1, 128, 64, 0x10000, 0x10000, 0x10000, st) == lm.LMOE_ERR_INVALID_ARG
    assert q(0x10000, 1, 64, 64, 0x10000, 0x10000, 0x10000, st) == lm.LMOE_ERR_UNSUPPORTED
    assert q(0x10000, 1, 128, 96, 0x10000, 0x10000, 0x10000, st) == lm.LMOE_ERR_UNSUPPORTED


def test_null_or_misaligned_weights_rejected(lib):
    s, h = lm.latentmoe_create(good_cfg(), fake_weights(0))
    assert s == lm.LMOE_ERR_INVALID_ARG and not h.value
    s, h = lm.latentmoe_create(good_cfg(), fake_weights(0x10008))
    assert s == lm.LMOE_ERR_INVALID_ARG and not h.value


def test_null_handle_paths(lib):
    assert lib.latentmoe_create(None, None, None) == lm.LMOE_ERR_INVALID_ARG
    assert lm.latentmoe_workspace_size(None, 4)[0] == lm.LMOE_ERR_INVALID_ARG
    assert lm.latentmoe_forward(None, None, 1, None, None, 0, None) == lm.LMOE_ERR_INVALID_ARG
    assert lm.latentmoe_route(None, None, 1, None, None, None, None, 0, None) == lm.LMOE_ERR_INVALID_ARG
    assert lm.latentmoe_set_option(None, 0, 0) == lm.LMOE_ERR_INVALID_ARG
    lm.latentmoe_destroy(None)


def test_status_strings(lib):
    for s in range(7):
        assert lm.status_string(s) and lm.status_string(s) != "unknown status"
    assert lm.status_string(99) == "unknown status"


# ---------------------------------------------------------------- GPU error paths
@pytest.mark.gpu
def test_call_errors_leave_outputs_untouched(lib):
    import torch
    import helpers as H
    shape = synth.TINY
    layer, dev = H.device_layer(shape, max_tokens=64)
    T = shape.T
    y = torch.full((T, shape.H), 7.0, device="cuda")
    ws, n = layer.workspace(T)
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    f = lm.latentmoe_forward
    assert f(layer.h, None, T, y.data_ptr(), ws.data_ptr(), n, st) == lm.LMOE_ERR_INVALID_ARG
    assert f(layer.h, dev["x"].data_ptr(), 65, y.data_ptr(), ws.data_ptr(), n, st) == lm.LMOE_ERR_INVALID_ARG
    assert f(layer.h, dev["x"].data_ptr(), -1, y.data_ptr(), ws.data_ptr(), n, st) == lm.LMOE_ERR_INVALID_ARG
    assert f(layer.h, dev["x"].data_ptr(), T, y.data_ptr(), ws.data_ptr(), n - 1, st) == lm.LMOE_ERR_WORKSPACE
    assert f(layer.h, dev["x"].data_ptr(), T, y.data_ptr(), ws.data_ptr() + 16, n, st) == lm.LMOE_ERR_WORKSPACE
    assert f(layer.h, dev["x"].data_ptr(), T, y.data_ptr() + 4, ws.data_ptr(), n, st) == lm.LMOE_ERR_INVALID_ARG
    assert f(layer.h, dev["x"].data_ptr() + 8, T, y.data_ptr(), ws.data_ptr(), n, st) == lm.LMOE_ERR_INVALID_ARG
    assert f(layer.h, dev["x"].data_ptr(), 0, y.data_ptr(), 0, 0, st) == lm.LMOE_OK
    torch.cuda.synchronize()
    assert bool((y == 7.0).all())
    assert lm.latentmoe_set_option(layer.h, 0, 9) == lm.LMOE_ERR_INVALID_ARG
    assert lm.latentmoe_set_option(layer.h, 3, 0) == lm.LMOE_ERR_INVALID_ARG
    assert lm.latentmoe_set_option(layer.h, lm.OPT_Z_RECHECK_DELTA, -1) == lm.LMOE_ERR_INVALID_ARG
    assert lm.latentmoe_set_option(layer.h, lm.OPT_Z_RECHECK_DELTA, 100000001) == lm.LMOE_ERR_INVALID_ARG
    assert lm.latentmoe_set_option(layer.h, lm.OPT_Z_RECHECK_DELTA, 0) == lm.LMOE_OK
    assert lm.latentmoe_set_option(layer.h, lm.OPT_ACT_RECHECK_TAU, -1) == lm.LMOE_ERR_INVALID_ARG
    # below tau = 0.5 the re-rounding list could not hold every activation the flag test lists
    assert lm.latentmoe_set_option(layer.h, lm.OPT_ACT_RECHECK_TAU, 499) == lm.LMOE_ERR_INVALID_ARG
    assert lm.latentmoe_set_option(layer.h, lm.OPT_ACT_RECHECK_TAU, 500) == lm.LMOE_OK
    assert lm.latentmoe_set_option(layer.h, lm.OPT_ACT_RECHECK_TAU, 0) == lm.LMOE_OK
    assert lm.latentmoe_set_option(layer.h, 6, 0) == lm.LMOE_ERR_INVALID_ARG


@pytest.mark.gpu
def test_bounded_wait_times_out_and_context_survives(lib):
    import torch
    import helpers as H
    layer, dev = H.device_layer(synth.TINY)
    layer.set_option(lm.OPT_SPIN_LIMIT, 20000)
    assert lm.latentmoe_selftest_bounded_wait(layer.h) == lm.LMOE_ERR_TIMEOUT
    layer.set_option(lm.OPT_SPIN_LIMIT, 1 << 24)
    y = layer.forward(dev["x"])
    torch.cuda.synchronize()
    assert torch.isfinite(y).all()
    assert layer.stats().device_error == 0



@pytest.mark.gpu
def test_profile_events_must_exist(lib):
    # a NULL event (e.g. a framework event never recorded, hence not created yet) is refused;
    # created events are accepted and a forward with them succeeds
    import torch
    import helpers as H
    layer, dev = H.device_layer(synth.TINY, max_tokens=64)
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(8)]
    unrecorded = (ctypes.c_void_p * 8)(*[e.cuda_event for e in evs])
    assert lm.latentmoe_set_profile_events(layer.h, ctypes.cast(unrecorded, ctypes.c_void_p), 8) == \
        lm.LMOE_ERR_INVALID_ARG
    for e in evs:
        e.record()
    torch.cuda.synchronize()
    created = (ctypes.c_void_p * 8)(*[e.cuda_event for e in evs])
    assert lm.latentmoe_set_profile_events(layer.h, ctypes.cast(created, ctypes.c_void_p), 8) == lm.LMOE_OK
    layer.forward(dev["x"])
    torch.cuda.synchronize()
    assert evs[0].elapsed_time(evs[7]) > 0
    assert lm.latentmoe_set_profile_events(layer.h, None, 0) == lm.LMOE_OK
    layer.close()


def test_binding_matches_header_stats_and_options():
    """The ctypes view of lmoe_stats and the option ids equal the header's."""
    import re
    hdr = open(os.path.join(ROOT, "include", "latentmoe.h")).read()
    body = re.search(r"typedef struct \{([^}]*)\} lmoe_stats;", hdr).group(1)
    body = re.sub(r"/\*.*?\*/", "", body, flags=re.S)
    fields = re.findall(r"int\s+(\w+)\s*;", body)
    assert fields == [f for f, _ in lm.lmoe_stats._fields_]
    opts = dict((k, int(v)) for k, v in re.findall(r"LMOE_OPT_(\w+)\s*=\s*(\d+)", hdr))
    assert opts == {"GEMM_PATH": lm.OPT_GEMM_PATH, "ROUTER_FP64_ALL": lm.OPT_ROUTER_FP64_ALL,
                    "FLAG_DELTA": lm.OPT_FLAG_DELTA, "SPIN_LIMIT": lm.OPT_SPIN_LIMIT,
                    "Z_RECHECK_DELTA": lm.OPT_Z_RECHECK_DELTA, "ACT_RECHECK_TAU": lm.OPT_ACT_RECHECK_TAU}
