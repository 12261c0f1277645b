"""Shared helpers of the GPU parity tests (tests only)."""
from __future__ import annotations

import numpy as np

import oracle
import synth

BF16_MAXABS = 2e-2      # stated bound (bf16 operands, fp32 accumulation), every GEMM path and width
BF16_RELFRO = 1e-2
FP32_RELFRO = 1e-5      # stated bound of the fp32 validation mode


def bf16_to_bits(t) -> np.ndarray:
    import torch
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def device_layer(shape, mode=0, max_tokens=None, seed=0):
    """Generate every input in HBM and build a LatentMoE handle around them."""
    import latentmoe_layer_b200 as lm
    dev = synth.device_inputs(shape, seed)
    layer = lm.LatentMoE(shape, dev, max_tokens or shape.T, x_f32=shape.x_f32, mode=mode)
    return layer, dev


def check_device_inputs_match_generator(shape, dev, seed=0, samples=512):
    """The device copy of every input equals the host generator's values (sampled)."""
    import torch
    rng = np.random.default_rng(1234)
    for key, _, shp, _ in synth.tensor_specs(shape):
        t = dev[key]
        n = int(np.prod(shp))
        flat = rng.integers(0, n, size=min(samples, n))
        got = t.reshape(-1)[torch.from_numpy(flat).to(t.device)].cpu()
        if t.dtype == torch.bfloat16:
            got_bits = got.view(torch.int16).numpy().view(np.uint16)
            ref = [synth.element(shape, key, int(i), seed) for i in flat]
            assert np.array_equal(got_bits, np.array(ref, dtype=np.uint16)), key
        else:
            ref = [synth.element(shape, key, int(i), seed) for i in flat]
            assert np.array_equal(got.numpy(), np.array(ref, dtype=np.float32)), key


def host_weights_for(shape, dev, experts):
    """Host copies of the dense weights and of the listed experts' weights,
    copied from the device generator's output (checked against the host
    generator by check_device_inputs_match_generator)."""
    out = {}
    for key in ("router_w", "fc1_w", "fc2_w", "shared_up_w", "shared_down_w"):
        out[key] = bf16_to_bits(dev[key])
    out["e_bias"] = dev["e_bias"].cpu().numpy()
    up = [None] * shape.E
    down = [None] * shape.E
    for e in experts:
        up[int(e)] = bf16_to_bits(dev["up_w"][int(e)])
        down[int(e)] = bf16_to_bits(dev["down_w"][int(e)])
    out["up_w"], out["down_w"] = up, down
    return out


def host_x(shape, dev, rows):
    import torch
    x = dev["x"][torch.as_tensor(rows, device=dev["x"].device)]
    if shape.x_f32:
        return x.cpu().numpy()
    return bf16_to_bits(x)


def errors(y, ref):
    y = np.asarray(y, dtype=np.float64)
    d = y - ref
    return float(np.abs(d).max()), float(np.linalg.norm(d) / max(np.linalg.norm(ref), 1e-300))


def assert_bf16_close(y, ref):
    ma, rf = errors(y, ref)
    assert ma <= BF16_MAXABS and rf <= BF16_RELFRO, (ma, rf)
    return ma, rf


def flagged_tokens(layer, T):
    """Ids of the tokens whose routing the last call on the layer's workspace
    re-decided in fp64 (the flag list the routing kernel writes)."""
    import torch
    n = layer.stats().flagged_tokens
    if n == 0:
        return np.zeros(0, dtype=np.int64)
    lay = layer.layout(T)
    return np.sort(layer.ws_view(lay.flag_list, (n,), torch.int32).cpu().numpy().astype(np.int64))


def assert_fp32_close(y, ref):
    ma, rf = errors(y, ref)
    assert rf <= FP32_RELFRO, (ma, rf)
    return ma, rf


def oracle_forward(shape, x_rows, wts, fp32_mode=False):
    cfg = oracle.make_cfg(shape, fp32_mode=fp32_mode)
    return oracle.forward(cfg, x_rows, wts)


def oracle_route(shape, x_rows, wts):
    cfg = oracle.make_cfg(shape)
    return oracle.route(cfg, x_rows, wts["router_w"], wts["e_bias"])
