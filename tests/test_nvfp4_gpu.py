"""GPU parity of the NVFP4 expert path against the fp64 oracle, through the C ABI.

The library's quantiser must give the oracle's codes, block scales and matrix
scales byte for byte. The layer with NVFP4 experts is compared with the oracle
run on the oracle's own quantisation of the same bf16 weights (dequantised
code * scale values plus per-expert matrix scales): routing bit-exact, y within
the bf16-mode tolerances (the dequantised weights are exact in bf16, so the
arithmetic is that of the bf16 path).
"""
from dataclasses import replace

import numpy as np
import pytest

import synth
from synth import LayerShape, NANO_DECODE, ULTRA_DECODE, ULTRA_PREFILL
import helpers as H
import oracle

pytestmark = pytest.mark.gpu

GEMM_AUTO, GEMM_PREFILL, GEMM_DECODE, GEMM_SIMT, GEMM_PREFILL_PAIR = range(5)

# several weight tiles (I = 3 x 128, L = 2 x 128) and ragged token tiles
RAGGED4 = LayerShape("ragged_nvfp4", T=333, H=512, L=256, E=64, k=6, G=4, Gk=2, I=384, Is=640)


def to_bits(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16).view(torch.int16) \
        .numpy().view(np.uint16)


def device_quantise(dev):
    import latentmoe_layer_b200 as lm
    uc, us, ug = lm.quantize_nvfp4(dev["up_w"])
    dc, ds, dg = lm.quantize_nvfp4(dev["down_w"])
    return dict(up_w=uc, up_sf=us, up_gs=ug, down_w=dc, down_sf=ds, down_gs=dg)


def nvfp4_layer(shape, path=GEMM_AUTO, max_tokens=None):
    import latentmoe_layer_b200 as lm
    dev = synth.device_inputs(shape, 0)
    q = device_quantise(dev)
    layer = lm.LatentMoE(shape, dict(dev, **q), max_tokens or shape.T, x_f32=shape.x_f32,
                         expert_format=lm.LMOE_EXPERTS_NVFP4)
    if path != GEMM_AUTO:
        layer.set_option(0, path)
    return layer, dev, q


def oracle_experts(shape, src, q, experts, wts):
    """Quantise the listed experts' bf16 weights (src: host arrays [E, ...] from the
    generator, or the device tensors it filled) on the host with the oracle, check
    the device quantiser's bytes for them, and put the oracle's dequantised experts
    and matrix scales in wts."""
    E, I, L = shape.E, shape.I, shape.L
    experts = [int(e) for e in experts]

    def bits(a, e):
        return np.ascontiguousarray(a[e]) if isinstance(a, np.ndarray) else H.bf16_to_bits(a[e])

    up = np.stack([bits(src["up_w"], e) for e in experts])
    dn = np.stack([bits(src["down_w"], e) for e in experts])
    uc, us, ug = oracle.nvfp4_quantize(up)
    dc, ds, dg = oracle.nvfp4_quantize(dn)
    gq = {k: v.cpu().numpy() for k, v in q.items()}
    nc, ns = I * L // 2, I * L // 16
    for j, e in enumerate(experts):
        assert np.array_equal(gq["up_w"][e * nc:(e + 1) * nc], uc[j * nc:(j + 1) * nc]), e
        assert np.array_equal(gq["up_sf"][e * ns:(e + 1) * ns], us[j * ns:(j + 1) * ns]), e
        assert np.array_equal(gq["down_w"][e * nc:(e + 1) * nc], dc[j * nc:(j + 1) * nc]), e
        assert np.array_equal(gq["down_sf"][e * ns:(e + 1) * ns], ds[j * ns:(j + 1) * ns]), e
        assert gq["up_gs"][e] == ug[j] and gq["down_gs"][e] == dg[j], e
    up_d = oracle.nvfp4_dequant(uc, us, len(experts), I, L)
    dn_d = oracle.nvfp4_dequant(dc, ds, len(experts), L, I)
    wts["up_w"], wts["down_w"] = [None] * E, [None] * E
    wts["up_gs"], wts["down_gs"] = np.ones(E, np.float32), np.ones(E, np.float32)
    for j, e in enumerate(experts):
        wts["up_w"][e], wts["down_w"][e] = up_d[j], dn_d[j]
        wts["up_gs"][e], wts["down_gs"][e] = ug[j], dg[j]
    return wts


def test_quantiser_bytes_match_oracle():
    import torch
    import latentmoe_layer_b200 as lm
    rng = np.random.default_rng(21)
    n_mat, R, K = 4, 256, 192
    w = rng.normal(0, 0.02, (n_mat, R, K)).astype(np.float32)
    # matrix 1: magnitudes over 2^-24 .. 2^4 per row (subnormal and saturating block scales)
    w[1] *= np.exp2(rng.uniform(-24, 4, (R, 1))).astype(np.float32)
    # matrix 2: zero, except the hand-worked example row (ties, saturation, zero and subnormal blocks)
    w[2] = 0
    ex = {0: 1.3125, 1: -1.3125, 2: 0.875, 3: 0.65625, 4: 0.4375, 5: 0.328125, 6: 0.21875, 7: 0.109375, 9: 1.09375,
          10: 0.546875, 11: 0.0546875, 12: 0.1640625, 13: -0.65625, 14: -0.109375, 15: 0.2734375, 16: 0.109375,
          17: -0.0546875, 18: 0.02734375, 19: 0.0703125, 20: 0.080078125, 48: 2.0 ** -14, 49: -2.0 ** -15}
    for k, v in ex.items():
        w[2, 5, k] = v
    # matrix 3: values on exact E2M1 midpoints of a power-of-two grid, both signs
    w[3] = rng.choice([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0], (R, K)) * rng.choice([-1, 1], (R, K))
    bits = to_bits(w).reshape(n_mat, R, K)
    wd = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()
    codes, sf, gs = lm.quantize_nvfp4(wd)
    torch.cuda.synchronize()
    oc, osf, og = oracle.nvfp4_quantize(bits)
    assert np.array_equal(gs.cpu().numpy(), og)
    assert np.array_equal(sf.cpu().numpy(), osf)
    assert np.array_equal(codes.cpu().numpy(), oc)
    # a zero matrix set: g = 1, all codes 0
    z = torch.zeros((1, 128, 64), dtype=torch.bfloat16, device="cuda")
    c0, s0, g0 = lm.quantize_nvfp4(z)
    assert float(g0[0]) == 1.0 and not c0.any() and not s0.any()


def run_nvfp4(shape, path=GEMM_AUTO):
    import torch
    layer, dev, q = nvfp4_layer(shape, path)
    T = shape.T
    idx = torch.empty((T, shape.k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, shape.k), dtype=torch.float32, device="cuda")
    counts = torch.empty((shape.E,), dtype=torch.int32, device="cuda")
    y = layer.forward(dev["x"], idx=idx, w=w, counts=counts)
    y2 = layer.forward(dev["x"])
    torch.cuda.synchronize()
    assert layer.stats().device_error == 0
    assert torch.equal(y, y2), "two runs differ"
    host = synth.host_inputs(shape)
    wts = oracle_experts(shape, host, q, range(shape.E), dict(host))
    yref, iref, wref = H.oracle_forward(shape, host["x"], wts)
    assert np.array_equal(idx.cpu().numpy(), iref)
    assert np.array_equal(counts.cpu().numpy(), np.bincount(iref.ravel(), minlength=shape.E))
    np.testing.assert_allclose(w.cpu().numpy(), wref, rtol=2e-6, atol=1e-6)
    ma, rf = H.assert_bf16_close(y.cpu().numpy(), yref)
    print("%s path=%d max_abs=%.3g rel_fro=%.3g" % (shape.name, path, ma, rf))
    return layer, dev, q, y


@pytest.mark.parametrize("path", [GEMM_AUTO, GEMM_PREFILL, GEMM_DECODE])
def test_nvfp4_ragged(path):
    run_nvfp4(RAGGED4, path)


def test_nvfp4_ragged_small_batches():
    # one token, and a batch whose experts see at most a few tokens each
    for T in (1, 7):
        run_nvfp4(replace(RAGGED4, name="ragged_nvfp4_T%d" % T, T=T), GEMM_AUTO)


def test_nvfp4_differs_from_bf16_by_the_quantisation_only():
    # the NVFP4 layer is not the bf16 layer: its error against the bf16 oracle is the
    # weight quantisation's, far above the bf16 tolerance but a small relative error
    import torch
    layer, dev, q, y = run_nvfp4(RAGGED4, GEMM_AUTO)
    host = synth.host_inputs(RAGGED4)
    yb, _, _ = H.oracle_forward(RAGGED4, host["x"], host)
    ma, rf = H.errors(y.cpu().numpy(), yb)
    print("nvfp4 vs bf16 weights: max_abs=%.3g rel_fro=%.3g" % (ma, rf))
    assert 1e-3 < rf < 0.3


def test_nvfp4_nano_full():
    run_nvfp4(NANO_DECODE, GEMM_AUTO)


def _nvfp4_sampled(shape, rows, path=GEMM_AUTO):
    import torch
    layer, dev, q = nvfp4_layer(shape, path)
    H.check_device_inputs_match_generator(shape, dev)
    T = shape.T
    idx = torch.empty((T, shape.k), dtype=torch.int32, device="cuda")
    counts = torch.empty((shape.E,), dtype=torch.int32, device="cuda")
    y = layer.forward(dev["x"], idx=idx, counts=counts)
    torch.cuda.synchronize()
    assert layer.stats().device_error == 0
    gi = idx.cpu().numpy()
    experts = np.unique(gi[rows])
    wts = oracle_experts(shape, dev, q, experts, H.host_weights_for(shape, dev, []))
    yref, iref, _ = H.oracle_forward(shape, H.host_x(shape, dev, rows), wts)
    assert np.array_equal(iref, gi[rows])
    ma, rf = H.assert_bf16_close(y.cpu().numpy()[rows], yref)
    print("%s nvfp4 max_abs=%.3g rel_fro=%.3g experts checked=%d" % (shape.name, ma, rf, len(experts)))


def test_nvfp4_ultra_decode_sampled():
    rng = np.random.default_rng(22)
    _nvfp4_sampled(ULTRA_DECODE, np.sort(rng.choice(64, 3, replace=False)))


def test_nvfp4_ultra_prefill_sampled():
    rng = np.random.default_rng(23)
    T = ULTRA_PREFILL.T
    _nvfp4_sampled(ULTRA_PREFILL, np.sort(np.concatenate([[T - 1], rng.choice(T - 1, 2, replace=False)])))


def test_nvfp4_inside_the_pre_norm_residual_block():
    # the block (y = x + layer(rmsnorm(x))) with NVFP4 experts
    import torch
    shape = RAGGED4
    layer, dev, q = nvfp4_layer(shape)
    rng = np.random.default_rng(31)
    g = torch.from_numpy(rng.uniform(0.5, 1.5, shape.H).astype(np.float32)).to(torch.bfloat16).cuda()
    idx = torch.empty((shape.T, shape.k), dtype=torch.int32, device="cuda")
    y = layer.forward_block(dev["x"], g, 1e-5, idx=idx)
    torch.cuda.synchronize()
    host = synth.host_inputs(shape)
    wts = oracle_experts(shape, host, q, range(shape.E), dict(host))
    yref, iref, _ = oracle.forward_block(oracle.make_cfg(shape), host["x"], H.bf16_to_bits(g), 1e-5, wts)
    assert np.array_equal(idx.cpu().numpy(), iref)
    ma, rf = H.assert_bf16_close(y.cpu().numpy(), yref)
    print("nvfp4 block max_abs=%.3g rel_fro=%.3g" % (ma, rf))


def test_nvfp4_ultra_skew_sampled():
    # hot experts with thousands of tokens each run the 128-token NVFP4 tiles
    from synth import ULTRA_SKEW
    rng = np.random.default_rng(24)
    _nvfp4_sampled(ULTRA_SKEW, np.sort(rng.choice(ULTRA_SKEW.T, 3, replace=False)))
