"""Pins of the fp64 oracle against what the pages and the mathematics fix.

None of these tests retypes the oracle's loops: each checks the oracle against
a property, a special case that reduces to a library routine (numpy matmul),
brute force on tiny inputs, a closed form, or a figure printed on the pages.
"""
import itertools
import os
from dataclasses import replace

import numpy as np
import pytest
import torch

import synth
from synth import TINY, LayerShape
from latentmoe_layer_b200 import accounting

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def f32_to_bf16_bits(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16).view(torch.int16) \
        .numpy().view(np.uint16)


def bits_to_f64(a):
    return synth.bf16_bits_to_f32(np.asarray(a, dtype=np.uint16)).astype(np.float64)


def small_shape(**kw):
    base = dict(name="pin", T=12, H=48, L=16, E=8, k=2, G=1, Gk=1, I=24, Is=32, s=5.0, x_f32=True)
    base.update(kw)
    return LayerShape(**base)


def inputs(w, seed=3):
    return synth.host_inputs(w, seed)


def dense_reference(w, x, wts, fp32_mode):
    """The k = E, G = 1 special case written as plain numpy matmuls: every expert is
    selected, so the layer is the dense, bias-free mixture
    y = fc2(rho(sum_e s sigma_e / sum sigma * Expert_e(z))) + Shared(x)."""
    def rho(v):
        if fp32_mode:
            return v
        # bf16 rounding through torch (fp64 -> fp32 -> bf16); a double rounding
        # can differ from the oracle's direct rounding in rare last-bit cases.
        return torch.from_numpy(v).to(torch.float32).to(torch.bfloat16).to(torch.float64).numpy()

    xf = x.astype(np.float64) if w.x_f32 else bits_to_f64(x)
    Wr, W1, W2 = bits_to_f64(wts["router_w"]), bits_to_f64(wts["fc1_w"]), bits_to_f64(wts["fc2_w"])
    Wu, Wd = bits_to_f64(wts["up_w"]), bits_to_f64(wts["down_w"])
    Wsu, Wsd = bits_to_f64(wts["shared_up_w"]), bits_to_f64(wts["shared_down_w"])
    sig = 1.0 / (1.0 + np.exp(-(xf @ Wr.T)))
    wgt = w.s * sig / sig.sum(axis=1, keepdims=True)
    xh = rho(xf)
    z = rho(xh @ W1.T)
    acc = np.zeros((x.shape[0], w.L))
    for e in range(w.E):
        a = rho(np.maximum(z @ Wu[e].T, 0.0) ** 2)
        acc += wgt[:, e:e + 1] * (a @ Wd[e].T)
    comb = rho(acc)
    a_s = rho(np.maximum(xh @ Wsu.T, 0.0) ** 2)
    return comb @ W2.T + a_s @ Wsd.T


# ------------------------------------------------------------------ rounding
def test_round_bf16_matches_torch_on_fp32_values(built_oracle):
    rng = np.random.default_rng(0)
    vals = np.concatenate([rng.standard_normal(2000).astype(np.float32) * 10.0 ** rng.integers(-30, 30, 2000),
                           np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -(1.0 + 2 ** -8), 2 ** -130, 3.0e-39,
                                     65504.0, 1.0 - 2 ** -9], dtype=np.float32)]).astype(np.float32)
    ref = bits_to_f64(f32_to_bf16_bits(vals))
    got = np.array([built_oracle.round_bf16(float(v)) for v in vals])
    assert np.array_equal(got, ref)


def test_round_bf16_ties_to_even(built_oracle):
    # 1 + 2^-8 is halfway between 1 and 1 + 2^-7: the even neighbour is 1.
    assert built_oracle.round_bf16(1.0 + 2 ** -8) == 1.0
    assert built_oracle.round_bf16(1.0 + 3 * 2 ** -8) == 1.0 + 2 ** -6
    assert built_oracle.round_bf16(1.0 + 2 ** -8 + 2 ** -40) == 1.0 + 2 ** -7


# ------------------------------------------------------------------ selection
def brute_force_select(c, E, k, G, Gk):
    per = E // G
    gscore = [sum(sorted(c[g * per:(g + 1) * per])[-2:]) if G > 1 else 0.0 for g in range(G)]
    best_groups = max(itertools.combinations(range(G), Gk), key=lambda gs: sum(gscore[g] for g in gs))
    elig = [e for g in best_groups for e in range(g * per, (g + 1) * per)]
    best = max(itertools.combinations(elig, k), key=lambda s: sum(c[e] for e in s))
    return sorted(best)


@pytest.mark.parametrize("G,Gk", [(1, 1), (2, 1), (2, 2), (4, 1), (4, 2), (4, 3)])
@pytest.mark.parametrize("k", [1, 2, 3])
def test_select_equals_brute_force(built_oracle, G, Gk, k):
    E = 16
    if k > Gk * (E // G):
        pytest.skip("k larger than the kept experts")
    cfg = built_oracle.make_cfg(small_shape(E=E, k=k, G=G, Gk=Gk))
    rng = np.random.default_rng(100 * G + 10 * Gk + k)
    for _ in range(40):
        c = rng.random(E)
        assert list(built_oracle.select(cfg, c)) == brute_force_select(list(c), E, k, G, Gk)


def test_select_exact_tie_prefers_lower_id(built_oracle):
    cfg = built_oracle.make_cfg(small_shape(E=8, k=2))
    c = np.array([0.1, 0.9, 0.5, 0.2, 0.5, 0.3, 0.5, 0.0])
    assert list(built_oracle.select(cfg, c)) == [1, 2]


def test_select_near_tie_band(built_oracle):
    cfg = built_oracle.make_cfg(small_shape(E=8, k=2))
    # expert 6 is larger than expert 2 by less than 1e-6: both are in the band,
    # one slot is left, the lower id wins.
    c = np.array([0.1, 0.9, 0.5, 0.2, 0.1, 0.3, 0.5 + 5e-7, 0.0])
    assert list(built_oracle.select(cfg, c)) == [1, 2]
    # by more than 1e-6 the larger one wins.
    c[6] = 0.5 + 2e-6
    assert list(built_oracle.select(cfg, c)) == [1, 6]


def test_select_band_reaches_above_tau(built_oracle):
    # tau (3rd largest) = 0.5 + 3e-7; expert 6 lies above tau but within 1e-6 of it,
    # so it competes in the band with 2 and 4, and the two lowest ids win.
    cfg = built_oracle.make_cfg(small_shape(E=8, k=3))
    c = np.array([0.1, 0.9, 0.5, 0.2, 0.5 + 3e-7, 0.3, 0.5 + 5e-7, 0.0])
    assert list(built_oracle.select(cfg, c)) == [1, 2, 4]


def test_group_near_tie_prefers_lower_group(built_oracle):
    cfg = built_oracle.make_cfg(small_shape(E=8, k=2, G=4, Gk=1))
    c = np.zeros(8)
    c[2:4] = [0.5, 0.5]            # group 1 score 1.0
    c[6:8] = [0.5, 0.5 + 4e-7]     # group 3 score 1.0 + 4e-7, within the band
    assert list(built_oracle.select(cfg, c)) == [2, 3]


# ------------------------------------------------------------------ routing
def test_logits_one_hot_picks_router_column(built_oracle):
    w = small_shape()
    cfg = built_oracle.make_cfg(w)
    wr = synth.host_tensor(w, "router_w", 1)
    x = np.zeros((w.H, w.H), dtype=np.float32)
    np.fill_diagonal(x, 1.0)
    lg = built_oracle.logits(cfg, x, wr)
    assert np.array_equal(lg, bits_to_f64(wr).T)


def test_latent_one_hot_picks_fc1_column(built_oracle):
    w = small_shape()
    cfg = built_oracle.make_cfg(w)
    w1 = synth.host_tensor(w, "fc1_w", 1)
    x = np.zeros((w.H, w.H), dtype=np.float32)
    np.fill_diagonal(x, 1.0)
    assert np.array_equal(built_oracle.latent(cfg, x, w1), bits_to_f64(w1).T)


@pytest.mark.parametrize("x_f32", [True, False])
def test_latent_is_the_matmul_of_the_rounded_input(built_oracle, x_f32):
    """bf16 mode: z before its rounding is rho(x) W_fc1^T (numpy fp64 matmul); with
    bf16 x the rounding of x is the identity."""
    w = small_shape(x_f32=x_f32, H=256, L=64, T=9)
    cfg = built_oracle.make_cfg(w)
    inp = inputs(w)
    x = inp["x"]
    xr = f32_to_bf16_bits(x) if x_f32 else x
    ref = bits_to_f64(xr) @ bits_to_f64(inp["fc1_w"]).T
    got = built_oracle.latent(cfg, x, inp["fc1_w"])
    assert np.allclose(got, ref, rtol=1e-13, atol=1e-13)
    if x_f32:  # rho(x) is applied: the unrounded x gives a different product
        assert not np.allclose(got, x.astype(np.float64) @ bits_to_f64(inp["fc1_w"]).T, rtol=1e-9, atol=0)


def test_weights_sum_to_scale(built_oracle):
    w = replace(TINY, T=64)
    cfg = built_oracle.make_cfg(w)
    inp = inputs(w)
    idx, wt = built_oracle.route(cfg, inp["x"], inp["router_w"], inp["e_bias"])
    assert np.allclose(wt.sum(1), w.s, rtol=0, atol=1e-12)
    assert np.all(np.diff(idx, axis=1) > 0)


def test_zero_input_routes_by_bias(built_oracle):
    w = small_shape(E=16, k=3, G=4, Gk=2, T=4)
    cfg = built_oracle.make_cfg(w)
    inp = inputs(w)
    x = np.zeros((4, w.H), dtype=np.float32)
    idx, wt = built_oracle.route(cfg, x, inp["router_w"], inp["e_bias"])
    expect = brute_force_select(list(0.5 + inp["e_bias"].astype(np.float64)), w.E, w.k, w.G, w.Gk)
    for t in range(4):
        assert list(idx[t]) == expect
        assert np.allclose(wt[t], w.s / w.k, atol=1e-15)


def test_bias_changes_selection_not_weights(built_oracle):
    w = small_shape(E=16, k=3, T=1)
    cfg = built_oracle.make_cfg(w)
    inp = inputs(w)
    x = inp["x"][:1]
    b0 = np.zeros(w.E, dtype=np.float32)
    idx0, _ = built_oracle.route(cfg, x, inp["router_w"], b0)
    lg = bits_to_f64(inp["router_w"]) @ x[0].astype(np.float64)
    sig = 1.0 / (1.0 + np.exp(-lg))
    order = np.argsort(-sig)
    kth, nxt = order[w.k - 1], order[w.k]
    assert kth in idx0 and nxt not in idx0
    b = b0.copy()
    b[nxt] = np.float32(sig[kth] - sig[nxt] + 0.01)   # lifts the (k+1)-th above the k-th
    idx1, w1 = built_oracle.route(cfg, x, inp["router_w"], b)
    assert nxt in idx1 and kth not in idx1
    sel = idx1[0]
    assert np.allclose(w1[0], w.s * sig[sel] / sig[sel].sum(), rtol=1e-14)


# ------------------------------------------------------------------ full layer
@pytest.mark.parametrize("fp32_mode", [True, False])
def test_k_equals_E_is_dense_mixture(built_oracle, fp32_mode):
    w = small_shape(E=6, k=6, T=10)
    cfg = built_oracle.make_cfg(w, fp32_mode=fp32_mode)
    inp = inputs(w)
    y, idx, _ = built_oracle.forward(cfg, inp["x"], inp)
    ref = dense_reference(w, inp["x"], inp, fp32_mode)
    assert np.all(idx == np.arange(6))
    if fp32_mode:
        np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-15)
    else:
        rel = np.linalg.norm(y - ref) / np.linalg.norm(ref)
        assert rel < 1e-3


def test_identical_experts_reduce_to_scale_times_one(built_oracle):
    w = small_shape(E=8, k=3, T=9, Is=16)
    cfg = built_oracle.make_cfg(w, fp32_mode=True)
    inp = inputs(w)
    inp["up_w"] = np.repeat(inp["up_w"][:1], w.E, axis=0)
    inp["down_w"] = np.repeat(inp["down_w"][:1], w.E, axis=0)
    y, _, _ = built_oracle.forward(cfg, inp["x"], inp)
    xf = inp["x"].astype(np.float64)
    z = xf @ bits_to_f64(inp["fc1_w"]).T
    o = np.maximum(z @ bits_to_f64(inp["up_w"][0]).T, 0) ** 2 @ bits_to_f64(inp["down_w"][0]).T
    shared = np.maximum(xf @ bits_to_f64(inp["shared_up_w"]).T, 0) ** 2 @ bits_to_f64(inp["shared_down_w"]).T
    ref = (w.s * o) @ bits_to_f64(inp["fc2_w"]).T + shared
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-15)


def test_token_permutation_equivariance(built_oracle):
    w = small_shape(E=16, k=3, G=4, Gk=2, T=20)
    for fp32_mode in (False, True):
        cfg = built_oracle.make_cfg(w, fp32_mode=fp32_mode)
        inp = inputs(w)
        perm = np.random.default_rng(5).permutation(w.T)
        y, idx, wt = built_oracle.forward(cfg, inp["x"], inp)
        yp, idxp, wtp = built_oracle.forward(cfg, inp["x"][perm], inp)
        assert np.array_equal(yp, y[perm]) and np.array_equal(idxp, idx[perm]) and np.array_equal(wtp, wt[perm])


def test_identity_closed_form(built_oracle):
    # H = L = I, fc1 = fc2 = up = down = identity, shared = 0, E = k = 1:
    # w = s and y = s * relu(x)^2 exactly.
    n = 32
    w = small_shape(H=n, L=n, I=n, Is=16, E=1, k=1, T=7)
    cfg = built_oracle.make_cfg(w, fp32_mode=True)
    eye = f32_to_bf16_bits(np.eye(n, dtype=np.float32))
    inp = inputs(w)
    inp.update(fc1_w=eye, fc2_w=eye, up_w=eye[None], down_w=eye[None],
               shared_up_w=np.zeros((16, n), np.uint16), shared_down_w=np.zeros((n, 16), np.uint16))
    y, idx, wt = built_oracle.forward(cfg, inp["x"], inp)
    xf = inp["x"].astype(np.float64)
    np.testing.assert_allclose(wt, w.s, rtol=1e-15, atol=0)   # s * sigma / sigma, one rounding each
    np.testing.assert_allclose(y, w.s * np.maximum(xf, 0) ** 2, rtol=1e-15, atol=0)


def torch_bf16(v):
    """Nearest-even bf16 of fp32-exact values, through torch (single rounding)."""
    t = torch.from_numpy(np.ascontiguousarray(v, dtype=np.float64))
    assert torch.equal(t.to(torch.float32).to(torch.float64), t), "value not fp32-exact"
    return t.to(torch.float32).to(torch.bfloat16).to(torch.float64).numpy()


def test_rounding_points_closed_form(built_oracle):
    # bf16 mode with fc1 = 1.5 I, up = I, down = 1.5 I, fc2 = I, shared = 0, E = k = 1,
    # s = 4 (so w = 4 exactly): every product is exact, and
    # y = rho(6 rho(relu(rho(1.5 rho(x)))^2)), which needs the bf16 rounding of x, z, a and comb.
    n = 32
    w = small_shape(H=n, L=n, I=n, Is=16, E=1, k=1, T=9, s=4.0)
    cfg = built_oracle.make_cfg(w, fp32_mode=False)
    eye = f32_to_bf16_bits(np.eye(n, dtype=np.float32))
    eye15 = f32_to_bf16_bits(1.5 * np.eye(n, dtype=np.float32))
    inp = inputs(w)
    inp.update(fc1_w=eye15, fc2_w=eye, up_w=eye[None], down_w=eye15[None],
               shared_up_w=np.zeros((16, n), np.uint16), shared_down_w=np.zeros((n, 16), np.uint16))
    y, _, wt = built_oracle.forward(cfg, inp["x"], inp)
    assert np.all(wt == 4.0)
    z = torch_bf16(1.5 * torch_bf16(inp["x"].astype(np.float64)))
    a = torch_bf16(np.maximum(z, 0) ** 2)
    assert np.array_equal(y, torch_bf16(6.0 * a))


def test_shared_rounding_closed_form(built_oracle):
    # bf16 mode, routed path switched off (fc2 = 0), shared up = down = 1.5 I:
    # y = 1.5 rho(relu(1.5 rho(x))^2), which needs the rounding of x and a_s.
    n = 32
    w = small_shape(H=n, L=16, I=16, Is=n, E=2, k=1, T=9)
    cfg = built_oracle.make_cfg(w, fp32_mode=False)
    eye15 = f32_to_bf16_bits(1.5 * np.eye(n, dtype=np.float32))
    inp = inputs(w)
    inp.update(fc2_w=np.zeros((n, 16), np.uint16), shared_up_w=eye15, shared_down_w=eye15)
    y, _, _ = built_oracle.forward(cfg, inp["x"], inp)
    xh = torch_bf16(inp["x"].astype(np.float64))
    assert np.array_equal(y, 1.5 * torch_bf16(np.maximum(1.5 * xh, 0) ** 2))


def test_single_expert_is_dense_mlp_pair(built_oracle):
    w = small_shape(E=1, k=1, T=5)
    cfg = built_oracle.make_cfg(w, fp32_mode=True)
    inp = inputs(w)
    y, _, _ = built_oracle.forward(cfg, inp["x"], inp)
    xf = inp["x"].astype(np.float64)
    Wu, Wd = bits_to_f64(inp["up_w"][0]), bits_to_f64(inp["down_w"][0])
    W1, W2 = bits_to_f64(inp["fc1_w"]), bits_to_f64(inp["fc2_w"])
    Wsu, Wsd = bits_to_f64(inp["shared_up_w"]), bits_to_f64(inp["shared_down_w"])
    ref = np.zeros((w.T, w.H))
    for t in range(w.T):   # naive triple loops, independent of the oracle's code
        z = [sum(xf[t, h] * W1[l, h] for h in range(w.H)) for l in range(w.L)]
        a = [max(sum(z[l] * Wu[i, l] for l in range(w.L)), 0.0) ** 2 for i in range(w.I)]
        o = [w.s * sum(a[i] * Wd[l, i] for i in range(w.I)) for l in range(w.L)]
        sa = [max(sum(xf[t, h] * Wsu[i, h] for h in range(w.H)), 0.0) ** 2 for i in range(w.Is)]
        for h in range(w.H):
            ref[t, h] = sum(o[l] * W2[h, l] for l in range(w.L)) + sum(sa[i] * Wsd[h, i] for i in range(w.Is))
    np.testing.assert_allclose(y, ref, rtol=1e-11, atol=1e-14)


def test_route_matches_forward_routing(built_oracle):
    w = small_shape(E=16, k=4, G=4, Gk=2, T=16, x_f32=False)
    cfg = built_oracle.make_cfg(w)
    inp = inputs(w)
    idx, wt = built_oracle.route(cfg, inp["x"], inp["router_w"], inp["e_bias"])
    _, idx2, wt2 = built_oracle.forward(cfg, inp["x"], inp)
    assert np.array_equal(idx, idx2) and np.array_equal(wt, wt2)


# ------------------------------------------------------------------ page figures
def read_golden(name):
    out = {}
    with open(os.path.join(GOLDEN, name), encoding="utf-8") as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                parts = line.split(None, 3)
                out[parts[0]] = (float(parts[1]), float(parts[2]))
    return out


def test_flop_and_param_counts_match_page_figures():
    g = read_golden("page_figures.txt")
    u = synth.ULTRA_PREFILL
    fl = accounting.flops_breakdown(u)
    pr = accounting.params(u)
    got = {
        "flops_routing_per_token": fl["routing"],
        "flops_latent_proj_per_token": fl["latent_proj"],
        "flops_experts_per_token": fl["experts"],
        "flops_shared_per_token": fl["shared"],
        "flops_per_extra_expert": fl["experts"] / u.k,
        "params_per_expert": pr["per_expert"],
        "params_experts_per_layer": pr["experts_per_layer"],
        "params_latent_proj": pr["latent_proj"],
    }
    for name, (val, tol) in g.items():
        assert abs(got[name] - val) <= tol * val, (name, got[name])


# ------------------------------------------------------------------ bias update (Q5.3, Q5.4)
def test_bias_update_uniform_load_is_a_fixed_point(built_oracle):
    b = synth.uniform_f32(32, 0, 3, -0.1, 0.1)
    nb, mv = built_oracle.update_bias(np.full(32, 7), b, 0.01)
    assert np.array_equal(nb, b) and mv == 0.0


def test_bias_update_moves_against_overload(built_oracle):
    counts = np.array([10, 0, 5, 5], dtype=np.int32)   # mean 5
    b = np.zeros(4, np.float32)
    nb, mv = built_oracle.update_bias(counts, b, 0.001)
    assert nb[0] < 0 < nb[1] and nb[2] == nb[3] == 0.0
    np.testing.assert_allclose(nb, np.float32([-0.005, 0.005, 0.0, 0.0]), rtol=1e-6)
    assert mv == 1.0                                       # (10 - 5) / 5
    # the deviations sum to zero, so the mean bias does not move (up to fp32 rounding)
    rng = np.random.default_rng(1)
    counts = rng.integers(0, 100, 64).astype(np.int32)
    b = rng.uniform(-0.1, 0.1, 64).astype(np.float32)
    nb, _ = built_oracle.update_bias(counts, b, 1e-4)
    assert abs(float(nb.astype(np.float64).sum() - b.astype(np.float64).sum())) < 64 * 1e-8


def test_bias_update_empty_batch(built_oracle):
    nb, mv = built_oracle.update_bias(np.zeros(8, np.int32), np.ones(8, np.float32), 0.5)
    assert np.array_equal(nb, np.ones(8, np.float32)) and mv == 0.0


# ------------------------------------------------------------------ pre-norm RMSNorm block (Q2.8, Q2.1)
def test_rmsnorm_is_a_correct_rounding_of_torch_rms_norm(built_oracle):
    rng = np.random.default_rng(4)
    H = 512
    x = f32_to_bf16_bits(rng.standard_normal((6, H)).astype(np.float32) * 3.0)
    ones = f32_to_bf16_bits(np.ones(H, np.float32))
    out = bits_to_f64(built_oracle.rmsnorm(x, ones, 1e-5))
    ref = torch.nn.functional.rms_norm(torch.from_numpy(bits_to_f64(x)), (H,), eps=1e-5).numpy()
    half_ulp = np.ldexp(1.0, np.frexp(np.abs(ref))[1] - 9)   # half a bf16 ulp of each reference value
    assert np.all(np.abs(out - ref) <= half_ulp * (1 + 1e-9))


def test_rmsnorm_closed_forms(built_oracle):
    H = 64
    sign = np.where(np.arange(H) % 3 == 0, -1.0, 1.0).astype(np.float32)
    x = f32_to_bf16_bits(2.0 * sign[None, :])
    # |x| = 2 everywhere: r = 1/sqrt(4 + eps) and bf16(x r) = +-1; gamma = 1.5 gives +-1.5
    g = f32_to_bf16_bits(np.full(H, 1.5, np.float32))
    assert np.array_equal(bits_to_f64(built_oracle.rmsnorm(x, g, 1e-5)), 1.5 * sign[None, :])
    # without eps the norm is invariant to scaling x by a power of two
    rng = np.random.default_rng(5)
    xr = f32_to_bf16_bits(rng.standard_normal((3, H)).astype(np.float32))
    g = f32_to_bf16_bits(rng.uniform(0.5, 1.5, H).astype(np.float32))
    a = built_oracle.rmsnorm(xr, g, 0.0)
    b = built_oracle.rmsnorm(f32_to_bf16_bits(bits_to_f64(xr).astype(np.float32) * 8.0), g, 0.0)
    assert np.array_equal(a, b)


def test_block_is_residual_plus_layer_of_normed_input(built_oracle):
    w = small_shape(E=8, k=2, T=5, x_f32=False)
    cfg = built_oracle.make_cfg(w)
    inp = inputs(w)
    g = f32_to_bf16_bits(np.random.default_rng(6).uniform(0.5, 1.5, w.H).astype(np.float32))
    y, idx, _ = built_oracle.forward_block(cfg, inp["x"], g, 1e-5, inp)
    xn = built_oracle.rmsnorm(inp["x"], g, 1e-5)
    y2, idx2, _ = built_oracle.forward(cfg, xn, inp)
    assert np.array_equal(idx, idx2)
    assert np.array_equal(y, y2 + bits_to_f64(inp["x"]))


# ---------------------------------------------------------------- NVFP4 experts
E2M1_MAGNITUDES = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def test_e2m1_decode_follows_bit_fields(built_oracle):
    got = [built_oracle.e2m1_value(c) for c in range(16)]
    assert got[:8] == E2M1_MAGNITUDES
    assert got[8:] == [-v for v in E2M1_MAGNITUDES]


def test_e4m3_decode_matches_torch_float8(built_oracle):
    ref = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([built_oracle.e4m3_value(b) for b in range(256)])
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(got)) and nan.sum() == 2
    assert np.array_equal(ref[~nan], got[~nan])
    assert built_oracle.e4m3_value(0x7E) == 448.0 and built_oracle.e4m3_value(1) == 2.0 ** -9


def test_e4m3_encode_matches_torch_rounding(built_oracle):
    rng = np.random.default_rng(11)
    finite = [built_oracle.e4m3_value(b) for b in range(0x7F)]
    mids = [(a + b) / 2 for a, b in zip(finite[:-1], finite[1:])]      # exact ties
    us = np.concatenate([rng.uniform(0, 448, 4000), np.exp(rng.uniform(-12, 6, 4000)), finite, mids]).astype(np.float32)
    us = us[us <= 448]
    ref = torch.from_numpy(us).to(torch.float8_e4m3fn).view(torch.uint8).numpy().astype(int)
    got = np.array([built_oracle.e4m3_encode(float(u)) for u in us])
    assert np.array_equal(ref, got)
    assert built_oracle.e4m3_encode(1e6) == 0x7E and built_oracle.e4m3_encode(0.0) == 0


def test_e2m1_encode_nearest_with_even_ties(built_oracle):
    # exact midpoints go to the even mantissa (code & 1 == 0)
    ties = {0.25: 0, 0.75: 2, 1.25: 2, 1.75: 4, 2.5: 4, 3.5: 6, 5.0: 6}
    for q, c in ties.items():
        assert built_oracle.e2m1_encode(q) == c
        assert built_oracle.e2m1_encode(-q) == (c | 8)
    rng = np.random.default_rng(12)
    for q in rng.uniform(-8, 8, 3000).astype(np.float32):
        c = built_oracle.e2m1_encode(float(q))
        mag = E2M1_MAGNITUDES[c & 7]
        best = min(abs(abs(q) - m) for m in E2M1_MAGNITUDES) if abs(q) < 6 else abs(q) - 6.0
        assert abs(abs(q) - mag) == pytest.approx(best, abs=0) or (abs(q) >= 6 and c & 7 == 7)
        assert (c >> 3) == (q < 0)


def read_nvfp4_example():
    scales, elems, g = {}, {}, None
    with open(os.path.join(GOLDEN, "nvfp4_worked_example.txt"), encoding="utf-8") as f:
        for line in f:
            p = line.split()
            if not p or p[0].startswith("#"):
                continue
            if p[0] == "g":
                g = float(p[1])
            elif p[0] == "scale":
                scales[int(p[1])] = int(p[2], 16)
            elif p[0] == "elem":
                elems[int(p[1])] = (float(p[2]), int(p[3]))
    return g, scales, elems


def test_nvfp4_quantize_worked_example(built_oracle):
    g_ref, scales, elems = read_nvfp4_example()
    R, K, row = 128, 64, 5
    wf = np.zeros((1, R, K), dtype=np.float32)
    for k, (v, _) in elems.items():
        wf[0, row, k] = v
    w = f32_to_bf16_bits(wf).reshape(1, R, K)
    assert np.array_equal(bits_to_f64(w).reshape(1, R, K)[0, row], wf[0, row].astype(np.float64))  # values exact
    codes, sf, g = built_oracle.nvfp4_quantize(w)
    assert g[0] == np.float32(g_ref)
    for b, byte in scales.items():
        assert sf[row * 4 + b] == byte, b
    for k in range(K):
        byte = codes[row * 32 + k // 2]
        code = (byte >> 4) if k & 1 else (byte & 15)
        assert code == elems.get(k, (0.0, 0))[1], k
    other = np.ones(R, dtype=bool)
    other[row] = False
    assert not codes.reshape(R, 32)[other].any() and not sf.reshape(R, 4)[other].any()


def nvfp4_weights(rng, n_mat, R, K, std=0.02):
    return f32_to_bf16_bits(rng.normal(0, std, (n_mat, R, K)).astype(np.float32)).reshape(n_mat, R, K)


def test_nvfp4_error_bound_and_block_max(built_oracle):
    rng = np.random.default_rng(13)
    n_mat, R, K = 2, 128, 128
    w = nvfp4_weights(rng, n_mat, R, K)
    codes, sf, g = built_oracle.nvfp4_quantize(w)
    deq = bits_to_f64(built_oracle.nvfp4_dequant(codes, sf, n_mat, R, K)).reshape(n_mat, R, K)
    wf = bits_to_f64(w).reshape(n_mat, R, K)
    blocks = wf.reshape(n_mat, R, K // 16, 16)
    S = np.abs(deq.reshape(n_mat, R, K // 16, 16)).max(axis=3) / 6.0  # block max element decodes to 6 * S
    for m in range(n_mat):
        # block scale: S = E4M3(bmax / g / 6) within half an E4M3 step (relative 1/16)
        u = np.abs(blocks[m]).max(axis=2) / g[m] / 6.0
        assert np.all(np.abs(S[m] - u) <= u / 16 + 1e-30)
        d = S[m][..., None] * g[m]
        q = blocks[m] / d
        v = deq[m].reshape(R, K // 16, 16) * g[m]
        # per element: error at most half the E2M1 spacing at |q| (0.5 below 2, 1 below 4, 2 above), or the
        # saturation error above 6
        half = np.where(np.abs(q) < 2, 0.25, np.where(np.abs(q) < 4, 0.5, 1.0)) * d
        sat = np.maximum(np.abs(blocks[m]) - 6 * d, 0)
        assert np.all(np.abs(blocks[m] - v) <= np.maximum(half, sat) * (1 + 1e-6))


def test_nvfp4_requantising_the_dequantised_matrix_is_idempotent(built_oracle):
    rng = np.random.default_rng(14)
    n_mat, R, K = 2, 128, 64
    codes, sf, g = built_oracle.nvfp4_quantize(nvfp4_weights(rng, n_mat, R, K))
    deq = built_oracle.nvfp4_dequant(codes, sf, n_mat, R, K)
    codes2, sf2, g2 = built_oracle.nvfp4_quantize(deq)
    # the matrix maximum sits in a block with S = 448 and code 6, so g' = 6 * 448 / 2688 = 1
    assert np.all(g2 == 1.0)

    def plus_zero(c):  # -0 (code 8) dequantises to -0.0, which quantises to +0
        lo, hi = c & 15, c >> 4
        return np.where(lo == 8, 0, lo) | (np.where(hi == 8, 0, hi) << 4)

    assert np.array_equal(sf, sf2) and np.array_equal(plus_zero(codes), plus_zero(codes2))
    assert np.array_equal(codes2, plus_zero(codes2))


def test_nvfp4_rejects_untiled_shapes(built_oracle):
    with pytest.raises(ValueError):
        built_oracle.nvfp4_quantize(np.zeros((1, 64, 64), dtype=np.uint16))


def test_expert_matrix_scales_enter_before_the_activation(built_oracle):
    # A power-of-two matrix scale is exact in bf16 and fp64: scaling the weights by it or passing it as
    # the per-expert matrix scale must give bitwise the same layer (relu2 of 2h is 4 relu2(h), so a scale
    # applied after the activation would not).
    w = small_shape(E=8, k=3, T=6, x_f32=False)
    cfg = built_oracle.make_cfg(w)
    inp = inputs(w)
    up = bits_to_f64(inp["up_w"]).astype(np.float32)
    dn = bits_to_f64(inp["down_w"]).astype(np.float32)
    gu = np.array([2.0 ** (e % 3) for e in range(w.E)], dtype=np.float32)
    gd = np.array([2.0 ** -(e % 2) for e in range(w.E)], dtype=np.float32)
    scaled = dict(inp)
    scaled["up_w"] = f32_to_bf16_bits(up * gu[:, None, None]).reshape(inp["up_w"].shape)
    scaled["down_w"] = f32_to_bf16_bits(dn * gd[:, None, None]).reshape(inp["down_w"].shape)
    y1, idx1, _ = built_oracle.forward(cfg, inp["x"], dict(inp, up_gs=gu, down_gs=gd))
    y2, idx2, _ = built_oracle.forward(cfg, inp["x"], scaled)
    assert np.array_equal(idx1, idx2) and np.array_equal(y1, y2)
    y3, _, _ = built_oracle.forward(cfg, inp["x"], inp)
    assert not np.array_equal(y1, y3)
