"""Expert-load statistics and the load-balancing bias update on the GPU.

The pages ("Nemotron 3 Ultra 架构 QA", Q5.3) describe the bias as auxiliary
state the training framework moves against the measured load; Q5.4 reports the
resulting MaxVio. latentmoe_update_bias implements that step; these tests check
it bit for bit against the oracle and show it balancing a skewed router.
"""
import ctypes

import numpy as np
import pytest

import oracle
import synth
from synth import LayerShape

pytestmark = pytest.mark.gpu


def test_update_bias_matches_oracle_bit_for_bit():
    import torch
    import latentmoe_layer_b200 as lm
    import helpers as H
    layer, dev = H.device_layer(synth.TINY)
    rng = np.random.default_rng(2)
    E = synth.TINY.E
    for trial in range(3):
        counts = rng.integers(0, 200, E).astype(np.int32)
        bias = rng.uniform(-0.1, 0.1, E).astype(np.float32)
        eta = [1e-3, 0.37, 5e-6][trial]
        c_d = torch.from_numpy(counts).cuda()
        b_d = torch.from_numpy(bias).cuda()
        out = torch.empty_like(b_d)
        mv = torch.zeros(1, dtype=torch.float64, device="cuda")
        st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
        s = lm.latentmoe_update_bias(layer.h, c_d.data_ptr(), b_d.data_ptr(), eta, out.data_ptr(), mv.data_ptr(), st)
        assert s == lm.LMOE_OK
        ref, ref_mv = oracle.update_bias(counts, bias, float(np.float32(eta)))
        torch.cuda.synchronize()
        assert np.array_equal(out.cpu().numpy().view(np.uint32), ref.view(np.uint32))
        assert float(mv.item()) == ref_mv
        # in place
        s = lm.latentmoe_update_bias(layer.h, c_d.data_ptr(), b_d.data_ptr(), eta, b_d.data_ptr(), None, st)
        torch.cuda.synchronize()
        assert s == lm.LMOE_OK and np.array_equal(b_d.cpu().numpy().view(np.uint32), ref.view(np.uint32))


def test_bias_update_balances_a_skewed_router():
    """Four hot experts (+3.0 logit through the router weights) draw most of the
    load; repeated route -> update steps on the handle's own bias bring MaxVio down."""
    import torch
    import latentmoe_layer_b200 as lm
    import helpers as H
    shape = LayerShape("skewed", T=512, H=256, L=64, E=32, k=4, G=4, Gk=2, I=128, Is=128, skew_hot=4,
                       skew_offset=3.0)
    layer, dev = H.device_layer(shape)
    mv = torch.zeros(1, dtype=torch.float64, device="cuda")
    history = []
    for it in range(40):
        _, _, counts = layer.route(dev["x"])
        layer.update_bias(counts, 2e-4, maxvio=mv)
        torch.cuda.synchronize()
        history.append(float(mv.item()))
    print("MaxVio over steps:", " ".join("%.2f" % v for v in history[::5]), "->", "%.2f" % history[-1])
    assert history[0] > 1.0
    assert history[-1] < 0.5 * history[0]
    # the forward pass routes with the updated bias: its counts equal route()'s
    _, _, c1 = layer.route(dev["x"])
    c2 = torch.empty_like(c1)
    layer.forward(dev["x"], counts=c2)
    torch.cuda.synchronize()
    assert torch.equal(c1, c2)
