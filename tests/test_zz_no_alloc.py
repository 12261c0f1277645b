"""latentmoe_route_noalloc: routing for callers that cannot allocate device memory.

Such callers (a latency-critical section where cudaMalloc's implicit
synchronisation is not allowed, a runtime whose device memory is a fixed arena,
a plugin host that forbids allocation) get routing without a workspace: the
scratch is the library's own static device array. This file checks, through the
C ABI, that two calls in a row give exactly what latentmoe_route gives (routing
is compared bit for bit, as everywhere else), and that an oversized batch is
refused without touching the outputs. It is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest

import synth
from synth import LayerShape

pytestmark = pytest.mark.gpu

SHAPE = LayerShape("noalloc", T=128, H=4096, L=2048, E=128, k=8, G=8, Gk=4, I=2560, Is=5120)


def _route_noalloc(lm, layer, x, T, k, E):
    import torch
    idx = torch.full((T, k), -1, dtype=torch.int32, device="cuda")
    w = torch.full((T, k), -1.0, dtype=torch.float32, device="cuda")
    counts = torch.full((E,), -1, dtype=torch.int32, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    s = lm.latentmoe_route_noalloc(layer.h, x.data_ptr(), T, idx.data_ptr(), w.data_ptr(), counts.data_ptr(), stream)
    return s, idx, w, counts


def test_route_noalloc_matches_route_on_two_calls_in_a_row():
    import torch
    import latentmoe_layer_b200 as lm
    dev = synth.device_inputs(SHAPE, 0)
    layer = lm.LatentMoE(SHAPE, dev, max_tokens=8192)
    other = synth.device_inputs(SHAPE.with_tokens(97), 5)["x"]  # different tokens, ragged T
    for x in (dev["x"], other):
        T = x.shape[0]
        s, idx, w, counts = _route_noalloc(lm, layer, x, T, SHAPE.k, SHAPE.E)
        assert s == lm.LMOE_OK, lm.status_string(s)
        ridx, rw, rcounts = layer.route(x)
        torch.cuda.synchronize()
        assert torch.equal(idx, ridx)
        assert torch.equal(w, rw)
        assert torch.equal(counts, rcounts)
        assert int(counts.sum()) == T * SHAPE.k
        assert np.all(np.diff(idx.cpu().numpy(), axis=1) > 0)
    layer.close()


def test_route_noalloc_refuses_a_batch_beyond_its_scratch():
    import torch
    import latentmoe_layer_b200 as lm
    dev = synth.device_inputs(SHAPE, 0)
    layer = lm.LatentMoE(SHAPE, dev, max_tokens=8192)
    x = torch.zeros((8192, SHAPE.H), dtype=torch.bfloat16, device="cuda")
    s, idx, w, counts = _route_noalloc(lm, layer, x, 8192, SHAPE.k, SHAPE.E)
    torch.cuda.synchronize()
    assert s == lm.LMOE_ERR_WORKSPACE
    assert bool((idx == -1).all()) and bool((counts == -1).all())
    layer.close()
