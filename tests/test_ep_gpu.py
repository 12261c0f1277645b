"""Expert-parallel stages on the GPU (latentmoe_ep_front / _ep_experts / _ep_back).

- One rank (P = 1): the three stages give latentmoe_forward's y bit for bit,
  called directly and through ep_forward over a one-rank NCCL group.
- Two and four ranks emulated in one process: handles each holding E/P of the
  experts, the all-to-all done with plain buffer copies (nothing waits across
  ranks); each rank's y equals the single-handle forward of its tokens bit for
  bit, and the assembled y is within the stated tolerances of the fp64 oracle
  (ragged and Nano shapes).
"""
from dataclasses import replace

import numpy as np
import pytest

import synth
from synth import LayerShape
import helpers as H
import oracle

pytestmark = pytest.mark.gpu

GEMM_AUTO, GEMM_PREFILL, GEMM_DECODE = 0, 1, 2
RAGGED = LayerShape("ragged", T=333, H=512, L=256, E=64, k=6, G=4, Gk=2, I=384, Is=640)
NANO_EP = synth.NANO_DECODE


def stages(layer, x, n_src=1):
    import torch
    shape = layer.shape
    T = x.shape[0]
    A = T * shape.k
    send_rows = torch.empty((A, shape.L), dtype=torch.bfloat16, device="cuda")
    send_w = torch.empty((A,), dtype=torch.float32, device="cuda")
    counts = torch.empty((shape.E,), dtype=torch.int32, device="cuda")
    layer.ep_front(x, send_rows, send_w, counts)
    return send_rows, send_w, counts


@pytest.mark.parametrize("path", [GEMM_PREFILL, GEMM_DECODE])
def test_one_rank_stages_equal_forward_bitwise(path):
    import torch
    layer, dev = H.device_layer(RAGGED)
    layer.set_option(0, path)
    y_ref = layer.forward(dev["x"])
    send_rows, send_w, counts = stages(layer, dev["x"])
    o = torch.empty((send_rows.shape[0], RAGGED.L), dtype=torch.float32, device="cuda")
    layer.ep_experts(send_rows, send_w, counts, 1, o)
    y = torch.empty_like(y_ref)
    layer.ep_back(o, y)
    torch.cuda.synchronize()
    assert layer.stats().device_error == 0
    assert torch.equal(y, y_ref)


def test_one_rank_nvfp4_stages_equal_forward_bitwise():
    import torch
    import latentmoe_layer_b200 as lm
    shape = replace(RAGGED, name="ragged_fp4")
    dev = synth.device_inputs(shape, 0)
    q = {}
    q["up_w"], q["up_sf"], q["up_gs"] = lm.quantize_nvfp4(dev["up_w"])
    q["down_w"], q["down_sf"], q["down_gs"] = lm.quantize_nvfp4(dev["down_w"])
    layer = lm.LatentMoE(shape, dict(dev, **q), shape.T, expert_format=lm.LMOE_EXPERTS_NVFP4)
    y_ref = layer.forward(dev["x"])
    send_rows, send_w, counts = stages(layer, dev["x"])
    o = torch.empty((send_rows.shape[0], shape.L), dtype=torch.float32, device="cuda")
    layer.ep_experts(send_rows, send_w, counts, 1, o)
    y = torch.empty_like(y_ref)
    layer.ep_back(o, y)
    torch.cuda.synchronize()
    assert torch.equal(y, y_ref)


def emulate_ranks(shape, P, splits, dev=None):
    """P expert-parallel ranks emulated in one process: P shard handles (experts
    r*E/P .. (r+1)*E/P - 1 each), rank r on tokens splits[r]:splits[r+1] of x, the
    all-to-all done as buffer copies (nothing waits across ranks). Returns the
    ranks' y, the single-handle forward of the same tokens, and the inputs."""
    import torch
    import latentmoe_layer_b200 as lm
    from latentmoe_layer_b200 import ep
    El = shape.E // P
    dev = dev or synth.device_inputs(shape, 0)
    full = lm.LatentMoE(shape, dev, shape.T)
    xs = [dev["x"][splits[r]:splits[r + 1]] for r in range(P)]
    y_ref = [full.forward(x).clone() for x in xs]
    ranks = [lm.LatentMoE(shape, ep.shard_weights(dev, shape.E, r, P), shape.T, local_experts=El,
                          expert_base=r * El) for r in range(P)]
    fronts = [stages(ranks[r], xs[r]) for r in range(P)]
    # the all-to-all: rank r's rows for rank d are its rows of experts d*El .. (d+1)*El - 1
    offs = []
    for r in range(P):
        c = fronts[r][2].cpu().numpy()
        offs.append(np.concatenate([[0], np.cumsum([c[d * El:(d + 1) * El].sum() for d in range(P)])]))
    outs = [None] * P
    for d in range(P):
        rows = torch.cat([fronts[s][0][offs[s][d]:offs[s][d + 1]] for s in range(P)])
        w = torch.cat([fronts[s][1][offs[s][d]:offs[s][d + 1]] for s in range(P)])
        rc = torch.cat([fronts[s][2][d * El:(d + 1) * El] for s in range(P)]).contiguous()
        o = torch.empty((rows.shape[0], shape.L), dtype=torch.float32, device="cuda")
        ranks[d].ep_experts(rows, w, rc, P, o)
        outs[d] = (o, [int(offs[s][d + 1] - offs[s][d]) for s in range(P)])
    ys = []
    for r in range(P):
        back = []
        for d in range(P):
            o, sizes = outs[d]
            start = sum(sizes[:r])
            back.append(o[start:start + sizes[r]])
        send_o = torch.cat(back)
        y = torch.empty_like(y_ref[r])
        ranks[r].ep_back(send_o, y)
        ys.append(y)
    torch.cuda.synchronize()
    for r in range(P):
        assert ranks[r].stats().device_error == 0
    return ys, y_ref, ranks, dev


def check_ep_against_oracle(shape, P, splits):
    """Each emulated rank's y equals the single-handle forward bit for bit (the experts
    of a token are summed in ascending id on both paths), and the assembled y of all
    tokens is within the stated tolerances of the fp64 oracle."""
    import torch
    ys, y_ref, ranks, dev = emulate_ranks(shape, P, splits)
    for r in range(P):
        assert torch.equal(ys[r], y_ref[r]), "rank %d differs from the single handle" % r
    y = torch.cat(ys).cpu().numpy()
    host = synth.host_inputs(shape)
    yref, _, _ = H.oracle_forward(shape, host["x"][:splits[-1]], host)
    ma, rf = H.assert_bf16_close(y, yref)
    print("%s P=%d: bitwise equal to the single handle; vs oracle max_abs=%.3g rel_fro=%.3g" % (shape.name, P, ma, rf))
    return ranks, dev


def test_two_ranks_emulated_bitwise_and_oracle():
    import latentmoe_layer_b200 as lm
    ranks, dev = check_ep_against_oracle(RAGGED, 2, [0, 170, RAGGED.T])
    with pytest.raises(lm.LmoeError):  # a shard handle refuses the single-GPU forward
        ranks[0].forward(dev["x"][:170])


def test_four_ranks_emulated_bitwise_and_oracle():
    check_ep_against_oracle(RAGGED, 4, [0, 1, 120, 200, RAGGED.T])


def test_two_ranks_emulated_nano_bitwise_and_oracle():
    check_ep_against_oracle(NANO_EP, 2, [0, 61, NANO_EP.T])


def test_ep_forward_one_rank_nccl_group():
    import os
    import datetime
    import socket
    import torch
    import torch.distributed as dist
    from latentmoe_layer_b200 import ep
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    try:
        layer, dev = H.device_layer(RAGGED)
        y_ref = layer.forward(dev["x"])
        y = ep.ep_forward(layer, dev["x"])
        torch.cuda.synchronize()
        assert torch.equal(y, y_ref)
    finally:
        dist.destroy_process_group()


def test_ep_experts_rejects_counts_that_do_not_add_up():
    import torch
    import latentmoe_layer_b200 as lm
    layer, dev = H.device_layer(RAGGED)
    send_rows, send_w, counts = stages(layer, dev["x"])
    n = send_rows.shape[0]
    bad = counts.clone()
    bad[0] += 7  # more rows than given: no GEMM tile may run past the buffers
    o = torch.full((n, RAGGED.L), 3.0, dtype=torch.float32, device="cuda")
    layer.ep_experts(send_rows, send_w, bad, 1, o)
    torch.cuda.synchronize()
    assert bool((o == 3.0).all())
    with pytest.raises(lm.LmoeError) as ei:
        layer.ep_experts(send_rows, send_w, counts, 1, o)  # the recorded error surfaces on the next call
    assert ei.value.status == lm.LMOE_ERR_INVALID_ARG
