"""The N > 1 host logic of bench.py on CPU with gloo, world size 2.

The layer is token-independent, so N GPUs run N replicas over disjoint token
ranges with no exchange. This checks, with two gloo ranks: the ranks' token
ranges tile the generator's x stream, the per-rank results (the oracle stands
in for the device layer) equal one computation over all tokens, and the timing
reduction returns the slowest rank.
"""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

from synth import LayerShape

SHAPE = LayerShape("replica", T=6, H=64, L=32, E=8, k=2, G=2, Gk=1, I=64, Is=64)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out_dir):
    import datetime
    import torch.distributed as dist
    import bench
    import oracle
    import synth
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    off = bench.replica_x_offset(rank, SHAPE)
    x = synth.normal_bf16(SHAPE.T * SHAPE.H, 0, synth.TID_X, 1.0, off).reshape(SHAPE.T, SHAPE.H)
    wts = synth.host_inputs(SHAPE, 0)
    y, idx, _ = oracle.forward(oracle.make_cfg(SHAPE), x, wts)
    slowest = bench.max_over_ranks(10.0 * (rank + 1), dist, "cpu")
    np.savez(os.path.join(out_dir, "rank%d.npz" % rank), x=x, y=y, idx=idx, slowest=slowest)
    dist.barrier()
    dist.destroy_process_group()


def test_two_replicas_cover_disjoint_tokens_and_max_time(tmp_path, built_oracle):
    world = 2
    mp.spawn(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    import oracle
    import synth
    parts = [np.load(os.path.join(tmp_path, "rank%d.npz" % r)) for r in range(world)]
    x_all = synth.normal_bf16(world * SHAPE.T * SHAPE.H, 0, synth.TID_X, 1.0, 0).reshape(world * SHAPE.T, SHAPE.H)
    assert np.array_equal(np.concatenate([p["x"] for p in parts]), x_all)
    wts = synth.host_inputs(SHAPE, 0)
    big = LayerShape(**{**SHAPE.as_dict(), "T": world * SHAPE.T})
    y_all, idx_all, _ = oracle.forward(oracle.make_cfg(big), x_all, wts)
    assert np.array_equal(np.concatenate([p["y"] for p in parts]), y_all)
    assert np.array_equal(np.concatenate([p["idx"] for p in parts]), idx_all)
    assert all(float(p["slowest"]) == 20.0 for p in parts)
