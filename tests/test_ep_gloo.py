"""Host logic of the expert-parallel forward (latentmoe_layer_b200.ep) with two
gloo ranks on CPU.

The GPU stages are replaced by a mock with the same interface (test only): its
front emits rows tagged with (rank, token, slot, expert), its experts stage
records which rank processed which row and returns a value derived from the
tag, its back checks that every row came back to its sender in send order.
This covers the split sizes, the dispatch and the return paths of ep_forward
for uneven counts, including an expert block with no rows and a rank that
receives none.
"""
import os
import socket

import numpy as np
import torch
import torch.multiprocessing as mp

E, K, L, H = 8, 2, 4, 3


class Shape:
    pass


SHAPE = Shape()
SHAPE.E, SHAPE.k, SHAPE.L, SHAPE.H = E, K, L, H


def routing(rank, T):
    """Deterministic expert choices; rank 1 uses only experts 0..3 (rank 0's block)."""
    rng = np.random.default_rng(100 + rank)
    hi = E // 2 if rank == 1 else E
    idx = np.stack([np.sort(rng.choice(hi, K, replace=False)) for _ in range(T)])
    return idx.astype(np.int64)


class MockLayer:
    def __init__(self, rank, world):
        self.rank, self.world, self.shape = rank, world, SHAPE
        self.el = E // world

    def ep_front(self, x, send_rows, send_w, counts):
        T = x.shape[0]
        idx = routing(self.rank, T)
        pairs = sorted((int(idx[t, j]), t, j) for t in range(T) for j in range(K))  # expert order, stable in t
        self.sent = pairs
        for r, (e, t, j) in enumerate(pairs):
            send_rows[r] = torch.tensor([self.rank, t, j, e], dtype=send_rows.dtype)
            send_w[r] = float(e + 1)
        counts.copy_(torch.from_numpy(np.bincount(idx.ravel(), minlength=E).astype(np.int32)))

    def ep_experts(self, recv_rows, recv_w, recv_counts, n_src, recv_o):
        rc = recv_counts.reshape(n_src, self.el).numpy()
        r = 0
        for s in range(n_src):
            for el in range(self.el):
                for _ in range(rc[s, el]):
                    src, t, j, e = [int(v) for v in recv_rows[r].tolist()]
                    assert src == s and e == self.rank * self.el + el, (src, s, e, el)  # arrival order
                    assert float(recv_w[r]) == e + 1
                    recv_o[r] = torch.tensor([src, t, j, 1000 * self.rank + e], dtype=recv_o.dtype)
                    r += 1
        assert r == recv_rows.shape[0]

    def ep_back(self, send_o, y):
        for r, (e, t, j) in enumerate(self.sent):
            src, tt, jj, v = [int(x) for x in send_o[r].tolist()]
            assert (src, tt, jj) == (self.rank, t, j), (r, src, tt, jj)
            assert v == 1000 * (e // (E // self.world)) + e  # processed by the owner of expert e
        y.fill_(float(len(self.sent)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out_dir):
    import datetime
    import torch.distributed as dist
    from latentmoe_layer_b200 import ep
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    T = 5 + 2 * rank
    layer = MockLayer(rank, world)
    x = torch.zeros((T, H))
    counts = torch.from_numpy(np.bincount(routing(rank, T).ravel(), minlength=E).astype(np.int32))
    send_splits, recv_counts, recv_splits = ep.exchange_plan(counts, world)
    y = ep.ep_forward(layer, x)
    np.savez(os.path.join(out_dir, "rank%d.npz" % rank), counts=counts.numpy(), send=np.array(send_splits),
             recv=np.array(recv_splits), recv_counts=recv_counts.numpy(), y=y.numpy())
    dist.barrier()
    dist.destroy_process_group()


def test_exchange_plan_and_round_trip_two_ranks(tmp_path):
    world = 2
    mp.spawn(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    r = [np.load(os.path.join(tmp_path, "rank%d.npz" % i)) for i in range(world)]
    el = E // world
    for i in range(world):
        # rows sent to rank d = this rank's counts of d's experts
        assert list(r[i]["send"]) == [int(r[i]["counts"][d * el:(d + 1) * el].sum()) for d in range(world)]
        # rows received from source s for local expert e = s's count of expert i*el + e
        for s in range(world):
            assert np.array_equal(r[i]["recv_counts"][s], r[s]["counts"][i * el:(i + 1) * el])
        assert list(r[i]["recv"]) == [int(r[i]["recv_counts"][s].sum()) for s in range(world)]
        assert np.all(r[i]["y"] == (5 + 2 * i) * K)  # every row came back (checked in the mock's back)
    assert r[1]["send"][1] == 0  # rank 1 routes nothing to rank 1's experts: an empty exchange
