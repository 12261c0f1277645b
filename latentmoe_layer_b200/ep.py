"""Expert-parallel LatentMoE forward: one process per GPU, experts in contiguous
blocks of E/P ids per rank, the L-wide latent rows exchanged all-to-all.

The pages give the reason for the latent width ("Nemotron-3-Labs-Ultra-Math-SFT"
article, section 什么是 Latent 瓶颈: tokens cross between experts as 2048-wide
latent rows, a quarter of the hidden width, which cuts the traffic of multi-GPU
expert parallelism) and the deployment (its notes: the 512 experts sharded over
the GPUs). Every step of the arithmetic runs in the library's kernels
(latentmoe_ep_front / _ep_experts / _ep_back); this module only moves buffers
with torch.distributed (NCCL between GPUs; any backend that implements
all_to_all_single for the host-side plan).

Per forward, on every rank:
  1 front    routing, z = fc1(x), a_s; send_rows = z rows in expert order, which
             is also destination-rank order (rank r owns experts r*E/P ..)
  2 plan     all-to-all of the per-expert counts [P, E/P] -> split sizes
  3 dispatch all-to-all of the rows (bf16) and their routing weights (fp32)
  4 experts  this rank's experts on the received rows, in arrival order
  5 return   all-to-all of the fp32 results back to the senders
  6 back     combine in ascending expert id and fc2 + shared down -> y

Costs this design accepts:
  - The return leg carries fp32 rows, 4*L bytes per assignment (8 KB at L = 2048)
    against 2*L on the bf16 dispatch: the expert outputs o_e are fp32 up to the
    combine's single rounding, so a bf16 return would add a rounding the layer
    does not have. The exchange moves 6*L bytes per assignment in all, still
    under half of what hidden-width rows would (2*H out, 4*H back at H = 4*L).
  - exchange_plan reads the split sizes on the host (one device-to-host copy of
    P integers and the wait for it, per forward): all_to_all_single takes host
    split sizes. An exchange at fixed capacity would need no host read but move
    up to min(k, E/P) * T rows to every rank, P times the mean at the Ultra
    shape.
"""
from __future__ import annotations


def shard_weights(weights: dict, num_experts: int, rank: int, world: int, nvfp4: bool = False) -> dict:
    """This rank's view of the layer weights: everything shared, the up/down
    weights (and NVFP4 scales) of experts rank*E/P .. (rank+1)*E/P - 1 only.
    Slices of contiguous tensors, so no copy is made."""
    if num_experts % world:
        raise ValueError("the experts must split evenly over the ranks")
    el = num_experts // world
    lo, hi = rank * el, (rank + 1) * el
    out = dict(weights)
    if nvfp4:
        for key in ("up_w", "up_sf", "down_w", "down_sf"):
            t = weights[key]
            per = t.numel() // num_experts
            out[key] = t[lo * per:hi * per]
        out["up_gs"] = weights["up_gs"][lo:hi]
        out["down_gs"] = weights["down_gs"][lo:hi]
    else:
        out["up_w"] = weights["up_w"][lo:hi]
        out["down_w"] = weights["down_w"][lo:hi]
    return out


def exchange_plan(counts, world: int, group=None):
    """counts: this rank's rows per expert [E] int32, in expert order.
    Returns (send_splits, recv_counts [world, E/P], recv_splits): rows sent to
    each rank, and the per-(source, local expert) counts and rows received."""
    import torch.distributed as dist
    el = counts.numel() // world
    per_dest = counts.reshape(world, el).contiguous()
    recv_counts = per_dest.new_empty((world, el))
    dist.all_to_all_single(recv_counts, per_dest, group=group)
    send_splits = [int(v) for v in per_dest.sum(dim=1).tolist()]
    recv_splits = [int(v) for v in recv_counts.sum(dim=1).tolist()]
    return send_splits, recv_counts, recv_splits


def ep_forward(layer, x, group=None):
    """y = layer(x) with this rank holding experts rank*E/P .. of E. `layer`: a
    LatentMoE handle created with local_experts = E/P and expert_base =
    rank*E/P on this rank's shard (shard_weights). x: this rank's tokens."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    shape = layer.shape
    T = x.shape[0]
    A = T * shape.k
    dev = x.device
    send_rows = torch.empty((A, shape.L), dtype=torch.bfloat16, device=dev)
    send_w = torch.empty((A,), dtype=torch.float32, device=dev)
    counts = torch.empty((shape.E,), dtype=torch.int32, device=dev)
    layer.ep_front(x, send_rows, send_w, counts)
    send_splits, recv_counts, recv_splits = exchange_plan(counts, world, group)
    n_recv = sum(recv_splits)
    recv_rows = torch.empty((n_recv, shape.L), dtype=torch.bfloat16, device=dev)
    recv_w = torch.empty((n_recv,), dtype=torch.float32, device=dev)
    dist.all_to_all_single(recv_rows, send_rows, recv_splits, send_splits, group=group)
    dist.all_to_all_single(recv_w, send_w, recv_splits, send_splits, group=group)
    recv_o = torch.empty((n_recv, shape.L), dtype=torch.float32, device=dev)
    if n_recv:
        layer.ep_experts(recv_rows, recv_w, recv_counts.reshape(-1).contiguous(), world, recv_o)
    send_o = torch.empty((A, shape.L), dtype=torch.float32, device=dev)
    dist.all_to_all_single(send_o, recv_o, send_splits, recv_splits, group=group)
    y = torch.empty((T, shape.H), dtype=torch.float32, device=dev)
    layer.ep_back(send_o, y)
    return y
