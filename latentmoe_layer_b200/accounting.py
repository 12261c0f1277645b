"""Algorithmic work of one LatentMoE layer forward (FLOPs, parameters, bytes).

These are the counts the roofline numbers divide by. They count only the work
the method must do: selected experts only, no padding, no re-reads.

FLOPs per token (a multiply-add counts 2):
  routing        2 H E           (router linear; "Nemotron 3 Ultra 架构 QA", Q3.1)
  latent proj    4 H L           (fc1 H->L and fc2 L->H)
  experts        4 k L I         (k x (up L->I + down I->L))
  shared expert  4 H Is          (up H->Is + down Is->H)
"""
from __future__ import annotations


def flops_breakdown(w) -> dict:
    return {
        "routing": 2.0 * w.H * w.E,
        "latent_proj": 4.0 * w.H * w.L,
        "experts": 4.0 * w.k * w.L * w.I,
        "shared": 4.0 * w.H * w.Is,
    }


def flops_per_token(w) -> float:
    return sum(flops_breakdown(w).values())


def params(w) -> dict:
    return {
        "per_expert": 2.0 * w.L * w.I,
        "experts_per_layer": 2.0 * w.E * w.L * w.I,
        "latent_proj": 2.0 * w.H * w.L,
        "shared": 2.0 * w.H * w.Is,
        "router": 1.0 * w.E * w.H,
    }


def dense_weight_bytes(w) -> float:
    """bf16 bytes of the weights every call reads: router, fc1, fc2, shared up/down (+ fp32 bias)."""
    return 2.0 * (w.E * w.H + 2 * w.H * w.L + 2 * w.H * w.Is) + 4.0 * w.E


def expert_bytes(w, distinct_experts: int, nvfp4: bool = False) -> float:
    """Bytes of the expert weights a call must read: every hit expert's up and down once.
    bf16: 2 bytes per weight. NVFP4: half a byte per weight, one E4M3 scale byte per
    16 weights and one fp32 matrix scale per matrix."""
    if nvfp4:
        return distinct_experts * 2 * (w.L * w.I * (0.5 + 1.0 / 16) + 4.0)
    return 2.0 * distinct_experts * 2 * w.L * w.I


def io_bytes(w, x_bytes_per_elem: int = 2) -> float:
    """Layer input x and fp32 output y."""
    return w.T * w.H * (x_bytes_per_elem + 4.0)


def min_bytes_per_call(w, distinct_experts: int, nvfp4: bool = False) -> float:
    """Compulsory HBM traffic of one call: weights touched once plus x and y."""
    return dense_weight_bytes(w) + expert_bytes(w, distinct_experts, nvfp4) + io_bytes(w, 4 if w.x_f32 else 2)
