"""Synthetic LatentMoE layer workloads (shapes, distributions, skew recipe).

These are the layer shapes the tests and the benchmark use. Each is seeded
synthetic data; nothing here computes any part of the layer.

Shapes follow the Nemotron-3 family as described on the pages
"Nemotron 3 Ultra 架构 QA" (Q1.1: hidden 4096 / 8192, experts 128 / 512,
active 8 / 22; Q5.6: expert weights [E, I, L] and [E, L, I]) and the
Nemotron-3-Ultra-Math-SFT article ("LatentMoE 层" section: latent 2048,
expert intermediate 5120, shared intermediate 10240, scale 5.0).

Distributions: x ~ N(0, 1); every weight ~ N(0, 0.02) stored as bf16;
e_score_correction_bias ~ U(-0.1, 0.1) fp32; seed 0.

Skew recipe (ultra_skew): experts 0..15 are "hot". Their logit is raised by
+3.0 through the router weights alone, because the router is a bias-free
linear map: x[:, 0] = 1.0 and W_r[hot, 0] = 3.0.
"""
from __future__ import annotations

from dataclasses import dataclass, asdict, replace


@dataclass(frozen=True)
class LayerShape:
    name: str
    T: int          # tokens
    H: int          # hidden size
    L: int          # latent size (moe_latent_size)
    E: int          # routed experts
    k: int          # experts per token
    G: int          # n_group
    Gk: int         # topk_group
    I: int          # expert intermediate size
    Is: int         # shared-expert intermediate size
    s: float = 5.0  # routed_scaling_factor
    x_f32: bool = False    # x is given as fp32 (else bf16)
    skew_hot: int = 0      # number of hot experts (0 = no skew)
    skew_offset: float = 0.0

    def as_dict(self):
        return asdict(self)

    def with_tokens(self, T: int) -> "LayerShape":
        return replace(self, T=T)


TINY = LayerShape("tiny", T=64, H=256, L=64, E=16, k=2, G=1, Gk=1, I=128, Is=256, x_f32=True)
NANO_DECODE = LayerShape("nano_decode", T=128, H=4096, L=2048, E=128, k=8, G=8, Gk=4, I=2560, Is=5120)
ULTRA_DECODE = LayerShape("ultra_decode", T=64, H=8192, L=2048, E=512, k=22, G=8, Gk=4, I=5120, Is=10240)
ULTRA_PREFILL = LayerShape("ultra_prefill", T=16384, H=8192, L=2048, E=512, k=22, G=8, Gk=4, I=5120,
                           Is=10240)
ULTRA_SKEW = LayerShape("ultra_skew", T=8192, H=8192, L=2048, E=512, k=22, G=8, Gk=4, I=5120, Is=10240,
                        skew_hot=16, skew_offset=3.0)

# Profiling stand-in for the Ultra prefill expert GEMMs: the same H, L, I, k and
# the same ~704 rows per expert, but 64 experts (~3 GB of weights) so that a
# multi-pass ncu capture stays small.
PROBE_E64 = LayerShape("probe_e64", T=2048, H=8192, L=2048, E=64, k=22, G=8, Gk=4, I=5120, Is=10240)
# Decode-sized counterpart (64 tokens, ~22 per expert as in ultra_decode's swap-AB
# tiles), 2.7 GB of bf16 expert weights: small enough for a full profiler capture.
PROBE_DECODE_E64 = LayerShape("probe_decode_e64", T=64, H=8192, L=2048, E=64, k=22, G=8, Gk=4, I=5120, Is=10240)

WORKLOADS = {w.name: w for w in (TINY, NANO_DECODE, ULTRA_DECODE, ULTRA_PREFILL, ULTRA_SKEW, PROBE_E64,
                                 PROBE_DECODE_E64)}

# Stream ids of the generator, one per tensor.
TID_X, TID_ROUTER, TID_BIAS, TID_FC1, TID_FC2, TID_UP, TID_DOWN, TID_SUP, TID_SDOWN = range(1, 10)
W_SIGMA = 0.02
BIAS_LO, BIAS_HI = -0.1, 0.1


def tensor_specs(w: LayerShape):
    """(key, tensor id, shape, kind) for every input of the layer.

    kind: 'x' (N(0,1), fp32 or bf16), 'w' (N(0, 0.02) bf16), 'b' (U(-0.1, 0.1) fp32).
    """
    return [
        ("x", TID_X, (w.T, w.H), "x"),
        ("router_w", TID_ROUTER, (w.E, w.H), "w"),
        ("e_bias", TID_BIAS, (w.E,), "b"),
        ("fc1_w", TID_FC1, (w.L, w.H), "w"),
        ("fc2_w", TID_FC2, (w.H, w.L), "w"),
        ("up_w", TID_UP, (w.E, w.I, w.L), "w"),
        ("down_w", TID_DOWN, (w.E, w.L, w.I), "w"),
        ("shared_up_w", TID_SUP, (w.Is, w.H), "w"),
        ("shared_down_w", TID_SDOWN, (w.H, w.Is), "w"),
    ]
