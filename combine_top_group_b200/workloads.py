"""Seeded synthetic workloads for MoE expert-parallel dispatch / combine.

This module only describes workloads and draws their random inputs. It holds
none of the method's arithmetic (no routing, layout, quantisation or combine),
so both the CUDA path and the CPU oracle can take their inputs from it without
sharing any code with each other.

The five workloads mirror the shapes the DeepEP pages talk about:
- the low-latency decode shape is 128 tokens per rank over 8 EP ranks
  (DeepEP summary page, low-latency evaluation section);
- the intranode normal-mode prefill shape is a large batch
  (DeepEP notes page, "计算-通信重叠" and "节点内通信").
Hidden sizes, expert counts, top-k and gating parameters are the usual
DeepSeek-V3 MoE shapes. The pages themselves do not give them.

Input recipe:
- x ~ N(0, 1), drawn in fp32 from a seeded torch.Generator, then rounded to
  bf16 by torch (round to nearest even);
- router logits ~ N(0, 1), fp32, from a second, independent stream;
- the skewed workload adds the bias b_e = -s * ln(e + 1) to every logit
  column, with s = 1.2. The hottest experts then have the lowest ids and sit
  on emulated rank 0.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np
import torch

ROUTE_SOFTMAX = 0
ROUTE_SOFTMAX_RENORM = 1
ROUTE_GROUP_SIGMOID = 2

ROUTE_NAMES = {
    ROUTE_SOFTMAX: "softmax",
    ROUTE_SOFTMAX_RENORM: "softmax_renorm",
    ROUTE_GROUP_SIGMOID: "group_sigmoid",
}


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    R: int            # emulated EP ranks
    T: int            # tokens per rank
    H: int            # hidden size
    E: int            # experts
    K: int            # top-k
    G: int = 1        # expert groups (1 = no group limit)
    KG: int = 1       # groups kept per token
    route: int = ROUTE_SOFTMAX
    fp8: bool = False         # FP8 e4m3 dispatch with per-128-channel scales
    zipf_s: float = 0.0       # logit bias exponent (0 = none)
    mask_frac: float = 0.0    # fraction of top-k slots masked to -1
    mask_seed: int = 0x5EED
    low_latency: bool = False  # fixed (expert, source rank) receive regions of T rows

    @property
    def N(self) -> int:
        return self.R * self.T

    @property
    def L(self) -> int:
        return self.E // self.R

    def describe(self) -> str:
        fmt = "fp8" if self.fp8 else "bf16"
        grp = f" G{self.G}/KG{self.KG}" if self.G > 1 else ""
        extra = ""
        if self.zipf_s:
            extra += f" zipf{self.zipf_s}"
        if self.mask_frac:
            extra += f" mask{self.mask_frac}"
        if self.low_latency:
            extra += " low-latency-layout"
        return (f"{self.name} {self.R}x{self.T} H{self.H} E{self.E} top{self.K}{grp} "
                f"{ROUTE_NAMES[self.route]} {fmt}{extra}")

    def with_tokens(self, T: int) -> "Workload":
        return dataclasses.replace(self, T=T)


WORKLOADS = {
    "tiny": Workload("tiny", R=4, T=128, H=1024, E=16, K=4, route=ROUTE_SOFTMAX),
    "decode": Workload("decode", R=8, T=128, H=7168, E=256, K=8,
                       route=ROUTE_SOFTMAX_RENORM, fp8=True),
    "decode_ll": Workload("decode_ll", R=8, T=128, H=7168, E=256, K=8,
                          route=ROUTE_SOFTMAX_RENORM, fp8=True, low_latency=True),
    "prefill": Workload("prefill", R=8, T=4096, H=7168, E=256, K=8, G=8, KG=4,
                        route=ROUTE_GROUP_SIGMOID),
    "skewed": Workload("skewed", R=8, T=4096, H=4096, E=64, K=6,
                       route=ROUTE_SOFTMAX, fp8=True, zipf_s=1.2, mask_frac=0.05),
    "large": Workload("large", R=8, T=16384, H=7168, E=256, K=8, G=8, KG=4,
                      route=ROUTE_GROUP_SIGMOID, fp8=True),
}

SEEDS = (0, 1, 2)


def _gen(seed: int, stream: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed((seed * 1_000_003 + stream) & 0x7FFF_FFFF_FFFF_FFFF)
    return g


def make_logits(w: Workload, seed: int) -> np.ndarray:
    """Router logits, fp32 [N, E], row-major."""
    g = _gen(seed, 1)
    logits = torch.randn(w.N, w.E, generator=g, dtype=torch.float32)
    if w.zipf_s:
        bias = torch.tensor([-w.zipf_s * math.log(e + 1.0) for e in range(w.E)],
                            dtype=torch.float32)
        logits = logits + bias
    return logits.numpy()


def make_x(w: Workload, seed: int, rows: slice | None = None) -> np.ndarray:
    """Token hidden states as bf16 bit patterns, uint16 [N, H], row-major.

    The whole matrix is drawn in fixed blocks of 1024 rows. Block b uses its own
    generator stream, so a sub-range of rows can be made without drawing the
    rest.
    """
    blk = 1024
    lo, hi = (0, w.N) if rows is None else (rows.start or 0, rows.stop if rows.stop is not None else w.N)
    out = np.empty((hi - lo, w.H), dtype=np.uint16)
    b0, b1 = lo // blk, (hi + blk - 1) // blk
    for b in range(b0, b1):
        r0, r1 = b * blk, min((b + 1) * blk, w.N)
        g = _gen(seed, 1000 + b)
        blockx = torch.randn(r1 - r0, w.H, generator=g, dtype=torch.float32).to(torch.bfloat16)
        bits = blockx.view(torch.int16).numpy().view(np.uint16)
        s0, s1 = max(lo, r0), min(hi, r1)
        out[s0 - lo:s1 - lo] = bits[s0 - r0:s1 - r0]
    return out


def make_topk_idx_skew_all(w: Workload) -> np.ndarray:
    """Extreme skew edge case: every token picks experts 0..K-1 (all on rank 0
    when K <= E/R)."""
    idx = np.tile(np.arange(w.K, dtype=np.int32), (w.N, 1))
    return idx


def make_uniform_weights(w: Workload) -> np.ndarray:
    return np.full((w.N, w.K), 1.0 / w.K, dtype=np.float32)
