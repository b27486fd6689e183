"""The five MoE-layer workload shapes this library is tested and benchmarked on.

Shapes follow the model families that "MoE 训练加速实战：DeepEP + Grouped GeMM +
Aux-Loss-Free" lists in its §2.3 spec table (Mixtral 8x7B: 8 experts, top-2;
Qwen3-MoE: 128 experts, top-8; DeepSeek-V3: 256 experts, top-8 plus one shared
expert).  Hidden sizes are not given on the pages; the ones below are the public
model shapes.  The skewed layer reproduces the load skew reported in
"ms-swift + Megatron：MoE模型加速10倍实测" §2.1 (experts 0 and 3 take 68% of
the tokens, experts 5 and 6 under 3%).

This module holds shapes and input recipes only: no routing or FFN arithmetic.
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace
from typing import Optional, Tuple


@dataclass(frozen=True)
class Workload:
    name: str
    T: int                      # tokens in the batch
    d: int                      # model dimension
    N: int                      # routed experts
    k: int                      # experts per token
    f: int                      # SwiGLU hidden size of one routed expert
    f_shared: int = 0           # hidden size of the always-on shared expert (0: none)
    capacity_factor: float = 1.25
    dtype: str = "bf16"         # activation / expert-weight dtype: "f32" or "bf16"
    # Fixed router bias pattern (per expert), in units of (beta, gamma):
    # entry = a*beta + b*gamma for the pair (a, b).  None: no bias.
    bias_pattern: Optional[Tuple[Tuple[int, int], ...]] = None
    bias_beta_gamma: Tuple[float, float] = (0.0, 0.0)
    seed: int = 0
    description: str = ""

    def scaled(self, T: int) -> "Workload":
        """Same layer with a different token count (for small parity cases)."""
        return replace(self, T=T)

    @property
    def capacity_hint(self) -> str:
        return f"ceil({self.capacity_factor}*{self.T}*{self.k}/{self.N})"


# Skew bias (beta, gamma) for the skewed-stress layer.  Calibrated once on the
# seed-0 router logits by oracle/calibrate_skew.py so that experts {0,3} receive
# 68 +- 1 % of the top-2 assignments and experts {5,6} together < 3 %.
SKEW_BETA_GAMMA = (1.3505859375, 1.0966796875)

TINY = Workload(
    name="tiny-fp32", T=256, d=128, N=8, k=2, f=256, capacity_factor=1.25, dtype="f32",
    description="tiny MoE layer, fp32 throughout")
MIXTRAL = Workload(
    name="mixtral-8x7b-shaped", T=4096, d=4096, N=8, k=2, f=14336, capacity_factor=1.25,
    description="Mixtral-8x7B-shaped layer, batch 2 x seq 2048")
QWEN3 = Workload(
    name="qwen3-moe-shaped", T=8192, d=4096, N=128, k=8, f=1536, capacity_factor=1.0,
    description="Qwen3-MoE-shaped fine-grained layer")
DSV3 = Workload(
    name="deepseek-v3-shaped", T=8192, d=7168, N=256, k=8, f=2048, f_shared=2048,
    capacity_factor=1.25, description="DeepSeek-V3-shaped layer with one shared expert")
SKEW = Workload(
    name="skewed-stress", T=16384, d=2048, N=8, k=2, f=8192, capacity_factor=1.25,
    bias_pattern=((1, 0), (0, 0), (0, 0), (1, 0), (0, 0), (0, -1), (0, -1), (0, 0)),
    bias_beta_gamma=SKEW_BETA_GAMMA,
    description="skewed-load stress layer: experts 0,3 hot, 5,6 cold")

WORKLOADS = {w.name: w for w in (TINY, MIXTRAL, QWEN3, DSV3, SKEW)}
ALIASES = {"tiny": TINY.name, "mixtral": MIXTRAL.name, "qwen3": QWEN3.name,
           "dsv3": DSV3.name, "skew": SKEW.name}


def get(name: str) -> Workload:
    return WORKLOADS[ALIASES.get(name, name)]
