"""Calibrate the fixed router bias of the skewed-stress workload (test infrastructure).

"ms-swift + Megatron：MoE模型加速10倍实测" §2.1 reports a skewed top-2 router:
experts 0 and 3 take 68% of the tokens while experts 5 and 6 sit near idle
(< 3%).  The skewed-stress workload reproduces that load with a fixed bias
b = (beta, 0, 0, beta, 0, -gamma, -gamma, 0) added to the router logits.  This
script finds (beta, gamma) by bisection on the seed-0 logits computed by the
oracle, so that the {0,3} share of the T*k assignments is 68% (+-1%) and the
{5,6} share is about 2%.  beta and gamma are rounded to multiples of 2**-10 so
that they are exact in fp32.

Usage:  python -m oracle.calibrate_skew      (prints the pair and the shares)
"""
from __future__ import annotations

import numpy as np

from expert_router_gemm_b200 import configs, synth
from oracle import moe_oracle as orc


def shares(g0: np.ndarray, k: int, beta: float, gamma: float):
    w = configs.SKEW
    b = np.array([a * beta + c * gamma for (a, c) in w.bias_pattern])
    idx = orc.topk(g0 + b[None, :], k)
    counts = np.bincount(idx.reshape(-1), minlength=w.N) / idx.size
    return counts[0] + counts[3], counts[5] + counts[6], counts


def bisect(fn, lo, hi, target, increasing=True, iters=40):
    for _ in range(iters):
        mid = 0.5 * (lo + hi)
        v = fn(mid)
        if (v < target) == increasing:
            lo = mid
        else:
            hi = mid
    return 0.5 * (lo + hi)


def calibrate():
    w = configs.SKEW
    inp = synth.make_inputs(w, experts=False)
    g0 = orc.router_logits(inp.x, inp.w_router, None)
    beta, gamma = 0.0, 0.0
    for _ in range(8):
        beta = bisect(lambda b: shares(g0, w.k, b, gamma)[0], 0.0, 8.0, 0.68, True)
        gamma = bisect(lambda c: shares(g0, w.k, beta, c)[1], 0.0, 8.0, 0.02, False)
    q = 2.0 ** -10
    beta, gamma = round(beta / q) * q, round(gamma / q) * q
    s03, s56, counts = shares(g0, w.k, beta, gamma)
    return beta, gamma, s03, s56, counts


if __name__ == "__main__":
    beta, gamma, s03, s56, counts = calibrate()
    print(f"SKEW_BETA_GAMMA = ({beta!r}, {gamma!r})")
    print(f"share(0,3) = {s03:.4f}  share(5,6) = {s56:.4f}")
    print("per-expert shares:", np.round(counts, 4).tolist())
