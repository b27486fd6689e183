"""Seeded synthetic inputs for an MoE layer, shared by the CUDA path's tests/bench
and by the oracle.

Recipe (the same for every workload):
  * every tensor (and every expert slice of an expert-weight tensor) is drawn
    from its own counter-based Philox stream, keyed by (seed, stream id), with
    numpy's standard-normal sampler in float32;
  * x ~ N(0, 1); router W_r ~ N(0, 1/d); W1, W3 ~ N(0, 1/d); W2 ~ N(0, 1/f)
    (the standard deviation 1/sqrt(fan_in) is applied in float32);
  * for bf16 workloads the float32 draws of x and of the expert weights are
    rounded to bf16 (round to nearest, ties to even); the router weights and
    the router bias stay float32 (the router runs in fp32);
  * the optional router bias is the workload's fixed per-expert pattern.

This module holds no routing, softmax, top-k, dispatch or FFN arithmetic: it
only produces input bytes.  bf16 tensors are returned as uint16 bit patterns.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass
from typing import Optional

import numpy as np

from .configs import Workload

# stream ids: tensor id in the high bits, expert index in the low 20 bits
_X, _WR, _W1, _W3, _W2, _WS1, _WS3, _WS2, _LOGITS, _SELBIAS = range(1, 11)


def _stream(tensor_id: int, sub: int = 0) -> int:
    return (tensor_id << 20) | sub


def normal_f32(seed: int, stream: int, shape) -> np.ndarray:
    """float32 N(0,1) draws from the Philox stream keyed by (seed, stream)."""
    g = np.random.Generator(np.random.Philox(key=[seed & (2**64 - 1), stream]))
    return g.standard_normal(shape, dtype=np.float32)


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even); return uint16 bits.

    Inputs are finite normal-distribution draws, so no NaN/Inf handling is needed.
    """
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    rounded = u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return (rounded >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _threads() -> int:
    return max(1, min(32, os.cpu_count() or 1))


def _expert_tensor(seed, tensor_id, n_exp, rows, cols, scale, bf16, pool):
    out = np.empty((n_exp, rows, cols), dtype=np.uint16 if bf16 else np.float32)

    def one(e):
        a = normal_f32(seed, _stream(tensor_id, e), (rows, cols))
        a *= np.float32(scale)
        out[e] = f32_to_bf16_bits(a) if bf16 else a

    list(pool.map(one, range(n_exp)))
    return out


@dataclass
class LayerInputs:
    """Host copies of one layer's inputs.  bf16 arrays hold uint16 bit patterns."""
    x: np.ndarray                 # [T, d]
    w_router: np.ndarray          # [d, N] float32
    bias: Optional[np.ndarray]    # [N] float32 or None
    w1: np.ndarray                # [N, d, f]
    w3: np.ndarray                # [N, d, f]
    w2: np.ndarray                # [N, f, d]
    ws1: Optional[np.ndarray] = None  # [d, f_shared]
    ws3: Optional[np.ndarray] = None  # [d, f_shared]
    ws2: Optional[np.ndarray] = None  # [f_shared, d]
    bf16: bool = True


def router_bias(w: Workload) -> Optional[np.ndarray]:
    if w.bias_pattern is None:
        return None
    beta, gamma = w.bias_beta_gamma
    return np.array([a * beta + b * gamma for (a, b) in w.bias_pattern], dtype=np.float32)


def make_x(w: Workload, T: Optional[int] = None) -> np.ndarray:
    T = w.T if T is None else T
    x = normal_f32(w.seed, _stream(_X), (T, w.d))
    return f32_to_bf16_bits(x) if w.dtype == "bf16" else x


def make_router(w: Workload) -> np.ndarray:
    a = normal_f32(w.seed, _stream(_WR), (w.d, w.N))
    a *= np.float32(1.0 / np.sqrt(w.d))
    return a


def make_inputs(w: Workload, T: Optional[int] = None, experts: bool = True) -> LayerInputs:
    """All inputs of workload `w` (optionally with a different token count T).

    experts=False skips the expert weights (for routing-only uses).
    """
    bf16 = w.dtype == "bf16"
    x = make_x(w, T)
    wr = make_router(w)
    bias = router_bias(w)
    if not experts:
        empty = np.zeros((0,), dtype=np.uint16 if bf16 else np.float32)
        return LayerInputs(x, wr, bias, empty, empty, empty, bf16=bf16)
    with ThreadPoolExecutor(_threads()) as pool:
        s_d = 1.0 / np.sqrt(w.d)
        s_f = 1.0 / np.sqrt(w.f)
        w1 = _expert_tensor(w.seed, _W1, w.N, w.d, w.f, s_d, bf16, pool)
        w3 = _expert_tensor(w.seed, _W3, w.N, w.d, w.f, s_d, bf16, pool)
        w2 = _expert_tensor(w.seed, _W2, w.N, w.f, w.d, s_f, bf16, pool)
        ws1 = ws3 = ws2 = None
        if w.f_shared:
            s_fs = 1.0 / np.sqrt(w.f_shared)
            ws1 = _expert_tensor(w.seed, _WS1, 1, w.d, w.f_shared, s_d, bf16, pool)[0]
            ws3 = _expert_tensor(w.seed, _WS3, 1, w.d, w.f_shared, s_d, bf16, pool)[0]
            ws2 = _expert_tensor(w.seed, _WS2, 1, w.f_shared, w.d, s_fs, bf16, pool)[0]
    return LayerInputs(x, wr, bias, w1, w3, w2, ws1, ws3, ws2, bf16=bf16)


def make_logits(seed: int, T: int, N: int, pattern: str = "normal") -> np.ndarray:
    """Synthetic fp32 router logits [T, N] for the routing test entry point.

    pattern:
      "normal"  - i.i.d. N(0,1)
      "ties"    - small integers in [-2, 2], so many exact ties
      "onehot"  - every token strongly prefers expert 0 (one over-full expert)
      "zeros"   - all logits equal (every position ties)
      "skewed"  - N(0,1) plus a per-expert offset ramp (ragged expert loads)
    """
    if pattern == "normal":
        return normal_f32(seed, _stream(_LOGITS, 0), (T, N))
    if pattern == "ties":
        g = normal_f32(seed, _stream(_LOGITS, 1), (T, N))
        return np.clip(np.rint(g * 1.5), -2, 2).astype(np.float32)
    if pattern == "onehot":
        g = normal_f32(seed, _stream(_LOGITS, 2), (T, N)) * np.float32(0.1)
        g[:, 0] += np.float32(10.0)
        return g
    if pattern == "zeros":
        return np.zeros((T, N), dtype=np.float32)
    if pattern == "skewed":
        g = normal_f32(seed, _stream(_LOGITS, 3), (T, N))
        g += np.linspace(2.0, -2.0, N, dtype=np.float32)[None, :]
        return g
    raise ValueError(pattern)


def make_selection_bias(seed: int, N: int, pattern: str = "normal") -> np.ndarray:
    """Synthetic fp32 per-expert selection bias [N] (Aux-Loss-Free routing).

    pattern:
      "normal"  - N(0, 0.5^2)
      "dyadic"  - multiples of 1/4 in [-1, 1] (exact sums with the "ties" logits,
                  so biased scores tie too)
      "zeros"   - all zero (must route exactly as without a bias)
    """
    if pattern == "normal":
        return normal_f32(seed, _stream(_SELBIAS, 0), (N,)) * np.float32(0.5)
    if pattern == "dyadic":
        b = normal_f32(seed, _stream(_SELBIAS, 1), (N,))
        return (np.clip(np.rint(b * 2.0), -4, 4) / 4.0).astype(np.float32)
    if pattern == "zeros":
        return np.zeros((N,), dtype=np.float32)
    raise ValueError(pattern)
