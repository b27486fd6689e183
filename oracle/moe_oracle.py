"""fp64 CPU oracle for the forward pass of one Mixture-of-Experts layer.

TEST INFRASTRUCTURE.  Only the tests, the smoke check of the build entry and the
CPU-baseline / reference leg of the benchmark may import this module.  The
product path (the CUDA library and its Python binding) never imports, calls or
links anything here, and nothing here imports the product path: the oracle and
the CUDA path share no code.  Inputs are plain numpy arrays (bf16 tensors as
uint16 bit patterns, exactly as the seeded input generator produces them).

What is computed, in the pages' order and notation:

  1. router logits  g(x) = x W_r (+ b)           "MoE 训练加速实战：DeepEP + Grouped
     GeMM + Aux-Loss-Free" §2.2 "Router 数学"; the optional fixed bias b is the
     skewed-load workload's per-expert offset.
  2. scores = softmax(g(x)), computed with the maximum subtracted   (§2.2; the
     router is kept in fp32 against softmax 0/0 NaN, §1 pain point 4 / §9.2).
  3. top-k of g(x) and the renormalised weights  s_i / sum_{j in top-k} s_j
     (§2.2, the TopK formula).
  4. capacity C = ceil(capacity_factor * T * k / N) and the drop of overflow
     assignments ("负载均衡策略：MoE训练稳定性保障", section "专家容量裁剪",
     worked example 1024 tokens / 8 experts / factor 1.25 -> 160).
  5. permutation of kept assignments into expert-contiguous rows ("ETP专家并行
     加速MoE模型" section "动态路由下的高效通信": tokens are re-shuffled to their
     experts).
  6. per-expert SwiGLU FFN  y_i = W_i x_i over each expert's rows (§4.2
     "数学等价性" of the first page above: grouped GEMM == one GEMM per expert).
  7. weighted combine  y = sum_j w_j Expert_{idx_j}(x)  (§2.2 formula, §2.1
     "权重加和").
  8. load-balance statistics y_i (token fraction), z_i (mean gate score) and
     L_aux = (N_tok/E) sum y_i z_i ("负载均衡策略" section "辅助损失函数"), plus the
     Switch form N_exp * sum f_i P_i (§5.2 "传统方案：Auxiliary Loss").
  9. Aux-Loss-Free routing: a per-expert bias b added to g for the top-k choice
     only, and its update b_i <- b_i + gamma sign(1/N - f_i) (§5.3-5.4 of the
     first page).
 10. router z-loss and the load-health figures (load std, top-2 share, tokens
     per expert) ("负载均衡策略", hyper-parameter table, z_loss_weight; §9.1 of
     the first page; "ms-swift + Megatron：MoE模型加速10倍实测" §3.3 "监控与诊断").

Readings taken where the pages are silent or ambiguous (each also listed in the
design notes):
  (i)   top-k selects on the logits g, not on the softmax scores (the §2.2 formula
        writes top-k(g(x)); softmax is monotone so the set is the same in exact
        arithmetic);
  (ii)  ties go to the lower expert index; slots are ordered by descending logit;
  (iii) the expert FFN is SwiGLU: h = silu(x W1) * (x W3), o = h W2, with
        silu(u) = u / (1 + exp(-u)); in bf16 mode h is rounded to bf16 before W2
        (the stated bf16-compute / fp32-accumulate mixed precision);
  (iv)  C = ceil(capacity_factor * T * k / N), evaluated exactly on the given
        double capacity_factor (the §"专家容量裁剪" example fixes the k = 1 case);
  (v)   overflow is dropped in token-index order within each expert (the earliest
        C assignments are kept); no re-routing; kept weights are NOT renormalised;
  (vi)  both L_aux forms are reported (the two pages use N for different things);
  (vii) y_i counts the top-k selections before the capacity drop, over T*k;
  (viii) z_i is the mean of the full softmax score over all T tokens;
  (ix)  the shared expert is added with weight 1 after the routed sum;
  (x)   segment starts are rounded up to `align` rows (a layout choice that the
        oracle takes as a parameter).
  (xi)  the selection bias is added to the fp32 logits in fp32; the weights and
        z_i come from the unbiased softmax; f_i in the bias update counts the
        top-k selections before the capacity drop;
  (xii) the z-loss is the mean over tokens of (logsumexp_i g_ti)^2, the squared
        log-partition of the router (the pages call it an L2 penalty on the
        gate logits and give only its weight);
  (xiii) the load figures follow the readings stated in load_metrics.
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from fractions import Fraction
from typing import Dict, Optional, Sequence

import numpy as np


# ----------------------------------------------------------------------------
# number formats
# ----------------------------------------------------------------------------

def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> exact fp64 values (a bf16 is the top half of an fp32)."""
    u32 = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u32.view(np.float32).astype(np.float64)


def as_f64(a: np.ndarray) -> np.ndarray:
    """Input tensor (uint16 bf16 bits, float32 or float64) -> fp64 values."""
    a = np.asarray(a)
    if a.dtype == np.uint16:
        return bf16_bits_to_f64(a)
    return a.astype(np.float64)


def round_to_bf16(v: np.ndarray) -> np.ndarray:
    """Round fp64 values to the nearest bf16 value (ties to even), returned as fp64.

    bf16 keeps 8 significant bits.  Writing v = m * 2**e with 0.5 <= |m| < 1, the
    spacing of bf16 values near v is 2**(e - 8) for normal numbers and 2**-133 in
    the subnormal range (|v| < 2**-126).  np.rint rounds half to even.
    """
    v = np.asarray(v, dtype=np.float64)
    _, e = np.frexp(v)
    e = np.maximum(e, -125)              # below 2**-126 the spacing stays 2**-133
    q = np.ldexp(1.0, e - 8)
    return np.rint(v / q) * q


# ----------------------------------------------------------------------------
# steps 1-3: router, softmax, top-k and renormalised weights
# ----------------------------------------------------------------------------

def router_logits(x: np.ndarray, w_router: np.ndarray,
                  bias: Optional[np.ndarray] = None) -> np.ndarray:
    """g = x W_r (+ b) in fp64.  x [T, d] (bf16 bits or fp32), W_r [d, N] fp32."""
    g = as_f64(x) @ as_f64(w_router)
    if bias is not None:
        g = g + as_f64(bias)[None, :]
    return g


def softmax(g: np.ndarray) -> np.ndarray:
    """scores = softmax(g) per token, with the per-token maximum subtracted."""
    g = np.asarray(g, dtype=np.float64)
    z = np.exp(g - g.max(axis=1, keepdims=True))
    return z / z.sum(axis=1, keepdims=True)


def topk(g: np.ndarray, k: int, selection_bias: Optional[np.ndarray] = None) -> np.ndarray:
    """Indices of the k largest logits per token, in descending order.

    Equal logits are ordered by the lower expert index first: a stable sort of
    -g keeps equal keys in index order.  Returns int32 [T, k].

    With a selection bias b (Aux-Loss-Free balancing, "MoE 训练加速实战" §5.3:
    a per-expert offset that only steers the top-k choice) the experts are
    ranked on g + b.  That sum is formed in fp32, the precision in which the
    GPU takes the same decision; the weights are unaffected (topk_weights uses
    the unbiased scores).
    """
    g = np.asarray(g, dtype=np.float64)
    if selection_bias is not None:
        g = (g.astype(np.float32) + np.asarray(selection_bias, np.float32)[None, :]).astype(np.float64)
    order = np.argsort(-g, axis=1, kind="stable")
    return order[:, :k].astype(np.int32)


def bias_update(selection_bias: np.ndarray, counts: np.ndarray, T: int, k: int,
                gamma: float) -> np.ndarray:
    """One Aux-Loss-Free step ("MoE 训练加速实战" §5.4):
    b_i <- b_i + gamma * sign(1/N - f_i), with f_i = counts_i / (T k) the share
    of the batch's top-k assignments that expert i received (before the
    capacity drop).  The sign is taken exactly, as sign(T k - N counts_i); the
    update is one fp32 addition (b_i and gamma are fp32)."""
    counts = np.asarray(counts, dtype=np.int64)
    N = counts.shape[0]
    sgn = np.sign(T * k - N * counts).astype(np.float32)
    return np.asarray(selection_bias, np.float32) + np.float32(gamma) * sgn


def router_z_loss(g: np.ndarray) -> float:
    """Router z-loss: the mean over tokens of (log sum_i exp g_ti)^2.  The pages
    name it as an L2 penalty on the gate logits that keeps them from growing
    ("负载均衡策略：MoE训练稳定性保障", hyper-parameter table, z_loss_weight, and
    section "常见问题"; "MoE 训练加速实战" §9.1 router_z_loss); the penalised
    quantity is the log-partition z = logsumexp(g) of each token."""
    g = np.asarray(g, dtype=np.float64)
    if g.shape[0] == 0:
        return 0.0
    m = g.max(axis=1)
    lse = m + np.log(np.exp(g - m[:, None]).sum(axis=1))
    return float(np.mean(lse ** 2))


def topk_weights(s: np.ndarray, idx: np.ndarray) -> np.ndarray:
    """w[t, j] = s[t, idx[t, j]] / sum_j' s[t, idx[t, j']]  (fp64)."""
    sel = np.take_along_axis(s, idx.astype(np.int64), axis=1)
    return sel / sel.sum(axis=1, keepdims=True)


# ----------------------------------------------------------------------------
# steps 4-5: capacity, drop and permutation
# ----------------------------------------------------------------------------

def capacity(capacity_factor: float, T: int, k: int, N: int) -> int:
    """C = ceil(capacity_factor * T * k / N), exact on the given double."""
    return int(math.ceil(Fraction(capacity_factor) * T * k / N))


@dataclass
class Dispatch:
    counts: np.ndarray    # [N] int32, assignments per expert before the drop
    kept: np.ndarray      # [N] int32, min(counts, C)
    seg_off: np.ndarray   # [N+1] int32, segment starts (rounded up to align)
    row_map: np.ndarray   # [T, k] int32, row in the permuted buffer or -1 (dropped)
    rank: np.ndarray      # [T, k] int32, position of the assignment in its expert's queue
    num_dropped: int


def dispatch(idx: np.ndarray, N: int, C: int, align: int = 128) -> Dispatch:
    """Capacity clip in token-index order, then expert-contiguous row numbering.

    Each expert's queue is walked in token order t = 0..T-1; the assignment gets
    the number of earlier assignments to the same expert as its rank, and is kept
    iff rank < C.  Segment e starts at the sum of the kept counts of experts
    0..e-1, each rounded up to a multiple of `align`.
    """
    T, k = idx.shape
    counts = np.zeros(N, dtype=np.int64)
    rank = np.zeros((T, k), dtype=np.int64)
    for t in range(T):
        for j in range(k):
            e = int(idx[t, j])
            rank[t, j] = counts[e]
            counts[e] += 1
    kept = np.minimum(counts, C)
    seg_off = np.zeros(N + 1, dtype=np.int64)
    for e in range(N):
        seg_off[e + 1] = seg_off[e] + (kept[e] + align - 1) // align * align
    row_map = np.full((T, k), -1, dtype=np.int64)
    for t in range(T):
        for j in range(k):
            e = int(idx[t, j])
            if rank[t, j] < C:
                row_map[t, j] = seg_off[e] + rank[t, j]
    return Dispatch(counts.astype(np.int32), kept.astype(np.int32),
                    seg_off.astype(np.int32), row_map.astype(np.int32),
                    rank.astype(np.int32), int(counts.sum() - kept.sum()))


def permuted_rows(x: np.ndarray, disp: Dispatch) -> Dict[int, np.ndarray]:
    """The permuted buffer as {row: copy of x[t]} for every kept assignment."""
    rows = {}
    T, k = disp.row_map.shape
    for t in range(T):
        for j in range(k):
            r = int(disp.row_map[t, j])
            if r >= 0:
                rows[r] = x[t]
    return rows


# ----------------------------------------------------------------------------
# steps 6-7: SwiGLU experts and the weighted combine
# ----------------------------------------------------------------------------

def silu(u: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):
        return u / (1.0 + np.exp(-u))


def swiglu_ffn(x64: np.ndarray, w1: np.ndarray, w3: np.ndarray, w2: np.ndarray,
               round_h_bf16: bool) -> np.ndarray:
    """Rows of x (fp64, [n, d]) through one SwiGLU expert: (silu(x W1) * x W3) W2."""
    h = silu(x64 @ as_f64(w1)) * (x64 @ as_f64(w3))
    if round_h_bf16:
        h = round_to_bf16(h)
    return h @ as_f64(w2)


# ----------------------------------------------------------------------------
# step 8: load-balance statistics
# ----------------------------------------------------------------------------

@dataclass
class AuxStats:
    y_frac: np.ndarray    # [N] fraction of the T*k top-k selections per expert
    z_mean: np.ndarray    # [N] mean softmax score per expert over the T tokens
    l_aux_p3: float       # (T / N) * sum_i y_i z_i   (tokens over experts)
    l_aux_switch: float   # N * sum_i y_i z_i          (experts)


def aux_stats(idx: np.ndarray, s: np.ndarray, N: int) -> AuxStats:
    T, k = idx.shape
    if T == 0:
        z = np.zeros(N)
        return AuxStats(z, z.copy(), 0.0, 0.0)
    counts = np.bincount(idx.reshape(-1).astype(np.int64), minlength=N).astype(np.float64)
    y = counts / (T * k)
    z = s.mean(axis=0)
    yz = float(np.sum(y * z))
    return AuxStats(y, z, (T / N) * yz, N * yz)


@dataclass
class LoadMetrics:
    load_std: float               # population std over experts of f_i = counts_i / (T k)
    top2_ratio: float             # share of the T k selections taken by the two busiest experts
    avg_tokens_per_expert: float  # rows the experts process, sum_i kept_i, over N


def load_metrics(counts: np.ndarray, kept: np.ndarray, T: int, k: int) -> LoadMetrics:
    """The three load-health figures of "ms-swift + Megatron：MoE模型加速10倍实测"
    §3.3 "监控与诊断" (expert load std, top2_expert_ratio, avg_tokens_per_expert).

    Readings: the load of expert i is its share f_i of the batch's T k top-k
    selections (before the capacity drop) and the std is the population one
    (over the N experts); top2_expert_ratio is the share of the selections
    that the two most selected experts received (2/N when balanced, the page's
    0.25 for 8 experts); avg_tokens_per_expert counts the rows an expert
    actually processes, i.e. the kept assignments, averaged over the N experts.
    An empty batch gives zeros.
    """
    counts = np.asarray(counts, dtype=np.int64)
    kept = np.asarray(kept, dtype=np.int64)
    N = counts.shape[0]
    if T == 0:
        return LoadMetrics(0.0, 0.0, 0.0)
    f = counts / float(T * k)
    load_std = float(np.sqrt(np.mean((f - f.mean()) ** 2)))
    top = np.sort(counts)[::-1][:2]
    top2 = float(top.sum()) / float(T * k)
    return LoadMetrics(load_std, top2, float(kept.sum()) / float(N))


# ----------------------------------------------------------------------------
# the whole layer
# ----------------------------------------------------------------------------

@dataclass
class LayerResult:
    logits: np.ndarray            # [T, N] fp64 (or the given logits)
    scores: np.ndarray            # [T, N] fp64 softmax
    idx: np.ndarray               # [T, k] int32
    w: np.ndarray                 # [T, k] fp64 renormalised weights
    capacity: int
    disp: Dispatch
    stats: AuxStats
    tokens: np.ndarray            # token ids whose outputs are in y
    y: np.ndarray                 # [len(tokens), d] fp64


def layer_forward(x: np.ndarray, w_router: np.ndarray, bias: Optional[np.ndarray],
                  w1: np.ndarray, w3: np.ndarray, w2: np.ndarray, k: int,
                  capacity_factor: float = 1.0, cap: Optional[int] = None,
                  bf16: bool = True, ws1=None, ws3=None, ws2=None, align: int = 128,
                  tokens: Optional[Sequence[int]] = None,
                  logits: Optional[np.ndarray] = None,
                  selection_bias: Optional[np.ndarray] = None) -> LayerResult:
    """Forward pass of one MoE layer.

    Routing and dispatch always cover all T tokens (the capacity clip depends on
    every earlier token); the expert FFN and combine are evaluated for `tokens`
    (default: all).  `logits`, if given, replaces step 1 (routing-parity mode).
    `selection_bias` (Aux-Loss-Free routing) steers only the top-k choice.
    """
    T = x.shape[0]
    N = w_router.shape[1]
    g = router_logits(x, w_router, bias) if logits is None else np.asarray(logits, np.float64)
    s = softmax(g) if T else np.zeros((0, N))
    idx = topk(g, k, selection_bias) if T else np.zeros((0, k), np.int32)
    w = topk_weights(s, idx) if T else np.zeros((0, k))
    C = capacity(capacity_factor, T, k, N) if cap is None else int(cap)
    disp = dispatch(idx, N, C, align)
    stats = aux_stats(idx, s, N)

    tok = np.arange(T) if tokens is None else np.asarray(tokens, dtype=np.int64)
    d = x.shape[1]
    y = np.zeros((len(tok), d))
    if len(tok):
        x64 = as_f64(x[tok])
        sub_idx = idx[tok]
        sub_kept = disp.row_map[tok] >= 0
        o = np.zeros((len(tok), k, d))
        for e in range(N):
            ti, tj = np.nonzero((sub_idx == e) & sub_kept)
            if len(ti):
                o[ti, tj] = swiglu_ffn(x64[ti], w1[e], w3[e], w2[e], bf16)
        for j in range(k):                       # y = sum_j w_j o_j, slot order
            y += np.where(sub_kept[:, j:j + 1], w[tok, j:j + 1] * o[:, j], 0.0)
        if ws1 is not None:
            y += swiglu_ffn(x64, ws1, ws3, ws2, bf16)
    return LayerResult(g, s, idx, w, C, disp, stats, tok, y)


def rel_frobenius(a: np.ndarray, b: np.ndarray) -> float:
    """||a - b||_F / ||b||_F  (0 when both are zero)."""
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    nb = np.linalg.norm(b)
    na = np.linalg.norm(a - b)
    return float(na / nb) if nb > 0 else float(na)
