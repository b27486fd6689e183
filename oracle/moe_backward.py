"""fp64 CPU oracle of the backward pass of one MoE layer.

TEST INFRASTRUCTURE, like moe_oracle: only the tests, the smoke check and the
benchmark's CPU legs may use it; it shares no code with the CUDA path.

The pages train MoE layers: the loss is the main loss plus lambda times the
auxiliary load-balance loss ("MoE 训练加速实战：DeepEP + Grouped GeMM +
Aux-Loss-Free" §5.2), plus the router z-loss with its own weight
("负载均衡策略：MoE训练稳定性保障", hyper-parameter table, z_loss_weight; §9.1 of
the first page), and only the experts a token was routed to receive gradient
from it ("ms-swift + Megatron：MoE模型加速10倍实测" §2.3: MoE gradients are
sparse).  This module differentiates the forward pass of moe_oracle (exact
arithmetic, no bf16 rounding of h) for the scalar

    L = <dy, y> + aux_weight * L_aux + z_weight * z_loss

where dy is the upstream gradient of the layer output, L_aux = N sum_i f_i P_i
(the Switch form of §5.2: f_i the share of the T k selections, a count with no
gradient; P_i the mean softmax score) and z_loss = mean_t logsumexp(g_t)^2.
The routing decisions (top-k set, capacity drops) are piecewise constant: their
derivative is zero almost everywhere, so the gradient flows through the
renormalised weights of the chosen experts, the softmax and the router GEMM.

Readings: the selection bias of Aux-Loss-Free routing gets no gradient (§5.3:
b does not take part in gradient updates); a dropped slot contributes nothing to
y, so its weight gets no gradient either; the fixed router bias of the skewed
workload gets the gradient sum_t dg_t like any additive bias.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional, Sequence

import numpy as np

from oracle import moe_oracle as orc


@dataclass
class LayerGrads:
    dx: np.ndarray          # [T, d]
    dw_router: np.ndarray   # [d, N]
    dbias: Optional[np.ndarray]   # [N] or None
    dw1: np.ndarray         # [N, d, f]
    dw3: np.ndarray         # [N, d, f]
    dw2: np.ndarray         # [N, f, d]
    dws1: Optional[np.ndarray]
    dws3: Optional[np.ndarray]
    dws2: Optional[np.ndarray]
    dlogits: np.ndarray     # [T, N] gradient of L with respect to g
    dweights: np.ndarray    # [T, k] gradient with respect to the routing weights


def silu_grad(u: np.ndarray) -> np.ndarray:
    """d/du [u sigma(u)] = sigma(u) (1 + u (1 - sigma(u)))."""
    with np.errstate(over="ignore"):
        sig = 1.0 / (1.0 + np.exp(-u))
    return sig * (1.0 + u * (1.0 - sig))


def expert_backward(x64, w1, w3, w2, dout):
    """One SwiGLU expert o = (silu(x W1) * (x W3)) W2 on rows x64 [n, d], given
    dout = dL/do [n, d]: returns (dx, dW1, dW3, dW2)."""
    W1, W3, W2 = orc.as_f64(w1), orc.as_f64(w3), orc.as_f64(w2)
    g = x64 @ W1
    u = x64 @ W3
    h = orc.silu(g) * u
    dh = dout @ W2.T
    dg = dh * u * silu_grad(g)
    du = dh * orc.silu(g)
    return dg @ W1.T + du @ W3.T, x64.T @ dg, x64.T @ du, h.T @ dout


def layer_backward(x, w_router, bias, w1, w3, w2, dy, k: int, capacity_factor: float = 1.0,
                   cap: Optional[int] = None, ws1=None, ws3=None, ws2=None, align: int = 128,
                   aux_weight: float = 0.0, z_weight: float = 0.0,
                   selection_bias: Optional[np.ndarray] = None,
                   weight_experts: Optional[Sequence[int]] = None) -> LayerGrads:
    """With weight_experts, dw1 / dw3 / dw2 hold only those experts' gradients,
    in that order (the full arrays of a large layer do not fit in memory); every
    other gradient is complete."""
    T, d = x.shape
    N = w_router.shape[1]
    fwd = orc.layer_forward(x, w_router, bias, w1, w3, w2, k=k, capacity_factor=capacity_factor,
                            cap=cap, bf16=False, align=align, tokens=[],
                            selection_bias=selection_bias)
    x64 = orc.as_f64(x)
    dy = np.asarray(dy, dtype=np.float64)
    s, idx, w = fwd.scores, fwd.idx, fwd.w
    kept = fwd.disp.row_map >= 0

    dx = np.zeros((T, d))
    keep_w = list(range(N)) if weight_experts is None else [int(e) for e in weight_experts]
    slot = {e: i for i, e in enumerate(keep_w)}
    dw1 = np.zeros((len(keep_w),) + np.shape(w1)[1:])
    dw3 = np.zeros((len(keep_w),) + np.shape(w3)[1:])
    dw2 = np.zeros((len(keep_w),) + np.shape(w2)[1:])
    dwt = np.zeros((T, k))
    for e in range(N):
        ti, tj = np.nonzero((idx == e) & kept)
        if len(ti) == 0:
            continue                       # an expert no kept token chose gets no gradient
        xe = x64[ti]
        o = orc.swiglu_ffn(xe, w1[e], w3[e], w2[e], False)
        dwt[ti, tj] = np.sum(dy[ti] * o, axis=1)            # y = sum_j w_j o_j
        dxe, g1, g3, g2 = expert_backward(xe, w1[e], w3[e], w2[e], w[ti, tj][:, None] * dy[ti])
        np.add.at(dx, ti, dxe)
        if e in slot:
            dw1[slot[e]], dw3[slot[e]], dw2[slot[e]] = g1, g3, g2

    dws1 = dws3 = dws2 = None
    if ws1 is not None:                    # shared expert, weight 1
        dxs, dws1, dws3, dws2 = expert_backward(x64, ws1, ws3, ws2, dy)
        dx += dxs

    # renormalised top-k weights w_j = s_{e_j} / S, S = sum over the k chosen
    sel = np.take_along_axis(s, idx.astype(np.int64), axis=1)
    S = sel.sum(axis=1, keepdims=True)
    ds_sel = (dwt - np.sum(dwt * w, axis=1, keepdims=True)) / S
    ds = np.zeros((T, N))
    np.add.at(ds, (np.repeat(np.arange(T), k), idx.reshape(-1).astype(np.int64)), ds_sel.reshape(-1))
    # Switch auxiliary loss N sum_i f_i P_i, P_i = mean_t s_ti
    if aux_weight != 0.0 and T > 0:
        f = fwd.stats.y_frac
        ds += aux_weight * N * f[None, :] / T
    # softmax backward, then the z-loss (d/dg lse^2 = 2 lse s)
    dg = s * (ds - np.sum(ds * s, axis=1, keepdims=True))
    if z_weight != 0.0 and T > 0:
        g = fwd.logits
        m = g.max(axis=1, keepdims=True)
        lse = m + np.log(np.exp(g - m).sum(axis=1, keepdims=True))
        dg += z_weight * (2.0 / T) * lse * s
    dw_router = x64.T @ dg
    dx += dg @ orc.as_f64(w_router).T
    dbias = dg.sum(axis=0) if bias is not None else None
    return LayerGrads(dx, dw_router, dbias, dw1, dw3, dw2, dws1, dws3, dws2, dg, dwt)


def layer_loss(x, w_router, bias, w1, w3, w2, dy, k: int, capacity_factor: float = 1.0,
               cap: Optional[int] = None, ws1=None, ws3=None, ws2=None, align: int = 128,
               aux_weight: float = 0.0, z_weight: float = 0.0,
               selection_bias: Optional[np.ndarray] = None):
    """The scalar L whose gradient layer_backward returns, and the routing it
    used (for finite-difference checks)."""
    fwd = orc.layer_forward(x, w_router, bias, w1, w3, w2, k=k, capacity_factor=capacity_factor,
                            cap=cap, bf16=False, ws1=ws1, ws3=ws3, ws2=ws2, align=align,
                            selection_bias=selection_bias)
    L = float(np.sum(np.asarray(dy, np.float64) * fwd.y))
    L += aux_weight * fwd.stats.l_aux_switch
    L += z_weight * orc.router_z_loss(fwd.logits)
    return L, (fwd.idx.copy(), fwd.disp.row_map.copy())
