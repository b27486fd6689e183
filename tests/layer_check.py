"""Compare a GPU layer run with the fp64 oracle.  (Not a test module.)

The GPU router computes the logits in fp32 and the oracle in fp64, so a token
whose k-th and (k+1)-th logits are closer than the fp32 error can be routed
differently by the two (several routings are then correct).  The check:
  1. GPU logits match the oracle's within the fp32 accumulation bound of
     logit_bound() (K*u*sum|x*w| per element);
  2. every token whose selected expert set differs is a near tie under the
     oracle's logits (GPU choice within twice that bound of the boundary), and
     such tokens are rare;
  3. capacity decisions may then differ only in over-full experts, and only for
     as many tokens as the selection flips can shift;
  4. on all remaining tokens (or a sample of them) the layer output matches the
     oracle within the stated relative Frobenius tolerance, and every one of
     those tokens within PER_TOKEN_FACTOR times that tolerance on its own.
"""
from __future__ import annotations

import numpy as np

from oracle import moe_oracle as orc

U32 = 2.0 ** -24   # unit roundoff of fp32
PER_TOKEN_FACTOR = 5.0   # bound of each token's relative error, in units of the layer tolerance


def logit_bound(x, w_router, bias=None):
    """First-order bound of an fp32 dot product accumulated over K terms, with
    per-add relative error <= u (any order, round-to-nearest or truncating
    adders): |err| <= K * u * sum_c |x_c w_c|.  K = 3d covers the tensor-core
    router, which adds the products of the three bf16 parts of each weight; the
    bias adds one more rounding of at most u * (sum|x w| + |b|)."""
    xa = np.abs(orc.as_f64(x))
    wa = np.abs(orc.as_f64(w_router))
    s = xa @ wa
    if bias is not None:
        s = s + np.abs(orc.as_f64(bias))[None, :]
    return (3 * xa.shape[1] + 2) * U32 * s + 1e-7


def z_loss_tolerance(g64, N):
    """Bound on |z-loss(GPU) - z-loss(oracle)| for fp32 logits g64 (as float64).

    Per token the GPU forms lse = m + log(sum_i exp(g_i - m)) in fp32: the sum of
    at most N exponentials (each within 2 ulp) over at most N/32 + 5 sequential
    and butterfly additions has relative error below (N/32 + 9) u, so log(sum)
    is off by that much plus one ulp of log N; adding m rounds once more.  With
    delta_t that bound, (lse + delta)^2 - lse^2 <= 2 |lse| delta + delta^2; the
    mean over tokens then sums in double (negligible)."""
    m = g64.max(axis=1)
    lse = m + np.log(np.exp(g64 - m[:, None]).sum(axis=1))
    delta = (N / 32 + 9) * U32 + 2 * U32 * (np.abs(lse) + np.log(N) + 1)
    return float(np.mean(2 * np.abs(lse) * delta + delta ** 2)) * 2 + 1e-12


def check_route_extras(st, g64, idx, T, k, N):
    """The router z-loss and the load figures of a routing call's statistics."""
    zl = orc.router_z_loss(g64)
    assert abs(float(st["z_loss"][0]) - zl) <= z_loss_tolerance(g64, N), (st["z_loss"][0], zl)
    counts = np.bincount(idx.reshape(-1), minlength=N)
    ref = orc.load_metrics(counts, counts, T, k)
    np.testing.assert_allclose(st["load_std"][0], ref.load_std, rtol=1e-6, atol=1e-9)
    assert st["top2_ratio"][0] == np.float32(ref.top2_ratio), (st["top2_ratio"][0], ref.top2_ratio)


def oracle_routing(inp, w, align=128, cap=None, selection_bias=None):
    return orc.layer_forward(inp.x, inp.w_router, inp.bias, inp.w1, inp.w3, inp.w2, k=w.k,
                             capacity_factor=w.capacity_factor, cap=cap, bf16=inp.bf16,
                             align=align, tokens=[], selection_bias=selection_bias)


def compare_layer(inp, w, gpu_y, gpu_idx, gpu_row_map, gpu_logits=None, tol=2e-2,
                  sample=None, seed=0, align=128, cap=None, selection_bias=None, mxfp8=False):
    """Returns (rel_frobenius, n_compared, n_flips).  With a selection bias the
    near-tie test runs on the biased scores that decide the choice; with mxfp8
    the reference output is the block-scaled FP8 layer of oracle.mxfp8."""
    T = inp.x.shape[0]
    ref = oracle_routing(inp, w, align, cap, selection_bias)
    bound = logit_bound(inp.x, inp.w_router, inp.bias)
    if gpu_logits is not None:
        err = np.abs(gpu_logits.astype(np.float64) - ref.logits)
        assert np.all(err <= bound), f"router logits differ by {err.max():.3g}"

    g = ref.logits
    if selection_bias is not None:
        g = g + np.asarray(selection_bias, np.float64)[None, :]
    o_sets = [set(r) for r in ref.idx.tolist()]
    g_sets = [set(r) for r in gpu_idx.tolist()]
    flips = [t for t in range(T) if o_sets[t] != g_sets[t]]
    for t in flips:
        chosen = sorted(g_sets[t])
        rest = [e for e in range(g.shape[1]) if e not in g_sets[t]]
        assert g[t, chosen].min() >= g[t, rest].max() - 2 * bound[t].max(), \
            f"token {t}: GPU selection is not a near tie"
    assert len(flips) <= max(2, T // 500), f"{len(flips)} routing flips"

    def kept_pairs(idx, row_map, t):
        return {(int(e), bool(r >= 0)) for e, r in zip(idx[t], row_map[t])}

    over_full = set(np.nonzero(ref.disp.counts > ref.capacity)[0].tolist())
    flip_set = set(flips)
    cascade = []
    for t in range(T):
        if t in flip_set:
            continue
        a = kept_pairs(ref.idx, ref.disp.row_map, t)
        b = kept_pairs(gpu_idx, gpu_row_map, t)
        if a != b:
            diff_experts = {e for (e, _) in a ^ b}
            assert diff_experts <= over_full, f"token {t}: capacity decision differs"
            cascade.append(t)
    assert len(cascade) <= 2 * len(flips), f"{len(cascade)} capacity differences"

    good = np.array(sorted(set(range(T)) - flip_set - set(cascade)), dtype=np.int64)
    if sample is not None and sample < len(good):
        good = np.sort(np.random.default_rng(seed).choice(good, size=sample, replace=False))
    if mxfp8:
        from oracle import mxfp8 as mxo
        res = mxo.layer_forward_mxfp8(inp.x, inp.w_router, inp.bias, inp.w1, inp.w3, inp.w2, k=w.k,
                                      capacity_factor=w.capacity_factor, cap=cap, ws1=inp.ws1,
                                      ws3=inp.ws3, ws2=inp.ws2, align=align, tokens=good,
                                      logits=ref.logits, selection_bias=selection_bias)
    else:
        res = orc.layer_forward(inp.x, inp.w_router, inp.bias, inp.w1, inp.w3, inp.w2, k=w.k,
                                capacity_factor=w.capacity_factor, cap=cap, bf16=inp.bf16,
                                ws1=inp.ws1, ws3=inp.ws3, ws2=inp.ws2, align=align, tokens=good,
                                logits=ref.logits, selection_bias=selection_bias)
    y = gpu_y[good]
    if y.dtype == np.uint16:
        y = (y.astype(np.uint32) << np.uint32(16)).view(np.float32)
    rel = orc.rel_frobenius(y.astype(np.float64), res.y)
    assert rel <= tol, f"relative Frobenius error {rel:.3g} > {tol}"
    # every compared token on its own, so that an error confined to a few rows of
    # a large layer cannot hide in the Frobenius norm: each row's relative error
    # stays within PER_TOKEN_FACTOR times the layer tolerance (a row the oracle
    # leaves exactly zero, all slots dropped and no shared expert, must be zero)
    diff = np.linalg.norm(y.astype(np.float64) - res.y, axis=1)
    ref_n = np.linalg.norm(res.y, axis=1)
    zero = ref_n == 0
    assert np.all(diff[zero] == 0), "a token the oracle leaves at zero is not zero"
    if np.any(~zero):
        worst = float(np.max(diff[~zero] / ref_n[~zero]))
        assert worst <= PER_TOKEN_FACTOR * tol, f"token relative error {worst:.3g} > {PER_TOKEN_FACTOR} x {tol}"
    return rel, len(good), len(flips)
