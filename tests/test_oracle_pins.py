"""Pins of the fp64 oracle against values the pages and the mathematics fix.

Every pin is written as a `check_*` function over the oracle module so that the
mutation tests at the bottom can plant a plausible mistake in the oracle (on the
CPU) and confirm that at least one pin catches it.
"""
import itertools
import math
import struct

import numpy as np
import pytest
import scipy.special
import torch

from oracle import moe_oracle as orc
from tests.conftest import read_sections

RNG = np.random.default_rng(1234)


# --------------------------------------------------------------------------
# capacity
# --------------------------------------------------------------------------

def check_capacity_worked_example(o=orc):
    # "负载均衡策略：MoE训练稳定性保障", section "专家容量裁剪": 1024 tokens, 8 experts,
    # ideal 128; factor 1.25 -> 160.
    for row in read_sections("capacity_worked_example.txt")[""]:
        T, N, k, cf, cap = int(row[0]), int(row[1]), int(row[2]), float(row[3]), int(row[4])
        assert o.capacity(cf, T, k, N) == cap, (row, o.capacity(cf, T, k, N))


def check_capacity_closed_forms(o=orc):
    # C = ceil(cf * T * k / N) for the five workload shapes (exact integers) and
    # for products that are not integers (ceiling, not floor or round).
    assert o.capacity(1.25, 256, 2, 8) == 80
    assert o.capacity(1.25, 4096, 2, 8) == 1280
    assert o.capacity(1.0, 8192, 8, 128) == 512
    assert o.capacity(1.25, 8192, 8, 256) == 320
    assert o.capacity(1.25, 16384, 2, 8) == 5120
    assert o.capacity(1.5, 7, 1, 2) == 6          # 5.25 -> 6
    assert o.capacity(1.0, 10, 1, 4) == 3         # 2.5 -> 3
    assert o.capacity(1.0, 0, 2, 8) == 0


def test_capacity_worked_example():
    check_capacity_worked_example()


def test_capacity_closed_forms():
    check_capacity_closed_forms()


# --------------------------------------------------------------------------
# softmax
# --------------------------------------------------------------------------

def check_softmax_library(o=orc):
    # special case that reduces to a library routine: scipy's softmax
    g = RNG.normal(size=(64, 16)) * 4.0
    np.testing.assert_allclose(o.softmax(g), scipy.special.softmax(g, axis=1), rtol=1e-13, atol=0)
    # large logits: exp would overflow without the max subtraction
    big = np.array([[1000.0, 999.0, 0.0], [-1000.0, -1001.0, -1002.0]])
    np.testing.assert_allclose(o.softmax(big), scipy.special.softmax(big, axis=1), rtol=1e-13)
    assert np.all(np.isfinite(o.softmax(big)))


def test_softmax_library():
    check_softmax_library()


# --------------------------------------------------------------------------
# top-k selection and weights
# --------------------------------------------------------------------------

def _brute_topk(g_row, k):
    """The unique k-subset whose members all precede every non-member under the
    order 'larger logit first, then lower index', listed in that order."""
    N = len(g_row)
    key = lambda i: (-g_row[i], i)  # noqa: E731
    hits = []
    for S in itertools.combinations(range(N), k):
        rest = [j for j in range(N) if j not in S]
        if all(key(i) < key(j) for i in S for j in rest):
            hits.append(sorted(S, key=key))
    assert len(hits) == 1
    return hits[0]


def check_topk_bruteforce(o=orc):
    rng = np.random.default_rng(7)
    for N in (1, 2, 3, 5, 8):
        for k in range(1, N + 1):
            # small integers force many exact ties
            g = rng.integers(-2, 3, size=(40, N)).astype(np.float64)
            idx = o.topk(g, k)
            for t in range(g.shape[0]):
                assert list(idx[t]) == _brute_topk(list(g[t]), k), (N, k, g[t], idx[t])


def check_topk_argmax(o=orc):
    # k = 1 is argmax; numpy's argmax returns the first (lowest) index on ties
    g = np.random.default_rng(3).integers(-3, 4, size=(200, 8)).astype(np.float64)
    np.testing.assert_array_equal(o.topk(g, 1)[:, 0], np.argmax(g, axis=1))


def check_weights(o=orc):
    rng = np.random.default_rng(11)
    g = rng.normal(size=(50, 8)) * 2
    s = o.softmax(g)
    for k in (1, 2, 3, 8):
        idx = o.topk(g, k)
        w = o.topk_weights(s, idx)
        np.testing.assert_allclose(w.sum(axis=1), 1.0, rtol=0, atol=1e-12)
        if k == 1:
            np.testing.assert_allclose(w, 1.0, rtol=0, atol=1e-15)
        if k == 8:   # k = N: the renormalised weights are the softmax itself
            np.testing.assert_allclose(w, np.take_along_axis(s, idx.astype(np.int64), 1),
                                       rtol=1e-13)
    # N = 2, k = 2 closed form: the weight of the larger logit a vs b is
    # 1 / (1 + exp(b - a))
    a, b = 0.7, -0.4
    w = o.topk_weights(o.softmax(np.array([[b, a]])), o.topk(np.array([[b, a]]), 2))
    assert abs(w[0, 0] - 1.0 / (1.0 + math.exp(b - a))) < 1e-15


def test_topk_bruteforce():
    check_topk_bruteforce()


def test_topk_argmax():
    check_topk_argmax()


def test_weights():
    check_weights()


# --------------------------------------------------------------------------
# capacity clip and permutation
# --------------------------------------------------------------------------

def check_dispatch_hand(o=orc):
    sec = read_sections("dispatch_hand.txt")
    for name in ("A", "B"):
        kv = {r[0]: [int(v) for v in r[1:]] for r in sec[name]}
        T, N, k, C, align = kv["T"][0], kv["N"][0], kv["k"][0], kv["C"][0], kv["align"][0]
        idx = np.array(kv["idx"], dtype=np.int32).reshape(T, k)
        dp = o.dispatch(idx, N, C, align)
        np.testing.assert_array_equal(dp.counts, kv["counts"])
        np.testing.assert_array_equal(dp.kept, kv["kept"])
        np.testing.assert_array_equal(dp.seg_off, kv["seg_off"])
        np.testing.assert_array_equal(dp.row_map.reshape(-1), kv["row_map"])
        assert dp.num_dropped == kv["dropped"][0]


def check_dispatch_invariants(o=orc):
    rng = np.random.default_rng(5)
    for (T, N, k, C, align) in [(300, 8, 2, 40, 128), (257, 16, 4, 70, 32),
                                (100, 5, 5, 100, 1), (64, 4, 1, 0, 8), (50, 3, 2, 1000, 16)]:
        g = rng.normal(size=(T, N)) + np.linspace(1.5, -1.5, N)[None, :]
        idx = o.topk(g, k)
        dp = o.dispatch(idx, N, C, align)
        np.testing.assert_array_equal(dp.counts, np.bincount(idx.reshape(-1), minlength=N))
        np.testing.assert_array_equal(dp.kept, np.minimum(dp.counts, C))
        assert int(dp.kept.sum()) == T * k - dp.num_dropped
        assert np.all(dp.seg_off % align == 0)
        kept_rows = dp.row_map[dp.row_map >= 0]
        assert len(np.unique(kept_rows)) == len(kept_rows)           # injective
        for e in range(N):
            tok, slot = np.nonzero(idx == e)                          # token order
            order = np.argsort(tok, kind="stable")
            tok, slot = tok[order], slot[order]
            rows = dp.row_map[tok, slot]
            # the first min(count, C) tokens are kept, in order, at consecutive rows
            n_keep = min(len(tok), C)
            np.testing.assert_array_equal(rows[:n_keep], dp.seg_off[e] + np.arange(n_keep))
            assert np.all(rows[n_keep:] == -1)
            assert dp.seg_off[e + 1] - dp.seg_off[e] >= n_keep


def test_dispatch_hand():
    check_dispatch_hand()


def test_dispatch_invariants():
    check_dispatch_invariants()


def test_permuted_rows_are_copies():
    x = np.arange(24, dtype=np.float32).reshape(6, 4)
    idx = np.array([[0], [0], [1], [0], [2], [0]], dtype=np.int32)
    dp = orc.dispatch(idx, 3, 2, 4)
    rows = orc.permuted_rows(x, dp)
    assert sorted(rows) == [0, 1, 4, 8]
    for r, t in ((0, 0), (1, 1), (4, 2), (8, 4)):
        np.testing.assert_array_equal(rows[r], x[t])


# --------------------------------------------------------------------------
# FFN and combine
# --------------------------------------------------------------------------

def _py_matvec(xrow, W):
    """Plain-Python x . W for a row x and a matrix W[d][f] (lists)."""
    d, f = len(W), len(W[0])
    return [sum(xrow[c] * W[c][j] for c in range(d)) for j in range(f)]


def _py_swiglu(xrow, W1, W3, W2):
    g = _py_matvec(xrow, W1)
    u = _py_matvec(xrow, W3)
    h = [gi / (1.0 + math.exp(-gi)) * ui for gi, ui in zip(g, u)]
    return _py_matvec(h, W2)


def _tiny_weights(rng, N, d, f):
    w1 = rng.normal(size=(N, d, f)).astype(np.float32)
    w3 = rng.normal(size=(N, d, f)).astype(np.float32)
    w2 = rng.normal(size=(N, f, d)).astype(np.float32)
    return w1, w3, w2


def check_dense_mlp(o=orc):
    # N = 1, k = 1, capacity >= T: the layer is one dense SwiGLU MLP
    rng = np.random.default_rng(21)
    T, d, f = 3, 4, 5
    x = rng.normal(size=(T, d)).astype(np.float32)
    wr = rng.normal(size=(d, 1)).astype(np.float32)
    w1, w3, w2 = _tiny_weights(rng, 1, d, f)
    res = o.layer_forward(x, wr, None, w1, w3, w2, k=1, cap=T, bf16=False, align=1)
    for t in range(T):
        want = _py_swiglu([float(v) for v in x[t]], w1[0].tolist(), w3[0].tolist(), w2[0].tolist())
        np.testing.assert_allclose(res.y[t], want, rtol=1e-12, atol=1e-12)


def check_dense_mixture(o=orc):
    # k = N and capacity >= T: y = sum_i softmax_i(g) * Expert_i(x)
    rng = np.random.default_rng(22)
    T, d, f, N = 4, 3, 4, 3
    x = rng.normal(size=(T, d)).astype(np.float32)
    wr = rng.normal(size=(d, N)).astype(np.float32)
    w1, w3, w2 = _tiny_weights(rng, N, d, f)
    res = o.layer_forward(x, wr, None, w1, w3, w2, k=N, cap=T, bf16=False, align=1)
    for t in range(T):
        xr = [float(v) for v in x[t]]
        g = [sum(xr[c] * float(wr[c, i]) for c in range(d)) for i in range(N)]
        m = max(g)
        ex = [math.exp(v - m) for v in g]
        s = [v / sum(ex) for v in ex]
        want = [0.0] * d
        for i in range(N):
            oi = _py_swiglu(xr, w1[i].tolist(), w3[i].tolist(), w2[i].tolist())
            want = [a + s[i] * b for a, b in zip(want, oi)]
        np.testing.assert_allclose(res.y[t], want, rtol=1e-12, atol=1e-12)


def check_dropped_slots_contribute_zero(o=orc):
    # capacity 0: every assignment is dropped, the routed output is exactly zero
    rng = np.random.default_rng(23)
    T, d, f, N = 5, 4, 4, 3
    x = rng.normal(size=(T, d)).astype(np.float32)
    wr = rng.normal(size=(d, N)).astype(np.float32)
    w1, w3, w2 = _tiny_weights(rng, N, d, f)
    res = o.layer_forward(x, wr, None, w1, w3, w2, k=2, cap=0, bf16=False, align=1)
    assert np.all(res.y == 0.0)
    # capacity 1 with k=1, N=1: only token 0 is kept and nothing is renormalised
    wr1 = rng.normal(size=(d, 1)).astype(np.float32)
    res = o.layer_forward(x, wr1, None, w1[:1], w3[:1], w2[:1], k=1, cap=1, bf16=False, align=1)
    assert np.any(res.y[0] != 0.0) and np.all(res.y[1:] == 0.0)


def check_shared_expert_added(o=orc):
    # a shared expert is added with weight 1 on top of the routed sum
    rng = np.random.default_rng(24)
    T, d, f, N = 4, 3, 4, 2
    x = rng.normal(size=(T, d)).astype(np.float32)
    wr = rng.normal(size=(d, N)).astype(np.float32)
    w1, w3, w2 = _tiny_weights(rng, N, d, f)
    s1, s3, s2 = _tiny_weights(rng, 1, d, f)
    base = o.layer_forward(x, wr, None, w1, w3, w2, k=1, cap=T, bf16=False, align=1)
    both = o.layer_forward(x, wr, None, w1, w3, w2, k=1, cap=T, bf16=False, align=1,
                           ws1=s1[0], ws3=s3[0], ws2=s2[0])
    for t in range(T):
        sh = _py_swiglu([float(v) for v in x[t]], s1[0].tolist(), s3[0].tolist(), s2[0].tolist())
        np.testing.assert_allclose(both.y[t] - base.y[t], sh, rtol=1e-11, atol=1e-12)


def test_dense_mlp():
    check_dense_mlp()


def test_dense_mixture():
    check_dense_mixture()


def test_dropped_slots_contribute_zero():
    check_dropped_slots_contribute_zero()


def test_shared_expert_added():
    check_shared_expert_added()


# --------------------------------------------------------------------------
# load-balance statistics
# --------------------------------------------------------------------------

def check_aux_hand(o=orc):
    sec = read_sections("aux_loss_4x4.txt")
    p = np.array([[float(v) for v in r] for r in sec["probs"]])
    g = np.log(p)
    idx = o.topk(g, 1)
    np.testing.assert_array_equal(idx[:, 0], [int(v) for v in sec["top1"][0]])
    st = o.aux_stats(idx, o.softmax(g), 4)
    np.testing.assert_allclose(st.y_frac, [float(v) for v in sec["y"][0]], rtol=0, atol=1e-15)
    np.testing.assert_allclose(st.z_mean, [float(v) for v in sec["z"][0]], rtol=0, atol=1e-15)
    assert abs(st.l_aux_p3 - float(sec["l_aux_p3"][0][0])) < 1e-14
    assert abs(st.l_aux_switch - float(sec["l_aux_switch"][0][0])) < 1e-14


def check_aux_uniform(o=orc):
    # circulant logits: every expert sees the same score distribution and the same
    # number of tokens, so f_i = P_i = 1/N and the Switch loss is exactly 1
    N, k, reps = 8, 2, 5
    c = np.array([3.0, 1.0, 0.5, 0.2, 0.1, -0.3, -1.0, -2.0])
    T = N * reps
    g = np.array([[c[(i - t) % N] for i in range(N)] for t in range(T)])
    st = o.aux_stats(o.topk(g, k), o.softmax(g), N)
    np.testing.assert_allclose(st.y_frac, 1.0 / N, rtol=1e-14)
    np.testing.assert_allclose(st.z_mean, 1.0 / N, rtol=1e-13)
    assert abs(st.l_aux_switch - 1.0) < 1e-13
    assert abs(st.l_aux_p3 - T / N**2) < 1e-12


def test_aux_hand():
    check_aux_hand()


def test_aux_uniform():
    check_aux_uniform()


# --------------------------------------------------------------------------
# Aux-Loss-Free selection bias and its update ("MoE 训练加速实战" §5.3-5.4)
# --------------------------------------------------------------------------

def check_selection_bias_hand(o=orc):
    # g = (1, 7/8, 0, -1), b = (0, 1/4, 0, 0): the biased scores are (1, 9/8, 0, -1),
    # so expert 1 wins the choice while the weights stay those of the plain softmax
    g = np.array([[1.0, 0.875, 0.0, -1.0]])
    b = np.array([0.0, 0.25, 0.0, 0.0], np.float32)
    np.testing.assert_array_equal(o.topk(g, 1, b), [[1]])
    np.testing.assert_array_equal(o.topk(g, 2, b), [[1, 0]])
    np.testing.assert_array_equal(o.topk(g, 2), [[0, 1]])
    e1, e78 = math.exp(1.0), math.exp(0.875)
    w = o.topk_weights(o.softmax(g), o.topk(g, 2, b))
    np.testing.assert_allclose(w, [[e78 / (e1 + e78), e1 / (e1 + e78)]], rtol=1e-15)
    # an unbiased softmax: z_i of the statistics do not see the bias
    st = o.aux_stats(o.topk(g, 1, b), o.softmax(g), 4)
    np.testing.assert_allclose(st.y_frac, [0, 1, 0, 0])
    np.testing.assert_allclose(st.z_mean, np.exp(g[0]) / np.exp(g[0]).sum(), rtol=1e-15)


def check_selection_bias_bruteforce(o=orc):
    # dyadic logits and biases (exact in fp32): the chosen set maximises
    # sum_{i in S} (g_i + b_i) over all k-subsets; a bias constant over the
    # experts changes nothing; a large bias on a set S of k experts forces S,
    # ranked by g inside S
    rng = np.random.default_rng(77)
    N, k = 6, 3
    for _ in range(40):
        g = rng.integers(-64, 64, size=(1, N)) / 8.0
        b = (rng.integers(-16, 16, size=N) / 8.0).astype(np.float32)
        got = o.topk(g, k, b)[0]
        sc = g[0] + b
        best = max(itertools.combinations(range(N), k), key=lambda S: (sum(sc[i] for i in S), [-i for i in S]))
        assert sorted(got.tolist()) == sorted(best), (g, b, got, best)
        np.testing.assert_array_equal(o.topk(g, k, b + np.float32(0.5)), o.topk(g, k, b))
        S = rng.choice(N, size=k, replace=False)
        big = np.zeros(N, np.float32)
        big[S] = 1024.0
        want = sorted(S.tolist(), key=lambda i: (-g[0, i], i))
        np.testing.assert_array_equal(o.topk(g, k, big)[0], want)
        np.testing.assert_array_equal(o.topk(g, k, np.zeros(N, np.float32)), o.topk(g, k))


def check_bias_update_hand(o=orc):
    # T = 4 tokens, k = 2, N = 4: the fair share is T k / N = 2 selections.
    # counts (3, 1, 0, 4): experts 0 and 3 over-loaded (b - gamma), 1 and 2
    # under-loaded (b + gamma); an expert exactly at its share keeps its bias
    b = np.array([0.5, 0.5, -0.5, 0.0], np.float32)
    got = o.bias_update(b, np.array([3, 1, 0, 4]), T=4, k=2, gamma=0.25)
    np.testing.assert_array_equal(got, np.array([0.25, 0.75, -0.25, -0.25], np.float32))
    got = o.bias_update(b, np.array([2, 2, 2, 2]), T=4, k=2, gamma=0.25)
    np.testing.assert_array_equal(got, b)
    got = o.bias_update(b, np.array([2, 3, 1, 2]), T=4, k=2, gamma=0.25)
    np.testing.assert_array_equal(got, np.array([0.5, 0.25, -0.25, 0.0], np.float32))
    assert got.dtype == np.float32


def check_aux_loss_free_balances(o=orc):
    # the method's purpose: on logits with a per-expert ramp (experts 0..1 take
    # most of the load), repeated sign updates of the selection bias drive the
    # load std towards 0 and move the bias against the load ramp
    from expert_router_gemm_b200 import synth
    T, N, k = 4096, 8, 2
    g = synth.make_logits(5, T, N, "skewed").astype(np.float64)
    b = np.zeros(N, np.float32)
    first = None
    for _ in range(60):
        counts = np.bincount(o.topk(g, k, b).reshape(-1), minlength=N)
        m = o.load_metrics(counts, counts, T, k)
        first = m.load_std if first is None else first
        b = o.bias_update(b, counts, T, k, 0.05)
    assert first > 0.1 and m.load_std < 0.1 * first, (first, m.load_std)
    assert np.all(np.diff(b) > 0), b


def test_aux_loss_free_balances():
    check_aux_loss_free_balances()


def test_selection_bias_hand():
    check_selection_bias_hand()


def test_selection_bias_bruteforce():
    check_selection_bias_bruteforce()


def test_bias_update_hand():
    check_bias_update_hand()


# --------------------------------------------------------------------------
# router z-loss and the load-health figures
# --------------------------------------------------------------------------

def check_z_loss(o=orc):
    # equal logits c over N experts: logsumexp = c + log N
    for N, c in ((8, 0.0), (128, -2.5), (3, 7.0)):
        g = np.full((5, N), c)
        assert abs(o.router_z_loss(g) - (c + math.log(N)) ** 2) < 1e-12
    # library special case: scipy's logsumexp, then the mean of its squares
    g = np.random.default_rng(5).normal(size=(64, 32)) * 3
    want = float(np.mean(scipy.special.logsumexp(g, axis=1) ** 2))
    assert abs(o.router_z_loss(g) - want) < 1e-12 * want
    # large logits (a stable log-sum-exp) and the empty batch
    big = g + 1000.0
    want = float(np.mean((scipy.special.logsumexp(g, axis=1) + 1000.0) ** 2))
    assert abs(o.router_z_loss(big) - want) < 1e-12 * want
    assert o.router_z_loss(np.zeros((0, 4))) == 0.0


def check_load_metrics_hand(o=orc):
    # counts (3, 1, 0, 4) of T k = 8 selections: f = (3, 1, 0, 4) / 8, mean 1/4,
    # squared deviations (1, 1, 4, 4) / 64, so std = sqrt(10) / 16; the two
    # busiest experts take 7 of 8; kept (3, 1, 0, 3) under C = 3 -> 7 / 4 rows each
    m = o.load_metrics(np.array([3, 1, 0, 4]), np.array([3, 1, 0, 3]), T=4, k=2)
    assert abs(m.load_std - math.sqrt(10) / 16) < 1e-15
    assert m.top2_ratio == 7 / 8
    assert m.avg_tokens_per_expert == 7 / 4
    # perfectly balanced: std 0, top-2 share 2/N, T k / N rows per expert
    m = o.load_metrics(np.full(8, 64), np.full(8, 64), T=256, k=2)
    assert m.load_std == 0.0 and m.top2_ratio == 0.25 and m.avg_tokens_per_expert == 64.0
    m = o.load_metrics(np.zeros(4, np.int64), np.zeros(4, np.int64), T=0, k=2)
    assert (m.load_std, m.top2_ratio, m.avg_tokens_per_expert) == (0.0, 0.0, 0.0)


def test_z_loss():
    check_z_loss()


def test_load_metrics_hand():
    check_load_metrics_hand()


# --------------------------------------------------------------------------
# number formats
# --------------------------------------------------------------------------

def check_bf16_rounding(o=orc):
    one = 1.0
    assert o.round_to_bf16(np.array([one + 2.0**-8]))[0] == 1.0              # tie -> even
    assert o.round_to_bf16(np.array([one + 3 * 2.0**-8]))[0] == 1.0 + 2.0**-6  # tie -> even (up)
    assert o.round_to_bf16(np.array([one + 2.0**-8 + 2.0**-30]))[0] == 1.0 + 2.0**-7
    assert o.round_to_bf16(np.array([-3.0]))[0] == -3.0
    # library special case: torch's fp32 -> bf16 conversion rounds to nearest even
    v = np.random.default_rng(9).normal(size=4096).astype(np.float32) * 10
    v = np.concatenate([v, np.float32(2.0**-130) * np.arange(1, 64, dtype=np.float32)])
    want = torch.from_numpy(v).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(o.round_to_bf16(v.astype(np.float64)), want)


def check_bf16_decode(o=orc):
    bits = np.random.default_rng(10).integers(0, 2**16, size=4096).astype(np.uint16)
    bits = bits[((bits >> 7) & 0xFF) != 0xFF]                   # finite values only
    want = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(o.bf16_bits_to_f64(bits), want)


def _py_bf16_rne(v: float) -> float:
    """Round a Python float to the nearest bf16 value, ties to even, by integer
    arithmetic on its IEEE-754 double bit pattern (sign, 11-bit exponent, 52-bit
    fraction): bf16 keeps 7 fraction bits, so 45 fraction bits are dropped.
    Normal, finite values only (the cases below stay far from the extremes)."""
    bits = struct.unpack("<Q", struct.pack("<d", v))[0]
    drop = 45
    keep = bits >> drop
    rest = bits & ((1 << drop) - 1)
    half = 1 << (drop - 1)
    if rest > half or (rest == half and (keep & 1)):
        keep += 1                       # a carry into the exponent is the right result
    return struct.unpack("<d", struct.pack("<Q", keep << drop))[0]


def check_layer_bf16_h_rounding(o=orc):
    # bf16 compute with fp32 accumulation, read as: h = silu(x W1) * (x W3) is
    # formed exactly, rounded once to bf16 (nearest, ties to even), and only then
    # multiplied by W2 ("MoE 训练加速实战" §2.2 for the layer; reading (iii) for
    # where the one bf16 rounding sits).  Tokens are one-hot rows of a 4 x 4
    # identity, so token t's hidden unit j sees g = W1[t, j], u = W3[t, j]; for
    # g >= 64, e^-g < 2^-92 and silu(g) = g exactly in fp64, so h = g * u is an
    # exact dyadic number placed on or next to a bf16 rounding boundary.
    d = f = 4
    w1 = np.full((1, d, f), 64.0)
    w3 = np.zeros((1, d, f))
    cases = {  # (token, unit): (g, u, bf16(h) worked out by hand)
        (0, 0): (64.0, (1 + 2.0**-8) / 64, 1.0),                         # tie -> even (down)
        (0, 1): (64.0, (1 + 3 * 2.0**-8) / 64, 1 + 2.0**-6),             # tie -> even (up)
        (0, 2): (96.0, 2.0**-6 * (1 + 2.0**-8 + 2.0**-9), 1.5078125),    # h = 1.5087890625
        (0, 3): (64.0, -(1 + 2.0**-8 + 2.0**-30) / 64, -(1 + 2.0**-7)),  # just past a tie
        (1, 0): (64.0, 2.0**-6 * (1 + 2.0**-9), 1.0),                    # below half a step
        (1, 1): (128.0, 3 * 2.0**-7 * (1 + 2.0**-9), 3.0),
        (1, 2): (64.0, 2.0**-6 * 257 / 256 * 3, 3.015625),                # 3 (1 + 2^-8): 3/4 step, up
        (1, 3): (64.0, 2.0**-6 * (1 - 2.0**-10), 1.0),                   # rounds up to 1
    }
    for (t, j), (g, u, _) in cases.items():
        w1[0, t, j], w3[0, t, j] = g, u
    w2 = np.zeros((1, f, d))
    for j in range(f):
        w2[0, j, j] = 3.0                 # o_j = 3 bf16(h_j): rounding o instead of h shows
    x = np.eye(4, dtype=np.float32)
    wr = np.zeros((d, 1), dtype=np.float32)
    res = o.layer_forward(x, wr, None, w1, w3, w2, k=1, cap=4, bf16=True, align=1)
    for (t, j), (g, u, want_h) in cases.items():
        assert res.y[t, j] == 3.0 * want_h, ((t, j), res.y[t, j], 3.0 * want_h)
        assert _py_bf16_rne(g * u) == want_h, ((t, j), g * u)   # the hand values themselves
    # the same layer without the rounding keeps h exact
    res32 = o.layer_forward(x, wr, None, w1, w3, w2, k=1, cap=4, bf16=False, align=1)
    for (t, j), (g, u, _) in cases.items():
        assert res32.y[t, j] == 3.0 * g * u, ((t, j), res32.y[t, j])

    # random small layer: every output against a plain-Python loop that rounds h
    # with the integer rounding above and nothing else
    rng = np.random.default_rng(31)
    T, d, f, N = 5, 8, 6, 3
    x = rng.normal(size=(T, d)).astype(np.float32)
    wr = rng.normal(size=(d, N)).astype(np.float32)
    w1, w3, w2 = _tiny_weights(rng, N, d, f)
    res = o.layer_forward(x, wr, None, w1, w3, w2, k=N, cap=T, bf16=True, align=1)
    for t in range(T):
        xr = [float(v) for v in x[t]]
        gl = [sum(xr[c] * float(wr[c, i]) for c in range(d)) for i in range(N)]
        m = max(gl)
        ex = [math.exp(v - m) for v in gl]
        s = [v / sum(ex) for v in ex]
        want = [0.0] * d
        for i in range(N):
            gg = _py_matvec(xr, w1[i].tolist())
            uu = _py_matvec(xr, w3[i].tolist())
            h = [_py_bf16_rne(a / (1.0 + math.exp(-a)) * b) for a, b in zip(gg, uu)]
            oi = _py_matvec(h, w2[i].tolist())
            want = [acc + s[i] * b for acc, b in zip(want, oi)]
        np.testing.assert_allclose(res.y[t], want, rtol=1e-12, atol=1e-12)


def test_bf16_rounding():
    check_bf16_rounding()


def test_layer_bf16_h_rounding():
    check_layer_bf16_h_rounding()


def test_bf16_decode():
    check_bf16_decode()


# --------------------------------------------------------------------------
# mutation tests: plant a plausible mistake in the oracle, expect a pin to fail
# --------------------------------------------------------------------------

ALL_CHECKS = [check_capacity_worked_example, check_capacity_closed_forms, check_softmax_library,
              check_topk_bruteforce, check_topk_argmax, check_weights, check_dispatch_hand,
              check_dispatch_invariants, check_dense_mlp, check_dense_mixture,
              check_dropped_slots_contribute_zero, check_shared_expert_added, check_aux_hand,
              check_aux_uniform, check_bf16_rounding, check_bf16_decode, check_selection_bias_hand,
              check_selection_bias_bruteforce, check_bias_update_hand, check_z_loss,
              check_load_metrics_hand, check_aux_loss_free_balances, check_layer_bf16_h_rounding]


def _mut_topk_high_index_ties(g, k, selection_bias=None):
    g = np.asarray(g, np.float64)
    return np.argsort(g, axis=1, kind="stable")[:, ::-1][:, :k].astype(np.int32)


def _mut_weights_no_renorm(s, idx):
    return np.take_along_axis(s, idx.astype(np.int64), axis=1)


def _mut_capacity_floor(cf, T, k, N):
    from fractions import Fraction
    return int(math.floor(Fraction(cf) * T * k / N))


def _mut_capacity_no_k(cf, T, k, N):
    from fractions import Fraction
    return int(math.ceil(Fraction(cf) * T / N))


def _mut_dispatch_drop_whole_expert(idx, N, C, align=128):
    # the literal reading of the page's snippet: an over-full expert loses all tokens
    d = orc.Dispatch.__new__(orc.Dispatch)
    ref = _ORIG["dispatch"](idx, N, C, align)
    rm = ref.row_map.copy()
    for e in range(N):
        if ref.counts[e] > C:
            rm[idx == e] = -1
    d.__dict__.update(ref.__dict__)
    d.row_map = rm
    return d


def _mut_dispatch_keep_last(idx, N, C, align=128):
    ref = _ORIG["dispatch"](idx[::-1].copy(), N, C, align)
    d = orc.Dispatch.__new__(orc.Dispatch)
    d.__dict__.update(ref.__dict__)
    d.row_map = ref.row_map[::-1].copy()
    return d


def _mut_softmax_no_max(g):
    with np.errstate(over="ignore", invalid="ignore"):
        z = np.exp(np.asarray(g, np.float64))
        return z / z.sum(axis=1, keepdims=True)


def _mut_silu_sign(u):
    with np.errstate(over="ignore"):
        return u / (1.0 + np.exp(u))


def _mut_swiglu_swap(x64, w1, w3, w2, round_h_bf16):
    return _ORIG["swiglu_ffn"](x64, w3, w1, w2, round_h_bf16)


def _mut_aux_z_topk(idx, s, N):
    st = _ORIG["aux_stats"](idx, s, N)
    w = orc.topk_weights(s, idx)
    z = np.zeros(N)
    np.add.at(z, idx.reshape(-1), w.reshape(-1))
    z /= idx.shape[0]
    st.z_mean = z
    return st


def _mut_aux_p3_inverted(idx, s, N):
    st = _ORIG["aux_stats"](idx, s, N)
    T = idx.shape[0]
    st.l_aux_p3 = (N / T) * float(np.sum(st.y_frac * st.z_mean))
    return st


def _mut_bf16_truncate(v):
    v = np.asarray(v, np.float64).astype(np.float32)
    u = v.view(np.uint32) & np.uint32(0xFFFF0000)
    return u.view(np.float32).astype(np.float64)


def _mut_bf16_decode_low_half(bits):
    u32 = np.asarray(bits, dtype=np.uint16).astype(np.uint32)
    return u32.view(np.float32).astype(np.float64)


def _mut_topk_ignores_bias(g, k, selection_bias=None):
    return _ORIG["topk"](g, k)


def _mut_topk_bias_scaled(g, k, selection_bias=None):
    # the bias applied with the wrong sign (it penalises the experts it should favour)
    sb = None if selection_bias is None else -np.asarray(selection_bias, np.float32)
    return _ORIG["topk"](g, k, sb)


def _mut_bias_update_sign(b, counts, T, k, gamma):
    counts = np.asarray(counts, np.int64)
    return np.asarray(b, np.float32) + np.float32(gamma) * np.sign(counts.shape[0] * counts - T * k).astype(np.float32)


def _mut_bias_update_share_of_tokens(b, counts, T, k, gamma):
    counts = np.asarray(counts, np.int64)
    return np.asarray(b, np.float32) + np.float32(gamma) * np.sign(T - counts.shape[0] * counts).astype(np.float32)


def _mut_z_loss_unsquared(g):
    g = np.asarray(g, np.float64)
    return float(np.mean(scipy.special.logsumexp(g, axis=1))) if g.shape[0] else 0.0


def _mut_z_loss_no_max(g):
    g = np.asarray(g, np.float64)
    with np.errstate(over="ignore"):
        return float(np.mean(np.log(np.exp(g).sum(axis=1)) ** 2)) if g.shape[0] else 0.0


def _mut_load_std_sample(counts, kept, T, k):
    m = _ORIG["load_metrics"](counts, kept, T, k)
    f = np.asarray(counts) / float(max(T * k, 1))
    m.load_std = float(np.std(f, ddof=1))
    return m


def _mut_load_top1(counts, kept, T, k):
    m = _ORIG["load_metrics"](counts, kept, T, k)
    if T:
        m.top2_ratio = float(np.max(counts)) / float(T * k)
    return m


def _mut_load_avg_counts(counts, kept, T, k):
    m = _ORIG["load_metrics"](counts, kept, T, k)
    m.avg_tokens_per_expert = float(np.sum(counts)) / len(counts)
    return m


def _mut_swiglu_no_h_rounding(x64, w1, w3, w2, round_h_bf16):
    # the bf16 flag is ignored: h reaches W2 unrounded
    return _ORIG["swiglu_ffn"](x64, w1, w3, w2, False)


def _mut_swiglu_rounds_output(x64, w1, w3, w2, round_h_bf16):
    # the rounding is applied to the expert output instead of h
    o = _ORIG["swiglu_ffn"](x64, w1, w3, w2, False)
    return orc.round_to_bf16(o) if round_h_bf16 else o


def _mut_swiglu_rounds_gate_up(x64, w1, w3, w2, round_h_bf16):
    # g and u are rounded before silu and the product, h itself is not
    g = x64 @ orc.as_f64(w1)
    u = x64 @ orc.as_f64(w3)
    if round_h_bf16:
        g, u = orc.round_to_bf16(g), orc.round_to_bf16(u)
    return (orc.silu(g) * u) @ orc.as_f64(w2)


def _mut_swiglu_truncates_h(x64, w1, w3, w2, round_h_bf16):
    # h is cut to bf16 by dropping the low half of its fp32 pattern (no rounding)
    h = orc.silu(x64 @ orc.as_f64(w1)) * (x64 @ orc.as_f64(w3))
    if round_h_bf16:
        h = (h.astype(np.float32).view(np.uint32) & np.uint32(0xFFFF0000)).view(np.float32).astype(np.float64)
    return h @ orc.as_f64(w2)


_ORIG = {n: getattr(orc, n) for n in ("dispatch", "swiglu_ffn", "aux_stats", "topk", "load_metrics")}

MUTANTS = [
    ("topk", _mut_topk_high_index_ties),
    ("topk_weights", _mut_weights_no_renorm),
    ("capacity", _mut_capacity_floor),
    ("capacity", _mut_capacity_no_k),
    ("dispatch", _mut_dispatch_drop_whole_expert),
    ("dispatch", _mut_dispatch_keep_last),
    ("softmax", _mut_softmax_no_max),
    ("silu", _mut_silu_sign),
    ("swiglu_ffn", _mut_swiglu_swap),
    ("aux_stats", _mut_aux_z_topk),
    ("aux_stats", _mut_aux_p3_inverted),
    ("round_to_bf16", _mut_bf16_truncate),
    ("bf16_bits_to_f64", _mut_bf16_decode_low_half),
    ("topk", _mut_topk_ignores_bias),
    ("topk", _mut_topk_bias_scaled),
    ("bias_update", _mut_bias_update_sign),
    ("bias_update", _mut_bias_update_share_of_tokens),
    ("router_z_loss", _mut_z_loss_unsquared),
    ("router_z_loss", _mut_z_loss_no_max),
    ("load_metrics", _mut_load_std_sample),
    ("load_metrics", _mut_load_top1),
    ("load_metrics", _mut_load_avg_counts),
    ("swiglu_ffn", _mut_swiglu_no_h_rounding),
    ("swiglu_ffn", _mut_swiglu_rounds_output),
    ("swiglu_ffn", _mut_swiglu_rounds_gate_up),
    ("swiglu_ffn", _mut_swiglu_truncates_h),
]


@pytest.mark.parametrize("name,mutant", MUTANTS, ids=[f"{n}:{m.__name__}" for n, m in MUTANTS])
def test_mutant_is_caught(monkeypatch, name, mutant):
    monkeypatch.setattr(orc, name, mutant)
    caught = []
    for chk in ALL_CHECKS:
        try:
            chk(orc)
        except (AssertionError, ValueError, FloatingPointError, IndexError):
            caught.append(chk.__name__)
    assert caught, f"no pin caught the planted mistake in {name}"
