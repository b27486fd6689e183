"""GPU parity of Aux-Loss-Free routing and of the router z-loss / load figures.

Aux-Loss-Free routing ("MoE 训练加速实战：DeepEP + Grouped GeMM + Aux-Loss-Free"
§5.3-5.4): a per-expert bias b steers the top-k choice only, and the update
b_i += gamma * sign(1/N - f_i) runs on the device.  Given identical fp32 logits
the selection is bit-exact (both sides rank the fp32 sum g + b, ties to the
lower index) and so is the bias after any number of updates (the sign is an
integer decision, the update one fp32 addition).  The weights come from the
unbiased softmax (relative tolerance 2e-6, as for plain routing).

The z-loss ("负载均衡策略：MoE训练稳定性保障", z_loss_weight) is compared within
the fp32 bound of z_loss_tolerance(); the load std within 1e-6 relative; the
top-2 share and the tokens per expert bit for bit (exact integer ratios rounded
once to fp32 on both sides)."""
import numpy as np
import pytest
import torch

from expert_router_gemm_b200 import synth
from expert_router_gemm_b200.configs import Workload
from oracle import moe_oracle as orc

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from expert_router_gemm_b200 import moe  # noqa: E402
from tests import gpu_util as gu  # noqa: E402
from tests.layer_check import check_route_extras, compare_layer, z_loss_tolerance  # noqa: E402

W_RTOL = 2e-6


def _bits(a):
    return np.asarray(a, np.float32).view(np.uint32)


def _check_biased_route(T, N, k, lpat, bpat, seed):
    logits = synth.make_logits(seed, T, N, lpat)
    sb = synth.make_selection_bias(seed, N, bpat)
    cfg = moe.make_config(T=T, d=64, N=N, k=k, f=64, capacity_factor=1.0)
    idx, w, st, flags = gu.route_from_logits(cfg, logits, sb)
    assert flags == 0
    g = logits.astype(np.float64)
    want = orc.topk(g, k, sb)
    np.testing.assert_array_equal(idx, want)
    s = orc.softmax(g)
    np.testing.assert_allclose(w, orc.topk_weights(s, want), rtol=W_RTOL, atol=1e-7)
    ref = orc.aux_stats(want, s, N)
    np.testing.assert_array_equal(st["counts"], np.bincount(want.reshape(-1), minlength=N))
    np.testing.assert_allclose(st["y_frac"], ref.y_frac, rtol=1e-6, atol=0)
    np.testing.assert_allclose(st["z_mean"], ref.z_mean, rtol=1e-5, atol=1e-7)
    np.testing.assert_allclose(st["l_aux_p3"][0], ref.l_aux_p3, rtol=1e-5)
    check_route_extras(st, g, want, T, k, N)
    return idx


@pytest.mark.parametrize("N,k", [(8, 2), (8, 8), (5, 3), (16, 4), (33, 7), (64, 32), (128, 8),
                                 (256, 8), (1, 1)])
@pytest.mark.parametrize("lpat,bpat", [("normal", "normal"), ("ties", "dyadic"),
                                       ("zeros", "dyadic"), ("skewed", "normal"),
                                       ("onehot", "normal"), ("normal", "zeros")])
def test_route_selection_bias_bitexact(N, k, lpat, bpat):
    for T in (1, 37, 300):
        idx = _check_biased_route(T, N, k, lpat, bpat, seed=T + 17)
        if bpat == "zeros":   # a zero bias routes exactly as no bias
            plain, _, _, _ = gu.route_from_logits(
                moe.make_config(T=T, d=64, N=N, k=k, f=64), synth.make_logits(T + 17, T, N, lpat))
            np.testing.assert_array_equal(idx, plain)


def test_route_selection_bias_many_tokens():
    _check_biased_route(8192, 128, 8, "normal", "normal", seed=3)
    _check_biased_route(8192, 256, 8, "skewed", "normal", seed=4)
    _check_biased_route(16384, 8, 2, "ties", "dyadic", seed=5)


@pytest.mark.parametrize("N", [1, 8, 33, 256])
@pytest.mark.parametrize("gamma", [1e-3, 0.05, 3.0])
def test_bias_update_bitexact(N, gamma):
    k = min(N, 4)
    T = 256 * N                       # fair share T k / N = 256 k selections
    rng = np.random.default_rng(N)
    counts = rng.integers(0, 2 * 256 * k + 1, size=N).astype(np.int32)
    counts[0] = 256 * k               # exactly at the fair share: unchanged
    b = synth.make_selection_bias(N, N, "normal")
    cfg = moe.make_config(T=T, d=64, N=N, k=k, f=64)
    bd = gu.cuda_tensor(b)
    moe.moe_bias_update(cfg, bd, gu.cuda_tensor(counts), gamma)
    got = gu.host(bd)
    want = orc.bias_update(b, counts, T, k, gamma)
    np.testing.assert_array_equal(_bits(got), _bits(want))
    assert got[0] == b[0]


@pytest.mark.parametrize("T,N,k,pattern,gamma,steps", [
    (4096, 8, 2, "skewed", 0.05, 40),
    (8192, 256, 8, "skewed", 1e-3, 8),
    (2048, 64, 6, "ties", 0.25, 12),
])
def test_aux_loss_free_loop_bitexact(T, N, k, pattern, gamma, steps):
    """Route -> read counts -> update the bias, repeated on the device; the oracle
    repeats the same steps.  Selections and biases agree bit for bit at every step."""
    logits = synth.make_logits(9, T, N, pattern)
    cfg = moe.make_config(T=T, d=64, N=N, k=k, f=64, capacity_factor=1.0)
    lg = gu.cuda_tensor(logits)
    bd = torch.zeros(N, dtype=torch.float32, device="cuda")
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    ws = gu.op_workspace(cfg)
    bufs, st = gu.new_stats(N)
    g = logits.astype(np.float64)
    b = np.zeros(N, np.float32)
    stds = []
    for _ in range(steps):
        moe.moe_route_from_logits(cfg, lg, bd, idx, w, st, ws)
        moe.moe_bias_update(cfg, bd, bufs["counts"], gamma)
        want = orc.topk(g, k, b)
        counts = np.bincount(want.reshape(-1), minlength=N)
        b = orc.bias_update(b, counts, T, k, gamma)
        np.testing.assert_array_equal(gu.host(idx), want)
        np.testing.assert_array_equal(_bits(gu.host(bd)), _bits(b))
        stds.append(float(gu.host(bufs["load_std"])[0]))
    assert moe.moe_read_flags(ws) == 0
    if pattern == "skewed" and gamma >= 0.05:
        assert stds[-1] < 0.5 * stds[0], stds


def test_layer_with_selection_bias():
    """The whole bf16 layer with a selection bias, one call and staged, against the
    oracle layer with the same bias; the statistics of the GEMM-mode router."""
    wl = Workload("selbias-bf16", T=1024, d=256, N=16, k=4, f=256, capacity_factor=1.0)
    inp = synth.make_inputs(wl)
    cfg = moe.config_from_workload(wl)
    dl = moe.to_device(inp, cfg)
    sb = synth.make_selection_bias(2, wl.N, "normal")
    dl.selection_bias = gu.cuda_tensor(sb)
    staged = gu.staged_layer(dl)
    y, st, flags = gu.layer_fwd(dl)
    assert flags == 0 and staged["flags"] == 0
    np.testing.assert_array_equal(y, staged["y"])
    rel, n, flips = compare_layer(inp, wl, y, staged["idx"], staged["row_map"], staged["logits"],
                                  tol=2e-2, selection_bias=sb)
    # the bias changed the routing (else this test would not exercise it)
    plain = orc.topk(staged["logits"].astype(np.float64), wl.k)
    assert np.any(plain != staged["idx"])
    # statistics on the GPU's own logits and routing
    g = staged["logits"].astype(np.float64)
    check_route_extras(st, g, staged["idx"], wl.T, wl.k, wl.N)
    kept = st["kept"]
    assert st["avg_tokens_per_expert"][0] == np.float32(kept.sum() / wl.N)
    zl = orc.router_z_loss(g)
    assert abs(float(st["z_loss"][0]) - zl) <= z_loss_tolerance(g, wl.N)
