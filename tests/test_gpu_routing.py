"""GPU parity of routing and dispatch against the fp64 oracle.

Routing indices, the permutation (row map, segment offsets, permuted rows), the
drop mask and the expert counts must be bit-exact given identical fp32 logits,
which reach the GPU through the test entry point moe_route_from_logits.  The
routing weights and the load-balance statistics are fp32 on the GPU and fp64 in
the oracle: relative tolerance 2e-6 (a few fp32 ulps of the softmax)."""
import numpy as np
import pytest
import torch

from expert_router_gemm_b200 import synth
from oracle import moe_oracle as orc

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from expert_router_gemm_b200 import moe  # noqa: E402
from tests import gpu_util as gu  # noqa: E402
from tests.layer_check import check_route_extras, logit_bound  # noqa: E402

W_RTOL = 2e-6


def _check_route(T, N, k, pattern, seed=0):
    logits = synth.make_logits(seed, T, N, pattern)
    cfg = moe.make_config(T=T, d=64, N=N, k=k, f=64, capacity_factor=1.0, dtype="bf16")
    idx, w, st, flags = gu.route_from_logits(cfg, logits)
    assert flags == 0
    g = logits.astype(np.float64)
    want_idx = orc.topk(g, k)
    np.testing.assert_array_equal(idx, want_idx)
    s = orc.softmax(g)
    np.testing.assert_allclose(w, orc.topk_weights(s, want_idx), rtol=W_RTOL, atol=1e-7)
    ref = orc.aux_stats(want_idx, s, N)
    np.testing.assert_array_equal(st["counts"], np.bincount(want_idx.reshape(-1), minlength=N))
    np.testing.assert_allclose(st["y_frac"], ref.y_frac, rtol=1e-6, atol=0)
    np.testing.assert_allclose(st["z_mean"], ref.z_mean, rtol=1e-5, atol=1e-7)
    np.testing.assert_allclose(st["l_aux_p3"][0], ref.l_aux_p3, rtol=1e-5)
    np.testing.assert_allclose(st["l_aux_switch"][0], ref.l_aux_switch, rtol=1e-5)
    check_route_extras(st, g, want_idx, T, k, N)


@pytest.mark.parametrize("N,k", [(8, 1), (8, 2), (8, 8), (5, 3), (16, 4), (33, 7), (64, 32),
                                 (128, 8), (256, 8), (256, 1), (1, 1)])
@pytest.mark.parametrize("pattern", ["normal", "ties", "zeros", "onehot", "skewed"])
def test_route_from_logits_bitexact(N, k, pattern):
    for T in (1, 37, 300):
        _check_route(T, N, k, pattern, seed=T)


def test_route_from_logits_many_tokens():
    _check_route(8192, 128, 8, "normal", seed=3)
    _check_route(16384, 8, 2, "skewed", seed=4)


@pytest.mark.parametrize("T,d,N,k,dtype,bias", [
    (300, 128, 8, 2, "f32", False),      # CUDA-core router, fp32 x
    (257, 512, 8, 2, "bf16", True),      # CUDA-core router (N <= 32)
    (300, 320, 33, 4, "bf16", False),    # tensor-core router, N not a multiple of 16
    (1000, 256, 64, 8, "bf16", True),
    (300, 4096, 128, 8, "bf16", False),
    (129, 1024, 100, 6, "bf16", True),
    (4800, 256, 256, 8, "bf16", False),  # more tiles than SMs: 128-wide expert tiles
    (640, 7168, 256, 8, "bf16", True),
])
def test_route_gemm_logits(T, d, N, k, dtype, bias):
    """Router GEMM against the oracle's fp64 logits; the top-k taken on the GPU's
    own fp32 logits is checked as a property (larger logit first, ties to the
    lower index), and agrees with the oracle's except at near ties."""
    x = synth.normal_f32(7, 1, (T, d))
    if dtype == "bf16":
        x = synth.f32_to_bf16_bits(x)
    wr = synth.normal_f32(7, 2, (d, N)) * np.float32(1 / np.sqrt(d))
    b = synth.normal_f32(7, 3, (N,)) if bias else None
    cfg = moe.make_config(T=T, d=d, N=N, k=k, f=64, capacity_factor=1.0, dtype=dtype)
    logits = torch.full((T, N), float("nan"), device="cuda")
    idx = torch.full((T, k), -1, dtype=torch.int32, device="cuda")
    wt = torch.zeros((T, k), device="cuda")
    ws = gu.op_workspace(cfg)
    moe.moe_route(cfg, gu.cuda_tensor(x), gu.cuda_tensor(wr), None if b is None else gu.cuda_tensor(b),
                  None, logits, idx, wt, None, ws)
    assert moe.moe_read_flags(ws) == 0
    g = gu.host(logits).astype(np.float64)
    ref = orc.router_logits(x, wr, b)
    assert np.all(np.abs(g - ref) <= logit_bound(x, wr, b))
    got = gu.host(idx)
    # property: the selection is the top-k of the GPU's own logits (ties -> lower index)
    for t in range(T):
        sel = list(got[t])
        key = sorted(range(N), key=lambda e: (-g[t, e], e))[:k]
        assert sel == key, (t, sel, key)
    differ = np.any(got != orc.topk(ref, k), axis=1)
    assert differ.sum() <= max(1, T // 500)


@pytest.mark.parametrize("d,N,bias", [(256, 8, True), (320, 33, False), (512, 128, True),
                                      (1024, 256, True)])
def test_route_gemm_exact_on_one_hot_tokens(d, N, bias):
    """Token t = unit vector e_(t mod d): every logit is one product 1 * w, so
    the router GEMM must return the fp32 weight exactly (plus the bias, one fp32
    addition).  This pins the exact three-way bf16 split of the weights and the
    coverage of every K slab and expert tile, which the accumulation bound of
    the random-input test is too loose to see."""
    T = max(d, 300)
    x = np.zeros((T, d), np.float32)
    x[np.arange(T), np.arange(T) % d] = 1.0
    x = synth.f32_to_bf16_bits(x)
    wr = synth.normal_f32(8, 2, (d, N)) * np.float32(1 / np.sqrt(d))
    b = synth.normal_f32(8, 3, (N,)) if bias else None
    cfg = moe.make_config(T=T, d=d, N=N, k=min(N, 4), f=64, capacity_factor=1.0)
    logits = torch.full((T, N), float("nan"), device="cuda")
    idx = torch.empty((T, cfg.k), dtype=torch.int32, device="cuda")
    wt = torch.empty((T, cfg.k), device="cuda")
    ws = gu.op_workspace(cfg)
    moe.moe_route(cfg, gu.cuda_tensor(x), gu.cuda_tensor(wr), None if b is None else gu.cuda_tensor(b),
                  None, logits, idx, wt, None, ws)
    want = wr[np.arange(T) % d]
    if b is not None:
        want = want + b[None, :]          # one fp32 addition, round to nearest
    np.testing.assert_array_equal(gu.host(logits), want)


def test_route_nonfinite_flag():
    logits = synth.make_logits(0, 64, 8, "normal")
    logits[5, 3] = np.nan
    logits[9, 0] = np.inf
    cfg = moe.make_config(T=64, d=64, N=8, k=2, f=64)
    idx, w, st, flags = gu.route_from_logits(cfg, logits)
    assert flags & moe.MOE_FLAG_NONFINITE_LOGITS
    # the other tokens are routed as usual, and every index stays in range
    ok = np.ones(64, bool)
    ok[[5, 9]] = False
    np.testing.assert_array_equal(idx[ok], orc.topk(logits[ok].astype(np.float64), 2))
    assert idx.min() >= 0 and idx.max() < 8


def _check_dispatch(T, N, k, d, cap, align, dtype, pattern, seed=0):
    logits = synth.make_logits(seed, T, N, pattern)
    idx = orc.topk(logits.astype(np.float64), k)
    if dtype == "bf16":
        x = synth.f32_to_bf16_bits(synth.normal_f32(seed, 99, (T, d)))
    else:
        x = synth.normal_f32(seed, 99, (T, d))
    cfg = moe.make_config(T=T, d=d, N=N, k=k, f=64, capacity=cap, dtype=dtype, seg_align=align)
    r = gu.dispatch(cfg, gu.cuda_tensor(x), gu.cuda_tensor(idx))
    assert r["flags"] == 0
    want = orc.dispatch(idx, N, cap, align)
    np.testing.assert_array_equal(r["row_map"], want.row_map)
    np.testing.assert_array_equal(r["seg_off"], want.seg_off)
    np.testing.assert_array_equal(r["seg_count"], want.kept)
    np.testing.assert_array_equal(r["stats"]["counts"], want.counts)
    np.testing.assert_array_equal(r["stats"]["kept"], want.kept)
    assert int(r["stats"]["num_dropped"][0]) == want.num_dropped
    avg = orc.load_metrics(want.counts, want.kept, T, k).avg_tokens_per_expert
    assert r["stats"]["avg_tokens_per_expert"][0] == np.float32(avg)
    rows = orc.permuted_rows(x, want)
    for row, xr in rows.items():
        assert np.array_equal(r["xp"][row], xr), row


@pytest.mark.parametrize("T,N,k,d,cap,align,dtype,pattern", [
    (256, 8, 2, 128, 80, 128, "f32", "normal"),
    (300, 8, 2, 64, 40, 128, "bf16", "skewed"),
    (257, 16, 4, 64, 70, 32, "bf16", "normal"),
    (100, 5, 5, 64, 100, 1, "bf16", "ties"),
    (64, 4, 1, 64, 0, 8, "bf16", "normal"),          # capacity 0: everything dropped
    (50, 3, 2, 64, 1000, 16, "f32", "normal"),       # capacity >= T: nothing dropped
    (333, 8, 2, 64, 60, 128, "bf16", "onehot"),      # one over-full expert, others empty
    (1, 8, 2, 64, 1, 128, "bf16", "normal"),
    (1000, 128, 8, 256, 62, 128, "bf16", "normal"),
    (777, 256, 8, 128, 24, 128, "bf16", "skewed"),
    (129, 64, 32, 64, 80, 64, "bf16", "normal"),     # k = 32
])
def test_dispatch_bitexact(T, N, k, d, cap, align, dtype, pattern):
    _check_dispatch(T, N, k, d, cap, align, dtype, pattern)


def test_route_then_dispatch_bitexact():
    # the GPU's own top-k feeds the GPU dispatch; both match the oracle on the same logits
    T, N, k = 4096, 128, 8
    logits = synth.make_logits(11, T, N, "skewed")
    cfg = moe.make_config(T=T, d=64, N=N, k=k, f=64, capacity_factor=1.0, dtype="bf16")
    idx, _, _, _ = gu.route_from_logits(cfg, logits)
    x = synth.f32_to_bf16_bits(synth.normal_f32(1, 98, (T, 64)))
    r = gu.dispatch(cfg, gu.cuda_tensor(x), gu.cuda_tensor(idx))
    want = orc.dispatch(orc.topk(logits.astype(np.float64), k), N, orc.capacity(1.0, T, k, N), 128)
    np.testing.assert_array_equal(r["row_map"], want.row_map)
    np.testing.assert_array_equal(r["seg_off"], want.seg_off)
    assert want.num_dropped > 0


def test_dispatch_bad_index_flag():
    T, N, k = 40, 8, 2
    idx = orc.topk(synth.make_logits(2, T, N, "normal").astype(np.float64), k)
    idx[3, 1] = 8        # out of range
    idx[7, 0] = -1       # negative
    idx[11, 1] = idx[11, 0]  # repeated within the row
    x = synth.f32_to_bf16_bits(synth.normal_f32(2, 97, (T, 64)))
    cfg = moe.make_config(T=T, d=64, N=N, k=k, f=64, capacity=T, dtype="bf16")
    r = gu.dispatch(cfg, gu.cuda_tensor(x), gu.cuda_tensor(idx))
    assert r["flags"] & moe.MOE_FLAG_BAD_EXPERT_INDEX
    assert r["row_map"][3, 1] == -1 and r["row_map"][7, 0] == -1 and r["row_map"][11, 1] == -1
    # valid slots are ranked as if the invalid ones were absent
    clean = idx.copy()
    keep = np.ones_like(idx, bool)
    keep[3, 1] = keep[7, 0] = keep[11, 1] = False
    assert r["stats"]["counts"].sum() == keep.sum()


def test_empty_batch():
    cfg = moe.make_config(T=0, d=64, N=8, k=2, f=64, capacity_factor=1.25)
    idx, w, st, flags = gu.route_from_logits(cfg, np.zeros((0, 8), np.float32))
    assert flags == 0 and idx.shape == (0, 2)
    assert np.all(st["counts"] == 0) and np.all(st["y_frac"] == 0) and st["l_aux_p3"][0] == 0
    assert st["z_loss"][0] == 0 and st["load_std"][0] == 0 and st["top2_ratio"][0] == 0
    r = gu.dispatch(cfg, torch.empty((0, 64), dtype=torch.int16, device="cuda"),
                    torch.empty((0, 2), dtype=torch.int32, device="cuda"))
    assert np.all(r["seg_off"] == 0) and np.all(r["seg_count"] == 0)
    assert r["stats"]["avg_tokens_per_expert"][0] == 0


@pytest.mark.parametrize("T,d,N,k,bias,sel", [
    (300, 256, 8, 2, True, False),      # N <= 64: 64-expert tiles, K split four ways
    (8192, 4096, 128, 8, False, False),  # the Qwen3-shaped router: CTA pairs, two K splits
    (1000, 512, 100, 6, True, True),     # ragged N, selection bias
    (640, 7168, 256, 8, True, False),    # N = 256
    (33, 1024, 128, 8, False, True),     # fewer tokens than one tile
])
def test_router_decisions_match_routing_its_own_logits(T, d, N, k, bias, sel):
    """moe_route on the tensor cores (the router GEMM's K-slice partial sums, then
    the routing kernel) and the routing kernel fed
    the router's own fp32 logits through moe_route_from_logits take the same
    decisions bit for bit, and report the same statistics within the fp32
    summation-order difference of the two."""
    x = synth.f32_to_bf16_bits(synth.normal_f32(11, 1, (T, d)))
    wr = synth.normal_f32(11, 2, (d, N)) * np.float32(1 / np.sqrt(d))
    b = synth.normal_f32(11, 3, (N,)) if bias else None
    sb = synth.make_selection_bias(11, N) if sel else None
    cfg = moe.make_config(T=T, d=d, N=N, k=k, f=64, capacity_factor=1.0, dtype="bf16")
    logits = torch.full((T, N), float("nan"), device="cuda")
    idx = torch.full((T, k), -1, dtype=torch.int32, device="cuda")
    wt = torch.full((T, k), float("nan"), device="cuda")
    ws = gu.op_workspace(cfg)
    bufs, st = gu.new_stats(N)
    moe.moe_route(cfg, gu.cuda_tensor(x), gu.cuda_tensor(wr), None if b is None else gu.cuda_tensor(b),
                  None if sb is None else gu.cuda_tensor(sb), logits, idx, wt, st, ws)
    assert moe.moe_read_flags(ws) == 0
    lg = gu.host(logits)
    assert np.all(np.isfinite(lg))
    idx2, w2, st2, flags2 = gu.route_from_logits(cfg, lg, sb)
    assert flags2 == 0
    np.testing.assert_array_equal(gu.host(idx), idx2)
    np.testing.assert_array_equal(gu.host(wt), w2)
    fused = gu.stats_host(bufs)
    np.testing.assert_array_equal(fused["counts"], st2["counts"])
    for key in ("y_frac", "top2_ratio", "load_std"):
        np.testing.assert_array_equal(fused[key], st2[key], err_msg=key)
    for key in ("z_mean", "l_aux_p3", "l_aux_switch", "z_loss"):
        np.testing.assert_allclose(fused[key], st2[key], rtol=1e-5, atol=1e-9, err_msg=key)


def test_layer_with_a_router_split_made_once_is_unchanged():
    """moe_layer_fwd with the bf16 split of W_r passed in (moe_router_split, made
    once) gives the same bytes as the layer that splits W_r itself."""
    from expert_router_gemm_b200.configs import Workload
    w = Workload("presplit", T=1024, d=512, N=128, k=8, f=256, capacity_factor=1.0)
    inp = synth.make_inputs(w)
    dl = moe.to_device(inp, moe.config_from_workload(w))
    y0, st0, f0 = gu.layer_fwd(dl)
    dl.split_router()
    y1, st1, f1 = gu.layer_fwd(dl)
    assert f0 == 0 and f1 == 0
    np.testing.assert_array_equal(y0, y1)
    for key in st0:
        np.testing.assert_array_equal(st0[key], st1[key], err_msg=key)


@pytest.mark.parametrize("T,d,N,k,bias,sel,dtype", [
    (300, 256, 8, 2, True, False, "bf16"),       # 64-expert tiles, K split four ways
    (8192, 4096, 128, 8, False, False, "bf16"),  # the Qwen3-shaped router: CTA pairs
    (1000, 512, 100, 6, True, True, "bf16"),     # ragged N, selection bias
    (640, 7168, 256, 8, True, False, "bf16"),    # N = 256: two 128-expert column tiles
    (256, 128, 8, 2, True, False, "f32"),        # fp32 layer: no tensor-core router, split ignored
])
def test_route_with_split_matches_route(T, d, N, k, bias, sel, dtype):
    """moe_route_with_split, given the split that moe_router_split made once,
    writes the bytes that moe_route writes: logits, indices, weights and every
    statistic."""
    if dtype == "bf16":
        x = synth.f32_to_bf16_bits(synth.normal_f32(12, 1, (T, d)))
    else:
        x = synth.normal_f32(12, 1, (T, d))
    wr = synth.normal_f32(12, 2, (d, N)) * np.float32(1 / np.sqrt(d))
    b = gu.cuda_tensor(synth.normal_f32(12, 3, (N,))) if bias else None
    sb = gu.cuda_tensor(synth.make_selection_bias(12, N)) if sel else None
    cfg = moe.make_config(T=T, d=d, N=N, k=k, f=64, capacity_factor=1.0, dtype=dtype)
    xd, wrd = gu.cuda_tensor(x), gu.cuda_tensor(wr)
    split = torch.empty(moe.moe_router_split_bytes(d, N), dtype=torch.uint8, device="cuda")
    moe.moe_router_split(wrd, d, N, split)

    def run(with_split):
        logits = torch.full((T, N), float("nan"), device="cuda")
        idx = torch.full((T, k), -1, dtype=torch.int32, device="cuda")
        wt = torch.full((T, k), float("nan"), device="cuda")
        ws = gu.op_workspace(cfg)
        bufs, st = gu.new_stats(N)
        if with_split:
            moe.moe_route_with_split(cfg, xd, wrd, split, b, sb, logits, idx, wt, st, ws)
        else:
            moe.moe_route(cfg, xd, wrd, b, sb, logits, idx, wt, st, ws)
        assert moe.moe_read_flags(ws) == 0
        return gu.host(logits), gu.host(idx), gu.host(wt), gu.stats_host(bufs)

    lg0, idx0, wt0, st0 = run(False)
    lg1, idx1, wt1, st1 = run(True)
    np.testing.assert_array_equal(lg1, lg0)
    np.testing.assert_array_equal(idx1, idx0)
    np.testing.assert_array_equal(wt1, wt0)
    for key in ("y_frac", "z_mean", "l_aux_p3", "l_aux_switch", "counts", "z_loss", "load_std", "top2_ratio"):
        np.testing.assert_array_equal(st1[key], st0[key], err_msg=key)
