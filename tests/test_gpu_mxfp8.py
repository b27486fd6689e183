"""GPU parity of the block-scaled FP8 expert path against the FP8 oracle.

Weight quantization and the quantizing dispatch start from bf16 values, so the
E4M3 codes and the scale bytes are bit-exact.  The layer output is compared with
the oracle's FP8 layer (same quantization of x and the weights, h quantized
from its fp64 value): relative Frobenius error <= 1e-2.  Derivation: the GPU
rounds the expert outputs and y to bf16 (relative rounding error about
2^-9 / sqrt(3) ~ 1.1e-3 each) and forms h in fp32, so an h element within
fp32 error of a rounding boundary of its E4M3 code can take the neighbouring
code (one code step, 2^-3 relative at most, in a tiny fraction of elements);
1e-2 leaves a margin of about 4x over the two roundings.  The FP8 layer's own
accuracy against the exact bf16 layer is reported, not gated."""
import numpy as np
import pytest
import torch

from expert_router_gemm_b200 import synth
from expert_router_gemm_b200.configs import Workload
from oracle import moe_oracle as orc
from oracle import mxfp8 as mxo

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from expert_router_gemm_b200 import moe  # noqa: E402
from tests import gpu_util as gu  # noqa: E402
from tests.layer_check import compare_layer  # noqa: E402

TOL_MX = 1e-2
U8 = torch.uint8


def _bf16_weights(seed, G, K, N):
    w = synth.normal_f32(seed, 5, (G, K, N)) * np.float32(1 / np.sqrt(K))
    # special blocks: all zeros, tiny (E4M3 subnormals), large, and block maxima on
    # both sides of the 1.75 * 2^k boundary of the exponent rule
    w[0, :32, 0] = 0.0
    w[0, 32:64, 1] *= np.float32(2.0 ** -40)
    w[0, 64:96, 2] *= np.float32(2.0 ** 40)
    w[0, 96, 3] = np.float32(1.75)
    w[0, 97:128, 3] = np.float32(0.25)
    w[0, 128 % K, 4] = np.float32(1.7578125)
    return synth.f32_to_bf16_bits(w)


@pytest.mark.parametrize("G,K,N", [(3, 256, 384), (1, 128, 128), (2, 512, 256)])
def test_mx_quantize_weight_bitexact(G, K, N):
    w = _bf16_weights(G + K, G, K, N)
    codes = torch.full((G, N, K), 0xAB, dtype=U8, device="cuda")
    sf = torch.full((G * N * K // 32,), 0xAB, dtype=U8, device="cuda")
    moe.moe_mx_quantize_weight(gu.cuda_tensor(w), G, K, N, codes, sf)
    codes, sf = gu.host(codes), gu.host(sf).reshape(G, -1)
    for g in range(G):
        q = mxo.quantize_weight(w[g])
        np.testing.assert_array_equal(codes[g], q.codes())
        np.testing.assert_array_equal(mxo.sf_unpack(sf[g], N, K // 32), q.scale_bytes())


def _dispatch_mx(cfg, x_dev, idx_dev):
    T, N, k, d = cfg.T, cfg.N, cfg.k, cfg.d
    _, _, max_rows = moe.moe_workspace_size(cfg)
    row_map = torch.full((T, k), -7, dtype=torch.int32, device="cuda")
    seg_off = torch.full((N + 1,), -7, dtype=torch.int32, device="cuda")
    seg_count = torch.full((N,), -7, dtype=torch.int32, device="cuda")
    codes = torch.zeros((max_rows, d), dtype=U8, device="cuda")
    sf = torch.zeros(moe.mx_sf_bytes(max_rows, d), dtype=U8, device="cuda")
    ws = gu.op_workspace(cfg)
    bufs, st = gu.new_stats(N)
    moe.moe_dispatch_mx(cfg, x_dev, idx_dev, row_map, seg_off, seg_count, codes, sf, st, ws)
    return dict(row_map=row_map, seg_off=seg_off, seg_count=seg_count, codes=codes, sf=sf,
                stats=gu.stats_host(bufs), flags=moe.moe_read_flags(ws), max_rows=max_rows, ws=ws)


@pytest.mark.parametrize("T,N,k,d,cap", [(300, 8, 2, 256, 80), (257, 16, 4, 384, 70), (1000, 128, 8, 128, 62),
                                         (64, 4, 1, 128, 0)])
def test_dispatch_mx_bitexact(T, N, k, d, cap):
    logits = synth.make_logits(T, T, N, "skewed")
    idx = orc.topk(logits.astype(np.float64), k)
    xf = synth.normal_f32(T, 99, (T, d)) * np.float32(3.0)
    xf[0, :32] = 0.0
    xf[1, :64] *= np.float32(2.0 ** -50)
    x = synth.f32_to_bf16_bits(xf)
    cfg = moe.make_config(T=T, d=d, N=N, k=k, f=128, capacity=cap, gemm="mxfp8")
    r = _dispatch_mx(cfg, gu.cuda_tensor(x), gu.cuda_tensor(idx))
    assert r["flags"] == 0
    want = orc.dispatch(idx, N, cap, 128)
    np.testing.assert_array_equal(gu.host(r["row_map"]), want.row_map)
    np.testing.assert_array_equal(gu.host(r["seg_off"]), want.seg_off)
    np.testing.assert_array_equal(r["stats"]["kept"], want.kept)
    codes, sf = gu.host(r["codes"]), gu.host(r["sf"])
    q = mxo.mx_quantize(orc.as_f64(x))
    want_codes, want_sf = q.codes(), q.scale_bytes()
    gsf = mxo.sf_unpack(sf, r["max_rows"], d // 32)
    t_idx, j_idx = np.nonzero(want.row_map >= 0)
    rows = want.row_map[t_idx, j_idx]
    np.testing.assert_array_equal(codes[rows], want_codes[t_idx])
    np.testing.assert_array_equal(gsf[rows], want_sf[t_idx])


SMALL = [
    Workload("mx-basic", T=1024, d=512, N=8, k=2, f=512, capacity_factor=1.25),
    Workload("mx-ragged-n", T=700, d=384, N=8, k=2, f=384, capacity_factor=1.1),
    Workload("mx-finegrained", T=1024, d=256, N=128, k=8, f=256, capacity_factor=1.0),
    Workload("mx-shared", T=520, d=256, N=16, k=4, f=128, f_shared=256, capacity_factor=1.25),
    Workload("mx-deep-k", T=512, d=2048, N=4, k=2, f=1024, capacity_factor=1.0),
    # degenerate shapes: one token, top-1 routing over one expert
    Workload("mx-one-token", T=1, d=256, N=8, k=2, f=128, capacity_factor=1.0),
    Workload("mx-one-expert", T=300, d=128, N=1, k=1, f=256, capacity_factor=1.0),
]


def _run_mx(w: Workload):
    inp = synth.make_inputs(w)
    cfg = moe.config_from_workload(w, gemm="mxfp8")
    dl = moe.to_device(inp, cfg)
    dl.quantize_mx()
    y, st, flags = gu.layer_fwd(dl)
    assert flags == 0
    return inp, cfg, dl, y, st


@pytest.mark.slow
def test_mx_layer_at_the_bench_expert_shapes():
    """The FP8 layer at the Qwen3-shaped workload's per-expert shapes (d=4096,
    f=1536, top-8, capacity 512 rows per expert, about 500 rows each) with 32
    of its 128 experts and T=2048: GEMM1 accumulates over K=4096 and GEMM2
    writes 16 column tiles per row block, as in the benchmark's FP8 launches.
    256 sampled tokens against the FP8 oracle, within the same tolerance."""
    from dataclasses import replace
    from expert_router_gemm_b200 import configs
    w = replace(configs.QWEN3, name="qwen3-shaped-N32-T2048", T=2048, N=32)
    assert moe.moe_capacity(moe.config_from_workload(w)) == 512
    inp, cfg, dl, y, st = _run_mx(w)
    ws = gu.op_workspace(cfg)
    logits = torch.empty((w.T, w.N), device="cuda")
    idx = torch.empty((w.T, w.k), dtype=torch.int32, device="cuda")
    wt = torch.empty((w.T, w.k), device="cuda")
    moe.moe_route(cfg, dl.x, dl.w_router, dl.bias, None, logits, idx, wt, None, ws)
    r = _dispatch_mx(cfg, dl.x, idx)
    rel, n, flips = compare_layer(inp, w, y, gu.host(idx), gu.host(r["row_map"]), gu.host(logits),
                                  tol=TOL_MX, sample=256, mxfp8=True)
    print(f"{w.name}: rel_frob vs FP8 oracle {rel:.3e} ({n} tokens, {flips} flips)")


@pytest.mark.parametrize("w", SMALL, ids=[w.name for w in SMALL])
def test_mx_layer_vs_oracle(w):
    inp, cfg, dl, y, st = _run_mx(w)
    # routing is the bf16 layer's: run the staged routing for the GPU's own choice
    T, N, k = w.T, w.N, w.k
    ws = gu.op_workspace(cfg)
    logits = torch.empty((T, N), device="cuda")
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    wt = torch.empty((T, k), device="cuda")
    moe.moe_route(cfg, dl.x, dl.w_router, dl.bias, None, logits, idx, wt, None, ws)
    r = _dispatch_mx(cfg, dl.x, idx)
    rel, n, flips = compare_layer(inp, w, y, gu.host(idx), gu.host(r["row_map"]), gu.host(logits),
                                  tol=TOL_MX, mxfp8=True)
    assert n >= w.T - 3 * flips
    # the one-call layer equals the staged FP8 steps bit for bit
    _, _, max_rows = moe.moe_workspace_size(cfg)
    h8 = torch.zeros((max_rows, w.f), dtype=U8, device="cuda")
    hsf = torch.zeros(moe.mx_sf_bytes(max_rows, w.f), dtype=U8, device="cuda")
    out = torch.zeros((max_rows, w.d), dtype=torch.int16, device="cuda")
    wts = dl.weights()
    moe.moe_expert_ffn_mx(cfg, r["codes"], r["sf"], r["seg_off"], r["seg_count"], wts, h8, hsf, out, ws)
    sh = None
    if w.f_shared:
        hs = torch.zeros((T, w.f_shared), dtype=torch.int16, device="cuda")
        sh = torch.zeros((T, w.d), dtype=torch.int16, device="cuda")
        moe.moe_shared_expert_ffn(cfg, dl.x, wts, hs, sh, ws)
    y2 = torch.zeros((T, w.d), dtype=torch.int16, device="cuda")
    moe.moe_combine(cfg, out, r["row_map"], wt, sh, y2, ws)
    assert moe.moe_read_flags(ws) == 0
    np.testing.assert_array_equal(gu.host(y2), y)
    # accuracy of FP8 itself against the exact layer (reported)
    ref = orc.layer_forward(inp.x, inp.w_router, inp.bias, inp.w1, inp.w3, inp.w2, k=w.k,
                            capacity_factor=w.capacity_factor, bf16=True, ws1=inp.ws1, ws3=inp.ws3,
                            ws2=inp.ws2, tokens=np.arange(min(T, 128)))
    acc = orc.rel_frobenius(gu.y_as_f64(y)[:min(T, 128)], ref.y)
    print(f"{w.name}: rel_frob vs FP8 oracle {rel:.3e} ({n} tokens, {flips} flips); "
          f"vs exact bf16 layer {acc:.3e}")
    assert acc < 0.1


def test_mx_h_codes_match_oracle():
    """GEMM1's epilogue output (FP8 codes of h and their scales) against the
    oracle's quantization of the exact h: equal except for rare elements at an
    E4M3 rounding boundary (h is formed in fp32 on the GPU, in fp64 here)."""
    w = SMALL[0]
    inp, cfg, dl, y, st = _run_mx(w)
    T, N, k, d, f = w.T, w.N, w.k, w.d, w.f
    idx = orc.topk(orc.router_logits(inp.x, inp.w_router, inp.bias), k)
    r = _dispatch_mx(cfg, dl.x, gu.cuda_tensor(idx))
    max_rows = r["max_rows"]
    h8 = torch.zeros((max_rows, f), dtype=U8, device="cuda")
    hsf = torch.zeros(moe.mx_sf_bytes(max_rows, f), dtype=U8, device="cuda")
    out = torch.zeros((max_rows, d), dtype=torch.int16, device="cuda")
    ws = gu.op_workspace(cfg)
    moe.moe_expert_ffn_mx(cfg, r["codes"], r["sf"], r["seg_off"], r["seg_count"], dl.weights(), h8, hsf, out, ws)
    assert moe.moe_read_flags(ws) == 0
    h8, hsf = gu.host(h8), mxo.sf_unpack(gu.host(hsf), max_rows, f // 32)
    seg_off, seg_count = gu.host(r["seg_off"]), gu.host(r["seg_count"])
    rm = gu.host(r["row_map"])
    xq = mxo.mx_quantize(orc.as_f64(inp.x))
    total = same = same_sf = nblk = 0
    for e in range(N):
        lo, hi = seg_off[e], seg_off[e] + seg_count[e]
        t_idx, j_idx = np.nonzero((rm >= lo) & (rm < hi))
        if len(t_idx) == 0:
            continue
        order = np.argsort(rm[t_idx, j_idx])
        tok, rows = t_idx[order], rm[t_idx, j_idx][order]
        assert np.array_equal(rows, np.arange(lo, hi))
        xa = mxo.MxTensor(xq.q[tok], xq.e[tok]).dequantize()
        hq = mxo.mx_quantize(orc.silu(xa @ mxo.quantize_weight(inp.w1[e]).dequantize().T) *
                             (xa @ mxo.quantize_weight(inp.w3[e]).dequantize().T))
        total += hq.q.size
        same += int(np.sum(h8[rows] == hq.codes()))
        nblk += hq.e.size
        same_sf += int(np.sum(hsf[rows] == hq.scale_bytes()))
    assert same >= 0.999 * total, (same, total)
    assert same_sf >= 0.999 * nblk, (same_sf, nblk)


_MX_VARIANT_SCRIPT = r"""
import sys
sys.path.insert(0, {root!r})
import numpy as np
import torch
from expert_router_gemm_b200 import synth, moe
from expert_router_gemm_b200.configs import Workload
from tests import gpu_util as gu
from tests.layer_check import compare_layer
for w in (Workload("mxv-ragged", T=1500, d=384, N=6, k=2, f=384, capacity_factor=1.1),
          Workload("mxv-shared", T=700, d=256, N=8, k=2, f=256, f_shared=128, capacity_factor=1.25)):
    inp = synth.make_inputs(w)
    cfg = moe.config_from_workload(w, gemm="mxfp8")
    dl = moe.to_device(inp, cfg)
    dl.quantize_mx()
    y, st, flags = gu.layer_fwd(dl)
    assert flags == 0, flags
    ws = gu.op_workspace(cfg)
    logits = torch.empty((w.T, w.N), device="cuda")
    idx = torch.empty((w.T, w.k), dtype=torch.int32, device="cuda")
    wt = torch.empty((w.T, w.k), device="cuda")
    moe.moe_route(cfg, dl.x, dl.w_router, dl.bias, None, logits, idx, wt, None, ws)
    rm = np.asarray(gu.host(idx))   # routing only; the row map comes from the layer's own dispatch
    _, _, max_rows = moe.moe_workspace_size(cfg)
    row_map = torch.empty((w.T, w.k), dtype=torch.int32, device="cuda")
    seg_off = torch.empty(w.N + 1, dtype=torch.int32, device="cuda")
    seg_count = torch.empty(w.N, dtype=torch.int32, device="cuda")
    codes = torch.empty((max_rows, w.d), dtype=torch.uint8, device="cuda")
    sf = torch.empty(moe.mx_sf_bytes(max_rows, w.d), dtype=torch.uint8, device="cuda")
    moe.moe_dispatch_mx(cfg, dl.x, idx, row_map, seg_off, seg_count, codes, sf, None, ws)
    rel, n, flips = compare_layer(inp, w, y, rm, gu.host(row_map), gu.host(logits), tol=1e-2, mxfp8=True)
    print("REL", w.name, rel, n, flips)
"""


@pytest.mark.parametrize("cta_group", ["1", "2"])
def test_mx_gemm_cta_group_variants(cta_group):
    """Both tile shapes of the FP8 grouped GEMM (single CTAs with 128-row tiles,
    CTA pairs with 256-row tiles), each in its own process (the choice is made
    once per process)."""
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, MOE_FFN_CTA_GROUP=cta_group)
    r = subprocess.run([sys.executable, "-c", _MX_VARIANT_SCRIPT.format(root=root)], env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.count("REL") == 2, r.stdout
    print(r.stdout)
