"""GPU parity of the layer backward (moe_layer_bwd) against the fp64 backward
oracle (oracle/moe_backward.py, itself pinned to finite differences).

Every gradient tensor is compared by relative Frobenius error <= 2e-2, the bf16
layer tolerance: the GPU keeps o, dO, g, u, h, dG, dU, dXp and dx in bf16 (each
rounding 2^-9 relative at most) and accumulates in fp32, the oracle runs the
exact arithmetic of the same inputs in fp64.  The routing must agree: the test
cases are chosen without near ties between fp32 and fp64 logits (checked)."""
import numpy as np
import pytest
import torch

from expert_router_gemm_b200 import synth
from expert_router_gemm_b200.configs import Workload
from oracle import moe_backward as bwd
from oracle import moe_oracle as orc

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from expert_router_gemm_b200 import moe  # noqa: E402
from tests import gpu_util as gu  # noqa: E402

TOL = 2e-2
F32 = torch.float32
_BIAS16 = tuple((i % 3 - 1, i % 2) for i in range(16))

CASES = [
    (Workload("bwd-basic", T=256, d=256, N=8, k=2, f=256, capacity_factor=1.0), 0.01, 1e-3),
    (Workload("bwd-shared-bias", T=512, d=512, N=16, k=4, f=384, f_shared=256, capacity_factor=1.25,
              bias_pattern=_BIAS16, bias_beta_gamma=(0.25, -0.125)), 0.3, 0.2),
    (Workload("bwd-ragged", T=300, d=320, N=8, k=2, f=192, capacity_factor=1.1), 0.05, 0.0),
    (Workload("bwd-finegrained", T=768, d=256, N=128, k=8, f=128, capacity_factor=1.0, seed=1), 0.01, 1e-3),
    # wide routers (N > 64: the 128 x 128-tile router gradient kernels) with ragged T, d not a
    # multiple of 128 and N not a multiple of 4; and two 128-expert column tiles
    (Workload("bwd-wide-ragged", T=300, d=320, N=100, k=4, f=128, capacity_factor=1.1), 0.05, 1e-3),
    (Workload("bwd-n256", T=256, d=256, N=256, k=8, f=128, capacity_factor=1.25), 0.01, 1e-3),
    # ~256 rows per expert (the DeepSeek-shaped layer's tile occupancy)
    (Workload("bwd-256-rows", T=1024, d=256, N=8, k=2, f=256, capacity_factor=1.25), 0.01, 1e-3),
]


def _gpu_backward(dl, dy, aux, z):
    cfg = dl.cfg
    N, d, f, fs = cfg.N, cfg.d, cfg.f, cfg.f_shared
    dev = "cuda"
    g = dict(dx=torch.zeros((cfg.T, d), dtype=torch.int16, device=dev),
             dw_router=torch.full((d, N), float("nan"), dtype=F32, device=dev),
             drouter_bias=torch.full((N,), float("nan"), dtype=F32, device=dev),
             dw1=torch.full((N, d, f), float("nan"), dtype=F32, device=dev),
             dw3=torch.full((N, d, f), float("nan"), dtype=F32, device=dev),
             dw2=torch.full((N, f, d), float("nan"), dtype=F32, device=dev))
    if fs:
        g.update(dws1=torch.full((d, fs), float("nan"), dtype=F32, device=dev),
                 dws3=torch.full((d, fs), float("nan"), dtype=F32, device=dev),
                 dws2=torch.full((fs, d), float("nan"), dtype=F32, device=dev))
    ws = torch.zeros(moe.moe_backward_workspace_size(cfg), dtype=torch.uint8, device=dev)
    moe.moe_layer_bwd(cfg, dl.weights(), dl.x, gu.cuda_tensor(dy), aux, z, moe.make_grads(**g), ws)
    assert moe.moe_read_flags(ws) == 0
    return {k: gu.host(v) for k, v in g.items()}


@pytest.mark.parametrize("w,aux,z", CASES, ids=[c[0].name for c in CASES])
def test_layer_backward_vs_oracle(w, aux, z):
    _check_backward(w, aux, z)


def test_layer_backward_segments_aligned_to_64():
    """Segments padded to 64 rows: a 128- or 256-row GEMM tile of one expert
    reaches into the next expert's rows, which its epilogue must leave alone
    (about 37 kept rows per expert here)."""
    w = Workload("bwd-align64", T=300, d=256, N=16, k=2, f=128, capacity_factor=1.25)
    _check_backward(w, 0.05, 1e-3, seg_align=64)


def _check_backward(w, aux, z, seg_align=0):
    inp = synth.make_inputs(w)
    cfg = moe.config_from_workload(w, seg_align=seg_align)
    dl = moe.to_device(inp, cfg)
    dy = synth.f32_to_bf16_bits(synth.normal_f32(11, 77, (w.T, w.d)))
    # the routing of the GPU equals the oracle's (no near ties in these cases)
    ws = gu.op_workspace(cfg)
    idx = torch.empty((w.T, w.k), dtype=torch.int32, device="cuda")
    wt = torch.empty((w.T, w.k), device="cuda")
    moe.moe_route(cfg, dl.x, dl.w_router, dl.bias, None, None, idx, wt, None, ws)
    ref_idx = orc.topk(orc.router_logits(inp.x, inp.w_router, inp.bias), w.k)
    assert np.array_equal(np.sort(gu.host(idx), axis=1), np.sort(ref_idx, axis=1)), "routing flip"

    got = _gpu_backward(dl, dy, aux, z)
    ref = bwd.layer_backward(inp.x, inp.w_router, inp.bias, inp.w1, inp.w3, inp.w2, orc.as_f64(dy), k=w.k,
                             capacity_factor=w.capacity_factor, ws1=inp.ws1, ws3=inp.ws3, ws2=inp.ws2,
                             aux_weight=aux, z_weight=z)
    pairs = [("dx", gu.y_as_f64(got["dx"]), ref.dx), ("dw_router", got["dw_router"], ref.dw_router),
             ("dw1", got["dw1"], ref.dw1), ("dw3", got["dw3"], ref.dw3), ("dw2", got["dw2"], ref.dw2)]
    if inp.bias is not None:
        pairs.append(("drouter_bias", got["drouter_bias"], ref.dbias))
    if w.f_shared:
        pairs += [("dws1", got["dws1"], ref.dws1), ("dws3", got["dws3"], ref.dws3), ("dws2", got["dws2"], ref.dws2)]
    report = []
    for name, a, b in pairs:
        assert np.all(np.isfinite(a)), name
        rel = orc.rel_frobenius(np.asarray(a, np.float64), b)
        report.append(f"{name} {rel:.2e}")
        assert rel <= TOL, (name, rel)
    print(w.name, ", ".join(report))
    # experts that no kept token chose get exactly zero gradient
    fwd = orc.layer_forward(inp.x, inp.w_router, inp.bias, inp.w1, inp.w3, inp.w2, k=w.k,
                            capacity_factor=w.capacity_factor, tokens=[])
    kept = fwd.disp.row_map >= 0
    for e in range(w.N):
        if not np.any((fwd.idx == e) & kept):
            assert not np.any(got["dw1"][e]) and not np.any(got["dw2"][e])


def test_layer_backward_deterministic_and_empty():
    w, aux, z = CASES[1]
    inp = synth.make_inputs(w)
    cfg = moe.config_from_workload(w)
    dl = moe.to_device(inp, cfg)
    dy = synth.f32_to_bf16_bits(synth.normal_f32(12, 77, (w.T, w.d)))
    a, b = _gpu_backward(dl, dy, aux, z), _gpu_backward(dl, dy, aux, z)
    for key in a:
        assert np.array_equal(a[key].view(np.uint8), b[key].view(np.uint8)), key
    empty = moe.config_from_workload(w, T=0)
    dl0 = moe.to_device(synth.make_inputs(Workload("e", T=1, d=w.d, N=w.N, k=w.k, f=w.f, f_shared=w.f_shared,
                                                   bias_pattern=_BIAS16, bias_beta_gamma=(0.25, -0.125))),
                        empty)
    z0 = _gpu_backward(dl0, np.zeros((0, w.d), np.uint16), aux, z)
    for key in ("dw_router", "dw1", "dw3", "dw2", "dws1", "dws3", "dws2", "drouter_bias"):
        assert not np.any(z0[key]), key


def test_layer_backward_with_a_router_split_made_once_is_unchanged():
    """moe_layer_bwd with the bf16 split of W_r passed in (moe_router_split, made
    once) gives the gradients it gives when its forward recompute splits W_r
    itself, byte for byte (the wide router: CTA pairs)."""
    w, aux, z = CASES[3]
    inp = synth.make_inputs(w)
    dl = moe.to_device(inp, moe.config_from_workload(w))
    dy = synth.f32_to_bf16_bits(synth.normal_f32(12, 78, (w.T, w.d)))
    a = _gpu_backward(dl, dy, aux, z)
    dl.split_router()
    b = _gpu_backward(dl, dy, aux, z)
    for key in a:
        assert np.array_equal(a[key].view(np.uint8), b[key].view(np.uint8)), key


EDGE = [
    # capacity 0: every slot dropped, only the router path carries gradient
    (Workload("bwd-cap0", T=128, d=128, N=4, k=2, f=128, capacity_factor=0.0), 0.05, 0.01, None),
    # k = N: every expert chosen by every token
    (Workload("bwd-topN", T=200, d=128, N=4, k=4, f=128, capacity_factor=1.0), 0.05, 0.01, None),
    # one expert: the softmax is constant, the router gets only the z-loss gradient
    (Workload("bwd-one-expert", T=96, d=128, N=1, k=1, f=128, capacity_factor=1.0), 0.05, 0.01, None),
    # Aux-Loss-Free selection bias steering the choice (no gradient of its own)
    (Workload("bwd-selbias", T=256, d=256, N=8, k=2, f=256, capacity_factor=1.0), 0.01, 1e-3, "normal"),
]


@pytest.mark.parametrize("w,aux,z,sel", EDGE, ids=[c[0].name for c in EDGE])
def test_layer_backward_edge_cases(w, aux, z, sel):
    inp = synth.make_inputs(w)
    cfg = moe.config_from_workload(w)
    dl = moe.to_device(inp, cfg)
    sb = synth.make_selection_bias(3, w.N, sel) if sel else None
    if sb is not None:
        dl.selection_bias = gu.cuda_tensor(sb)
    dy = synth.f32_to_bf16_bits(synth.normal_f32(13, 77, (w.T, w.d)))
    got = _gpu_backward(dl, dy, aux, z)
    ref = bwd.layer_backward(inp.x, inp.w_router, inp.bias, inp.w1, inp.w3, inp.w2, orc.as_f64(dy), k=w.k,
                             capacity_factor=w.capacity_factor, aux_weight=aux, z_weight=z, selection_bias=sb)
    for name, a, b in (("dx", gu.y_as_f64(got["dx"]), ref.dx), ("dw_router", got["dw_router"], ref.dw_router),
                       ("dw1", got["dw1"], ref.dw1), ("dw3", got["dw3"], ref.dw3), ("dw2", got["dw2"], ref.dw2)):
        assert np.all(np.isfinite(a)), name
        if not np.any(b):
            assert not np.any(a), name          # exactly zero where the oracle is zero
            continue
        rel = orc.rel_frobenius(np.asarray(a, np.float64), b)
        assert rel <= TOL, (w.name, name, rel)


@pytest.mark.parametrize("cta_group", ["1", "2"])
def test_layer_backward_cta_group_variants(cta_group):
    """Both tile shapes of the backward GEMMs (single CTAs with 128-row tiles,
    CTA pairs with 256-row tiles) on every small case, each shape in its own
    process (the choice is made once per process)."""
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, MOE_BWD_CTA_GROUP=cta_group)
    sel = [__file__ + "::test_layer_backward_vs_oracle", __file__ + "::test_layer_backward_edge_cases",
           __file__ + "::test_layer_backward_segments_aligned_to_64"]
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider", *sel], env=env,
                       cwd=root, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
