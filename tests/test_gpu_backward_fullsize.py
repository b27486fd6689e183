"""The layer backward at the Qwen3-MoE-shaped bench size (T=8192, d=4096,
N=128, k=8, f=1536), against the fp64 backward oracle on sampled outputs: dx of
every token whose routing the fp32 and fp64 logits agree on, the router weight
gradient in full, and the expert weight gradients of four experts (busiest,
median, least busy and one more).  Relative Frobenius error <= 2e-2 per tensor,
as for the small cases; a token routed differently at a near tie changes the
gradients it feeds by one row of a few hundred, far inside the tolerance."""
import numpy as np
import pytest
import torch

from expert_router_gemm_b200 import configs, synth
from oracle import moe_backward as bwd
from oracle import moe_oracle as orc

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from expert_router_gemm_b200 import moe  # noqa: E402
from tests import gpu_util as gu  # noqa: E402

TOL = 2e-2


def test_backward_qwen3_shaped_sampled():
    w = configs.QWEN3
    inp = synth.make_inputs(w)
    cfg = moe.config_from_workload(w)
    dl = moe.to_device(inp, cfg)
    dy = synth.f32_to_bf16_bits(synth.normal_f32(21, 77, (w.T, w.d)))
    aux, z = 0.01, 1e-3
    T, d, N, k, f = w.T, w.d, w.N, w.k, w.f

    ws = gu.op_workspace(cfg)
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    wt = torch.empty((T, k), device="cuda")
    moe.moe_route(cfg, dl.x, dl.w_router, dl.bias, None, None, idx, wt, None, ws)
    g_idx = np.sort(gu.host(idx), axis=1)
    ref_idx = np.sort(orc.topk(orc.router_logits(inp.x, inp.w_router, inp.bias), k), axis=1)
    same = np.all(g_idx == ref_idx, axis=1)
    assert same.sum() >= T - max(2, T // 500)

    dev = "cuda"
    g = dict(dx=torch.zeros((T, d), dtype=torch.int16, device=dev),
             dw_router=torch.empty((d, N), device=dev),
             dw1=torch.empty((N, d, f), device=dev), dw3=torch.empty((N, d, f), device=dev),
             dw2=torch.empty((N, f, d), device=dev))
    wsb = torch.zeros(moe.moe_backward_workspace_size(cfg), dtype=torch.uint8, device=dev)
    moe.moe_layer_bwd(cfg, dl.weights(), dl.x, gu.cuda_tensor(dy), aux, z, moe.make_grads(**g), wsb)
    assert moe.moe_read_flags(wsb) == 0
    counts = np.bincount(ref_idx.reshape(-1), minlength=N)
    order = np.argsort(counts, kind="stable")
    experts = [int(order[-1]), int(order[N // 2]), int(order[np.nonzero(counts[order] > 0)[0][0]]), 7]
    got = {name: gu.host(g[name][experts]) for name in ("dw1", "dw3", "dw2")}
    got["dx"] = gu.y_as_f64(gu.host(g["dx"]))
    got["dw_router"] = gu.host(g["dw_router"])
    del g, wsb
    torch.cuda.empty_cache()

    ref = bwd.layer_backward(inp.x, inp.w_router, inp.bias, inp.w1, inp.w3, inp.w2, orc.as_f64(dy), k=k,
                             capacity_factor=w.capacity_factor, aux_weight=aux, z_weight=z,
                             weight_experts=experts)
    report = []
    for name, a, b in (("dx", got["dx"][same], ref.dx[same]), ("dw_router", got["dw_router"], ref.dw_router),
                       ("dw1", got["dw1"], ref.dw1), ("dw3", got["dw3"], ref.dw3), ("dw2", got["dw2"], ref.dw2)):
        assert np.all(np.isfinite(a)), name
        rel = orc.rel_frobenius(np.asarray(a, np.float64), b)
        report.append(f"{name} {rel:.2e}")
        assert rel <= TOL, (name, rel)
    print("qwen3 backward:", ", ".join(report), f"; {T - same.sum()} routing flips; experts {experts}")
