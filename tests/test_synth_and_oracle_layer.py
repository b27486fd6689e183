"""Seeded input generator checks and whole-layer invariants of the oracle (CPU)."""
import numpy as np
import torch

from expert_router_gemm_b200 import configs, synth
from oracle import moe_oracle as orc


def test_synth_deterministic_and_shaped():
    w = configs.TINY
    a = synth.make_inputs(w)
    b = synth.make_inputs(w)
    for name in ("x", "w_router", "w1", "w3", "w2"):
        np.testing.assert_array_equal(getattr(a, name), getattr(b, name))
    assert a.x.shape == (w.T, w.d) and a.x.dtype == np.float32
    assert a.w1.shape == (w.N, w.d, w.f) and a.w2.shape == (w.N, w.f, w.d)
    # N(0, 1/fan_in): sample std close to 1/sqrt(d)
    assert abs(a.w1.std() * np.sqrt(w.d) - 1.0) < 0.02


def test_synth_bf16_matches_torch_rounding():
    v = synth.normal_f32(3, 77, (10000,)) * np.float32(3.0)
    want = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(synth.f32_to_bf16_bits(v), want)
    np.testing.assert_array_equal(synth.bf16_bits_to_f32(want),
                                  torch.from_numpy(v).to(torch.bfloat16).float().numpy())


def test_workload_capacities():
    want = {"tiny-fp32": 80, "mixtral-8x7b-shaped": 1280, "qwen3-moe-shaped": 512,
            "deepseek-v3-shaped": 320, "skewed-stress": 5120}
    for name, w in configs.WORKLOADS.items():
        assert orc.capacity(w.capacity_factor, w.T, w.k, w.N) == want[name]


def test_skew_bias_reproduces_reported_load():
    # "ms-swift + Megatron：MoE模型加速10倍实测" §2.1: experts 0 and 3 take 68% of the
    # tokens, experts 5 and 6 under 3%
    w = configs.SKEW
    inp = synth.make_inputs(w, experts=False)
    g = orc.router_logits(inp.x, inp.w_router, inp.bias)
    share = np.bincount(orc.topk(g, w.k).reshape(-1), minlength=w.N) / (w.T * w.k)
    assert abs(share[0] + share[3] - 0.68) <= 0.01
    assert share[5] + share[6] < 0.03


def test_oracle_layer_tiny_invariants():
    w = configs.TINY
    inp = synth.make_inputs(w)
    res = orc.layer_forward(inp.x, inp.w_router, inp.bias, inp.w1, inp.w3, inp.w2, k=w.k,
                            capacity_factor=w.capacity_factor, bf16=False)
    assert res.capacity == 80
    assert abs(res.stats.y_frac.sum() - 1.0) < 1e-12
    assert abs(res.stats.z_mean.sum() - 1.0) < 1e-12
    assert res.y.shape == (w.T, w.d) and np.all(np.isfinite(res.y))
    # sampled evaluation agrees with the full evaluation (BLAS blocking differs)
    sub = orc.layer_forward(inp.x, inp.w_router, inp.bias, inp.w1, inp.w3, inp.w2, k=w.k,
                            capacity_factor=w.capacity_factor, bf16=False, tokens=[5, 0, 200])
    np.testing.assert_allclose(sub.y, res.y[[5, 0, 200]], rtol=1e-11, atol=1e-13)


def test_oracle_empty_batch():
    w = configs.TINY
    inp = synth.make_inputs(w, T=0)
    res = orc.layer_forward(inp.x, inp.w_router, None, inp.w1, inp.w3, inp.w2, k=2,
                            capacity_factor=1.25, bf16=False)
    assert res.capacity == 0 and res.y.shape == (0, w.d)
    assert np.all(res.disp.counts == 0) and res.disp.seg_off[-1] == 0
