"""GPU parity of the whole layer (routed experts on the tcgen05 grouped GEMM,
shared expert, combine) against the fp64 oracle, at sizes the oracle finishes in
seconds that still span several tiles and ragged tails.

Tolerances (relative Frobenius error of the layer output): 1e-5 for the fp32
layer and 2e-2 for bf16 compute with fp32 accumulation."""
import numpy as np
import pytest
import torch

from expert_router_gemm_b200 import configs, synth
from expert_router_gemm_b200.configs import Workload
from oracle import moe_oracle as orc

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from expert_router_gemm_b200 import moe  # noqa: E402
from tests import gpu_util as gu  # noqa: E402
from tests.layer_check import compare_layer  # noqa: E402

TOL_F32 = 1e-5
TOL_BF16 = 2e-2

SMALL = [
    # ragged tiles: d = 320 leaves a 64-column tail in the down projection's
    # 256-column tiles, f = 192 a 64-column tail in the 128-column SwiGLU tiles
    Workload("ragged-bf16", T=700, d=320, N=8, k=2, f=192, capacity_factor=1.1),
    Workload("finegrained-bf16", T=1024, d=512, N=128, k=8, f=256, capacity_factor=1.0),
    Workload("shared-bf16", T=520, d=256, N=16, k=4, f=128, f_shared=192, capacity_factor=1.25),
    Workload("skewed-bf16", T=2048, d=256, N=8, k=2, f=512, capacity_factor=1.25,
             bias_pattern=configs.SKEW.bias_pattern, bias_beta_gamma=configs.SKEW_BETA_GAMMA),
    Workload("topN-bf16", T=300, d=128, N=8, k=8, f=128, capacity_factor=1.0),
    Workload("manytiles-bf16", T=1536, d=1024, N=4, k=2, f=1024, capacity_factor=1.0),
    # the largest top-k (32 slots per token) and an odd one (the combine's
    # generic slot loop), the latter with a shared expert
    Workload("top32-bf16", T=512, d=256, N=64, k=32, f=128, capacity_factor=1.25),
    Workload("top3-shared-bf16", T=600, d=192, N=12, k=3, f=192, f_shared=64, capacity_factor=1.0),
    # the largest expert count with the largest top-k
    Workload("n256-top32-bf16", T=256, d=128, N=256, k=32, f=64, capacity_factor=1.25),
    # degenerate shapes: one token (capacity 1), top-1 routing, one expert (a
    # dense SwiGLU MLP with weight 1; the router's one column padded to 64)
    Workload("one-token-bf16", T=1, d=128, N=8, k=2, f=128, capacity_factor=1.0),
    Workload("top1-bf16", T=700, d=256, N=16, k=1, f=192, capacity_factor=1.0),
    Workload("one-expert-bf16", T=300, d=128, N=1, k=1, f=128, capacity_factor=1.0),
]

F32 = [
    configs.TINY,
    # ragged everywhere: d and f off every tile edge, an odd top-k, a shared expert
    Workload("odd-f32", T=300, d=100, N=6, k=3, f=72, f_shared=40, capacity_factor=1.25, dtype="f32"),
]


def _run(w: Workload, align=0):
    inp = synth.make_inputs(w)
    cfg = moe.config_from_workload(w, seg_align=align)
    dl = moe.to_device(inp, cfg)
    staged = gu.staged_layer(dl)
    y, st, flags = gu.layer_fwd(dl)
    assert flags == 0 and staged["flags"] == 0
    return inp, staged, y, st


@pytest.mark.parametrize("w", F32, ids=[w.name for w in F32])
def test_fp32_layers(w):
    inp, staged, y, st = _run(w)
    np.testing.assert_array_equal(y, staged["y"])
    rel, n, flips = compare_layer(inp, w, y, staged["idx"], staged["row_map"], staged["logits"],
                                  tol=TOL_F32)
    assert n == w.T - flips
    ref = orc.layer_forward(inp.x, inp.w_router, inp.bias, inp.w1, inp.w3, inp.w2, k=w.k,
                            capacity_factor=w.capacity_factor, bf16=False, tokens=[])
    np.testing.assert_array_equal(st["kept"], ref.disp.kept)
    np.testing.assert_allclose(st["z_mean"], ref.stats.z_mean, rtol=1e-5)


@pytest.mark.parametrize("w", SMALL, ids=[w.name for w in SMALL])
def test_small_bf16_layers(w):
    inp, staged, y, st = _run(w)
    np.testing.assert_array_equal(y, staged["y"])          # one-call layer == staged steps
    rel, n, flips = compare_layer(inp, w, y, staged["idx"], staged["row_map"], staged["logits"],
                                  tol=TOL_BF16)
    assert n >= w.T - 3 * flips
    print(f"{w.name}: rel_frob={rel:.3e} over {n} tokens, {flips} near-tie flips")


@pytest.mark.parametrize("align", [1, 32])
def test_segment_alignment_variants(align):
    w = SMALL[1]
    inp, staged, y, st = _run(w, align=align)
    compare_layer(inp, w, y, staged["idx"], staged["row_map"], staged["logits"], tol=TOL_BF16,
                  align=align)


_VARIANT_SCRIPT = r"""
import sys
sys.path.insert(0, {root!r})
from expert_router_gemm_b200 import synth, moe
from expert_router_gemm_b200.configs import Workload
from tests import gpu_util as gu
from tests.layer_check import compare_layer
w = Workload("variant", T=1500, d=320, N=6, k=2, f=192, f_shared=128, capacity_factor=1.1)
inp = synth.make_inputs(w)
dl = moe.to_device(inp, moe.config_from_workload(w))
st = gu.staged_layer(dl)
assert st["flags"] == 0
rel, n, flips = compare_layer(inp, w, st["y"], st["idx"], st["row_map"], st["logits"], tol=2e-2)
y, _, flags = gu.layer_fwd(dl)        # GEMM1 gathers the token rows of x itself
assert flags == 0
import numpy as np
np.testing.assert_array_equal(y, st["y"])
print("REL", rel)
"""


@pytest.mark.parametrize("cta_group,gather", [("1", "lsu"), ("2", "lsu"), ("1", "tma"), ("2", "tma")])
def test_grouped_gemm_cta_group_variants(cta_group, gather):
    """Both tile shapes of the grouped GEMM (one CTA per 128x256 tile, or CTA
    pairs per 256x256 tile), each with both ways the layer pass gathers token
    rows (cp.async copies or tile::gather4 TMA loads), on a ragged layer with a
    shared expert: the staged path against the oracle, the one-call layer bit
    for bit against the staged path.  The choices are made once per process, so
    each variant runs in its own process."""
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, MOE_FFN_CTA_GROUP=cta_group, MOE_GATHER=gather)
    r = subprocess.run([sys.executable, "-c", _VARIANT_SCRIPT.format(root=root)], env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "REL" in r.stdout


def test_capacity_zero_gives_shared_only():
    w = Workload("cap0-shared", T=96, d=128, N=4, k=2, f=64, f_shared=128, capacity_factor=0.0)
    inp, staged, y, st = _run(w)
    assert int(st["num_dropped"][0]) == w.T * w.k
    x64 = orc.as_f64(inp.x)
    want = orc.swiglu_ffn(x64, inp.ws1, inp.ws3, inp.ws2, True)
    got = gu.y_as_f64(y)
    assert orc.rel_frobenius(got, want) <= TOL_BF16


def test_deterministic_repeat():
    w = SMALL[2]
    inp = synth.make_inputs(w)
    dl = moe.to_device(inp, moe.config_from_workload(w))
    a, sa, _ = gu.layer_fwd(dl)
    b, sb, _ = gu.layer_fwd(dl)
    np.testing.assert_array_equal(a, b)
    for key in sa:
        np.testing.assert_array_equal(sa[key], sb[key])


def test_empty_layer():
    w = Workload("empty", T=0, d=128, N=8, k=2, f=128)
    inp = synth.make_inputs(w)
    dl = moe.to_device(inp, moe.config_from_workload(w))
    y, st, flags = gu.layer_fwd(dl)
    assert flags == 0 and y.shape == (0, 128)
    assert np.all(st["counts"] == 0) and np.all(st["kept"] == 0) and st["num_dropped"][0] == 0


_OVERLAP_SCRIPT = r"""
import sys
sys.path.insert(0, {root!r})
import numpy as np
from expert_router_gemm_b200 import synth, moe
from expert_router_gemm_b200.configs import Workload
from tests import gpu_util as gu
out = []
for w in (Workload("ov-pairs", T=1536, d=512, N=8, k=2, f=384, f_shared=128, capacity_factor=1.1),
          Workload("ov-single", T=1024, d=256, N=32, k=4, f=256, capacity_factor=1.25),
          Workload("ov-f32", T=300, d=100, N=6, k=3, f=72, capacity_factor=1.25, dtype="f32")):
    dl = moe.to_device(synth.make_inputs(w), moe.config_from_workload(w))
    y, st, flags = gu.layer_fwd(dl)
    assert flags == 0
    out.append(y.view(np.uint8).tobytes())
    out.append(b"".join(np.ascontiguousarray(st[k]).tobytes() for k in sorted(st)))
import hashlib
print("DIGEST", hashlib.sha256(b"".join(out)).hexdigest())
"""


def test_overlapped_launches_change_no_result():
    """Kernels launched to overlap the end of their predecessor (the default)
    give the same bytes as plain launches (MOE_PDL=0): layer outputs and every
    statistic, for CTA-pair and single-CTA GEMMs and the fp32 layer."""
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    digests = []
    for pdl in ("1", "0"):
        env = dict(os.environ, MOE_PDL=pdl)
        r = subprocess.run([sys.executable, "-c", _OVERLAP_SCRIPT.format(root=root)], env=env,
                           capture_output=True, text=True, timeout=600)
        assert r.returncode == 0, r.stdout + r.stderr
        digests.append([l for l in r.stdout.splitlines() if l.startswith("DIGEST")][0])
    assert digests[0] == digests[1]
