"""The grouped GEMM's wait-timeout path, made to run out without a fault.

Every mbarrier wait in the tcgen05 kernels is bounded.  moe_set_wait_limit_ns
shortens the bound of the bf16 grouped GEMM's pipeline waits (a stage's
operands, a free stage, an accumulator) to a few hundred nanoseconds, which
ordinary loads and MMAs outlast, so those waits give up on a normal small
layer.  The kernel must then raise MOE_FLAG_WAIT_TIMEOUT (moe_read_flags reports
MOE_ERR_DEVICE), wait with the full bound for its own copies and MMAs in flight,
free its tensor memory and return; the CUDA context stays usable, and the next
call with the default bound is correct.  No wait is left without a bound and
nothing traps: the failure is a status the host reads."""
import numpy as np
import pytest
import torch

from expert_router_gemm_b200 import synth
from expert_router_gemm_b200.configs import Workload

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from expert_router_gemm_b200 import moe  # noqa: E402
from tests import gpu_util as gu  # noqa: E402
from tests.layer_check import compare_layer  # noqa: E402

SHORT_NS = 300


@pytest.mark.parametrize("w", [
    Workload("timeout-pairs", T=4096, d=1024, N=8, k=2, f=1024, capacity_factor=1.25),    # CTA pairs
    Workload("timeout-single", T=2048, d=1024, N=64, k=4, f=512, capacity_factor=1.0),    # single CTAs
], ids=lambda w: w.name)
def test_pipeline_wait_timeout_is_reported_and_the_next_call_is_correct(w):
    inp = synth.make_inputs(w)
    dl = moe.to_device(inp, moe.config_from_workload(w))
    cfg = dl.cfg
    lb, _, _ = moe.moe_workspace_size(cfg)
    ws = torch.empty(lb, dtype=torch.uint8, device="cuda")
    y = torch.zeros((w.T, w.d), dtype=moe.act_dtype(cfg), device="cuda")
    moe.moe_set_wait_limit_ns(SHORT_NS)
    try:
        moe.moe_layer_fwd(cfg, dl.weights(), dl.x, y, None, ws)
        flags = moe.moe_read_flags(ws)          # waits for the stream: the call has returned
    finally:
        moe.moe_set_wait_limit_ns(0)
    assert flags & moe.MOE_FLAG_WAIT_TIMEOUT, f"flags {flags:#x}"
    assert torch.cuda.synchronize() is None     # no sticky CUDA error

    # default bound again: the same layer is correct and raises nothing
    staged = gu.staged_layer(dl)
    y2, _, flags2 = gu.layer_fwd(dl)
    assert flags2 == 0 and staged["flags"] == 0
    np.testing.assert_array_equal(y2, staged["y"])
    compare_layer(inp, w, y2, staged["idx"], staged["row_map"], staged["logits"], tol=2e-2)


def test_fp8_pipeline_wait_timeout_is_reported_and_the_next_call_is_correct():
    """The same for the block-scaled FP8 grouped GEMM (single CTAs, the default
    shape): a short bound makes its pipeline waits run out, the call returns
    with MOE_FLAG_WAIT_TIMEOUT, and the next call with the default bound gives
    the bytes the layer gave before."""
    w = Workload("timeout-mx", T=2048, d=1024, N=8, k=2, f=1024, capacity_factor=1.25)
    inp = synth.make_inputs(w)
    cfg = moe.config_from_workload(w, gemm="mxfp8")
    dl = moe.to_device(inp, cfg)
    dl.quantize_mx()
    before, _, f0 = gu.layer_fwd(dl)
    assert f0 == 0
    lb, _, _ = moe.moe_workspace_size(cfg)
    ws = torch.empty(lb, dtype=torch.uint8, device="cuda")
    y = torch.zeros((w.T, w.d), dtype=moe.act_dtype(cfg), device="cuda")
    moe.moe_set_wait_limit_ns(SHORT_NS)
    try:
        moe.moe_layer_fwd(cfg, dl.weights(), dl.x, y, None, ws)
        flags = moe.moe_read_flags(ws)
    finally:
        moe.moe_set_wait_limit_ns(0)
    assert flags & moe.MOE_FLAG_WAIT_TIMEOUT, f"flags {flags:#x}"
    assert torch.cuda.synchronize() is None
    after, _, f1 = gu.layer_fwd(dl)
    assert f1 == 0
    np.testing.assert_array_equal(after, before)


def test_router_pipeline_wait_timeout_is_reported_and_the_next_call_is_correct():
    """The tensor-core router GEMM (CTA pairs, K split) under the short bound:
    moe_route returns with MOE_FLAG_WAIT_TIMEOUT, and with the default bound
    again it gives the routing it gave before, bit for bit."""
    w = Workload("timeout-router", T=4096, d=2048, N=128, k=8, f=128, capacity_factor=1.0)
    inp = synth.make_inputs(w, experts=False)
    cfg = moe.config_from_workload(w)
    x, wr = gu.cuda_tensor(inp.x), gu.cuda_tensor(inp.w_router)

    def route():
        idx = torch.full((w.T, w.k), -7, dtype=torch.int32, device="cuda")
        wt = torch.full((w.T, w.k), float("nan"), dtype=torch.float32, device="cuda")
        ws = gu.op_workspace(cfg)
        moe.moe_route(cfg, x, wr, None, None, None, idx, wt, None, ws)
        flags = moe.moe_read_flags(ws)
        return gu.host(idx), gu.host(wt), flags

    idx0, wt0, f0 = route()
    assert f0 == 0
    moe.moe_set_wait_limit_ns(SHORT_NS)
    try:
        _, _, flags = route()
    finally:
        moe.moe_set_wait_limit_ns(0)
    assert flags & moe.MOE_FLAG_WAIT_TIMEOUT, f"flags {flags:#x}"
    assert torch.cuda.synchronize() is None
    idx1, wt1, f1 = route()
    assert f1 == 0
    np.testing.assert_array_equal(idx1, idx0)
    np.testing.assert_array_equal(wt1, wt0)
