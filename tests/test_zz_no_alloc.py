"""moe_dispatch_static — the dispatch entry point that allocates nothing.

Some callers cannot allocate device memory where they dispatch tokens: their
device memory belongs to another allocator, or they allocate only at start-up
and may not call cudaMalloc (which can fail and synchronises the device) while
serving.  moe_dispatch_static serves them with a fixed scratch array inside the
library instead of a caller workspace.  This test calls it through the C ABI
twice in a row on each case (the second call finds the first call's leftovers
in the shared array, and the second case the first case's) and requires the
same bytes as moe_dispatch, the entry point with a workspace, and the oracle's
dispatch itself: dispatch results are integers and copied rows, so the
tolerance of the dispatch tests applies, which is exact equality.  The file
sorts last so that a run stopping at the first failure has run every other test
before it.
"""
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

CASES = [  # (T, N, k, d, capacity, dtype, logits pattern, seed)
    (4096, 128, 8, 256, 240, "bf16", "skewed", 1),
    (333, 8, 2, 128, 60, "f32", "onehot", 2),
]


def _static_dispatch(cfg, x, idx):
    T, N, k = cfg.T, cfg.N, cfg.k
    _, _, max_rows = moe.moe_workspace_size(cfg)
    row_map = torch.full((T, k), -7, dtype=torch.int32, device="cuda")
    seg_off = torch.full((N + 1,), -7, dtype=torch.int32, device="cuda")
    seg_count = torch.full((N,), -7, dtype=torch.int32, device="cuda")
    xp = torch.zeros((max_rows, cfg.d), dtype=moe.act_dtype(cfg), device="cuda")
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    bufs, st = gu.new_stats(N)
    moe.moe_dispatch_static(cfg, x, idx, row_map, seg_off, seg_count, xp, st, flags)
    torch.cuda.synchronize()
    return dict(row_map=gu.host(row_map), seg_off=gu.host(seg_off), seg_count=gu.host(seg_count),
                xp=gu.host(xp), stats=gu.stats_host(bufs), flags=int(flags.item()))


def test_static_dispatch_matches_workspace_dispatch_twice():
    for (T, N, k, d, cap, dtype, pattern, seed) in CASES:
        idx = orc.topk(synth.make_logits(seed, T, N, pattern).astype(np.float64), k)
        x = synth.normal_f32(seed, 55, (T, d))
        if dtype == "bf16":
            x = synth.f32_to_bf16_bits(x)
        cfg = moe.make_config(T=T, d=d, N=N, k=k, f=64, capacity=cap, dtype=dtype)
        xt, it = gu.cuda_tensor(x), gu.cuda_tensor(idx)
        want = gu.dispatch(cfg, xt, it)
        ref = orc.dispatch(idx, N, cap, 128)
        for call in range(2):
            got = _static_dispatch(cfg, xt, it)
            assert got["flags"] == 0 and want["flags"] == 0, call
            for key in ("row_map", "seg_off", "seg_count", "xp"):
                np.testing.assert_array_equal(got[key], want[key], err_msg=f"{key}, call {call}")
            for key in ("counts", "kept", "num_dropped"):
                np.testing.assert_array_equal(got["stats"][key], want["stats"][key],
                                              err_msg=f"{key}, call {call}")
            # the oracle's capacity clip and permutation, compared directly
            np.testing.assert_array_equal(got["row_map"], ref.row_map, err_msg=f"oracle row_map, call {call}")
            np.testing.assert_array_equal(got["seg_off"], ref.seg_off, err_msg=f"oracle seg_off, call {call}")
            np.testing.assert_array_equal(got["seg_count"], ref.kept, err_msg=f"oracle kept, call {call}")
            np.testing.assert_array_equal(got["stats"]["counts"], ref.counts)
            assert int(got["stats"]["num_dropped"][0]) == ref.num_dropped
            t_of, j_of = np.nonzero(ref.row_map >= 0)
            np.testing.assert_array_equal(got["xp"][ref.row_map[t_of, j_of]], x[t_of],
                                          err_msg=f"permuted rows, call {call}")


def test_static_dispatch_rejects_batches_beyond_its_scratch():
    T, N = 32 * (moe.MOE_DISPATCH_STATIC_MAX_CELLS // 256) + 1, 256   # one block too many
    cfg = moe.make_config(T=T, d=64, N=N, k=8, f=64, capacity_factor=1.0)
    one = torch.zeros(64, dtype=torch.int32, device="cuda")
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_dispatch_static(cfg, one, one, one, one, one, one, None)
    assert ei.value.status == moe.MOE_ERR_WORKSPACE
