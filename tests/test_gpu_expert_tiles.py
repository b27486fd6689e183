"""The grouped expert GEMM (moe_expert_ffn) on groups whose sizes sit on every
tile edge, in both tile shapes, against the fp64 oracle's SwiGLU FFN row by row.

Group sizes 0, 1, 15-17, 63-65, 127-129, 191-193, 255-257, 320 and 383 put the
last tile of a group at every edge of the tile shapes: an empty group, a
single-CTA tile with one row, a TMEM lane quarter's worth (16 rows) and its
neighbours, half or all of its 128 rows, and a CTA-pair tile whose second CTA
holds no rows, some or all.  d = 320 and f = 192 leave 64-column tails in both
GEMMs' column tiles.  Each shape choice is made once per process, so each runs
in its own process.

Tolerance: per row, relative error <= 1e-2 of the oracle row's norm (bf16
operands with fp32 accumulation; h rounded to bf16 as the oracle does, the
output rounded to bf16 once); rows past the groups stay zero."""
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

_SCRIPT = r"""
import sys
sys.path.insert(0, {root!r})
import numpy as np
import torch
from expert_router_gemm_b200 import moe, synth
from expert_router_gemm_b200.configs import Workload
from oracle import moe_oracle as orc
from tests import gpu_util as gu

COUNTS = [0, 1, 15, 16, 17, 63, 64, 65, 127, 128, 129, 191, 192, 193, 255, 256, 257, 320, 383]
N = len(COUNTS)
w = Workload("tile-edges", T=2048, d=320, N=N, k=2, f=192, capacity_factor=2.0)
inp = synth.make_inputs(w)
cfg = moe.config_from_workload(w)
_, _, max_rows = moe.moe_workspace_size(cfg)
assert sum(COUNTS) <= max_rows
dl = moe.to_device(inp, cfg)
seg_count = np.array(COUNTS, np.int32)
seg_off = np.zeros(N + 1, np.int32)
seg_off[1:] = np.cumsum(seg_count)
src = (np.arange(max_rows) * 7) % w.T          # token behind each permuted row
xp_bits = np.ascontiguousarray(inp.x[src])
xp = gu.cuda_tensor(xp_bits)
h = torch.zeros((max_rows, w.f), dtype=torch.bfloat16, device="cuda")
out = torch.zeros((max_rows, w.d), dtype=torch.bfloat16, device="cuda")
ws = gu.op_workspace(cfg)
moe.moe_expert_ffn(cfg, xp, gu.cuda_tensor(seg_off), gu.cuda_tensor(seg_count), dl.weights(), h, out, ws)
assert moe.moe_read_flags(ws) == 0
y = gu.y_as_f64(gu.host(out.view(torch.int16)))
x64 = orc.as_f64(xp_bits)
worst = 0.0
for g in range(N):
    r0, c = int(seg_off[g]), int(seg_count[g])
    if c == 0:
        continue
    ref = orc.swiglu_ffn(x64[r0:r0 + c], inp.w1[g], inp.w3[g], inp.w2[g], round_h_bf16=True)
    err = np.linalg.norm(y[r0:r0 + c] - ref, axis=1) / np.maximum(np.linalg.norm(ref, axis=1), 1e-30)
    worst = max(worst, float(err.max()))
    assert err.max() <= 1e-2, (g, c, int(err.argmax()), float(err.max()))
assert not y[seg_off[N]:].any(), "rows past the groups were written"
print("WORST", worst)
"""


@pytest.mark.parametrize("cta_group", ["1", "2"])
def test_expert_ffn_group_sizes_on_tile_edges(cta_group):
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, MOE_FFN_CTA_GROUP=cta_group)
    r = subprocess.run([sys.executable, "-c", _SCRIPT.format(root=root)], env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "WORST" in r.stdout
