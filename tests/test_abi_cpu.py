"""The C-ABI library on the CPU: it loads, exports every function that
include/moe.h declares, and validates arguments on the host (no GPU needed:
validation happens before any CUDA call)."""
import ctypes
import subprocess

import numpy as np
import pytest

from oracle import moe_oracle as orc

moe = pytest.importorskip("expert_router_gemm_b200.moe",
                          reason="libmoe.so not built (python -m expert_router_gemm_b200.build)")

OK = moe.MOE_OK
INVALID = moe.MOE_ERR_INVALID_ARG
UNSUP = moe.MOE_ERR_UNSUPPORTED
MISAL = moe.MOE_ERR_MISALIGNED
WS = moe.MOE_ERR_WORKSPACE


def test_exports_every_declared_function():
    declared = moe.header_functions()
    assert {"moe_route", "moe_route_from_logits", "moe_dispatch", "moe_expert_ffn",
            "moe_shared_expert_ffn", "moe_combine", "moe_layer_fwd", "moe_capacity",
            "moe_workspace_size", "moe_read_flags"} <= set(declared)
    out = subprocess.run(["nm", "-D", "--defined-only", moe.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    missing = [f for f in declared if f not in exported]
    assert not missing, missing
    for f in declared:
        assert hasattr(moe._lib, f)


def test_version_and_status_strings():
    assert "sm_100a" in moe.moe_version()
    for s in range(8):
        assert moe.moe_status_string(s).startswith("MOE_")
    assert moe.moe_status_string(99) == "MOE_ERR_UNKNOWN"


def _cap(T, N, k, cf, capacity=-1):
    cfg = moe.make_config(T=T, d=64, N=N, k=k, f=64, capacity_factor=cf, capacity=capacity)
    return moe.moe_capacity(cfg)


def test_capacity_matches_oracle():
    # the pages' worked example and the five workloads
    assert _cap(1024, 8, 1, 1.25) == 160
    assert _cap(1024, 8, 1, 1.0) == 128
    for (T, N, k, cf, want) in [(256, 8, 2, 1.25, 80), (4096, 8, 2, 1.25, 1280),
                                (8192, 128, 8, 1.0, 512), (8192, 256, 8, 1.25, 320),
                                (16384, 8, 2, 1.25, 5120)]:
        assert _cap(T, N, k, cf) == want
    rng = np.random.default_rng(0)
    for _ in range(500):
        T = int(rng.integers(0, 100000))
        N = int(rng.integers(1, 257))
        k = int(rng.integers(1, min(N, 32) + 1))
        cf = float(rng.choice([1.0, 1.1, 1.25, 1.5, 0.3, 2.0, rng.uniform(0, 4)]))
        assert _cap(T, N, k, cf) == orc.capacity(cf, T, k, N), (T, N, k, cf)
    assert _cap(100, 8, 2, 9.9, capacity=7) == 7


def test_capacity_invalid():
    for cf in (float("nan"), float("inf"), -1.0):
        cfg = moe.make_config(T=10, d=64, N=4, k=1, f=64, capacity_factor=cf)
        with pytest.raises(moe.MoeError) as ei:
            moe.moe_capacity(cfg)
        assert ei.value.status == INVALID
    cfg = moe.make_config(T=10**9, d=64, N=1, k=1, f=64, capacity_factor=1e6)
    with pytest.raises(moe.MoeError):
        moe.moe_capacity(cfg)


def _ws_status(**kw):
    base = dict(T=256, d=128, N=8, k=2, f=256, capacity_factor=1.25, dtype="f32")
    base.update(kw)
    cfg = moe.make_config(**base)
    lb, ob, mr = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_int64()
    return moe.raw_call("moe_workspace_size", ctypes.byref(cfg), ctypes.byref(lb),
                        ctypes.byref(ob), ctypes.byref(mr)), lb.value, ob.value, mr.value


def test_workspace_size_and_shape_checks():
    st, lb, ob, mr = _ws_status()
    assert st == OK and lb > ob > 0
    assert mr == min(256 * 2, 8 * 80) + 8 * 127
    assert _ws_status(k=9)[0] == INVALID              # k > N
    assert _ws_status(k=0)[0] == INVALID
    assert _ws_status(N=0)[0] == INVALID
    assert _ws_status(T=-1)[0] == INVALID
    assert _ws_status(N=300, k=2)[0] == UNSUP         # N > 256
    assert _ws_status(N=64, k=33)[0] == UNSUP         # k > 32
    assert _ws_status(dtype="bf16", d=96)[0] == UNSUP  # bf16 needs d % 64
    assert _ws_status(dtype="bf16", f=80)[0] == UNSUP  # bf16 needs f % 64
    assert _ws_status(d=126)[0] == UNSUP              # fp32 rows need 16-byte multiples
    assert _ws_status(T=0)[0] == OK
    cfg = moe.make_config(T=10, d=64, N=4, k=1, f=64)
    cfg.act_dtype = 7
    assert moe.raw_call("moe_workspace_size", ctypes.byref(cfg), None, None, None) == INVALID
    assert moe.raw_call("moe_workspace_size", None, None, None, None) == INVALID


# The integer "pointers" below are never dereferenced: every call returns from
# host-side validation before it touches CUDA.
def _route_status(cfg, x=0x10000, wr=0x20000, idx=0x30000, w=0x40000, ws=0x50000, ws_bytes=None):
    if ws_bytes is None:
        ws_bytes = moe.moe_workspace_size(cfg)[1]
    return moe.raw_call("moe_route", ctypes.byref(cfg), x, wr, None, None, None, idx, w, None, ws,
                        ctypes.c_size_t(ws_bytes), None)


def test_route_argument_validation():
    cfg = moe.make_config(T=256, d=128, N=8, k=2, f=256, capacity_factor=1.25, dtype="f32")
    assert _route_status(cfg, x=None) == INVALID
    assert _route_status(cfg, idx=None) == INVALID
    assert _route_status(cfg, x=0x10008) == MISAL
    assert _route_status(cfg, ws=None) == WS
    assert _route_status(cfg, ws_bytes=16) == WS
    assert _route_status(cfg, ws=0x50008) == MISAL
    bad = moe.make_config(T=256, d=128, N=8, k=9, f=256)
    assert _route_status(bad, ws_bytes=1 << 20) == INVALID


def test_route_with_split_argument_validation():
    # the same checks as moe_route, plus the split's alignment (never dereferenced here)
    cfg = moe.make_config(T=256, d=128, N=128, k=8, f=256, capacity_factor=1.0, dtype="bf16")
    ob = moe.moe_workspace_size(cfg)[1]

    def call(x=0x10000, split=0x60000, idx=0x30000, ws=0x50000, ws_bytes=ob):
        return moe.raw_call("moe_route_with_split", ctypes.byref(cfg), x, 0x20000, split, None, None, None,
                            idx, 0x40000, None, ws, ctypes.c_size_t(ws_bytes), None)

    assert call(split=0x60008) == MISAL
    assert call(x=None) == INVALID
    assert call(idx=None) == INVALID
    assert call(x=0x10008) == MISAL
    assert call(ws_bytes=16) == WS
    assert call(ws=None) == WS


def test_bias_update_argument_validation():
    cfg = moe.make_config(T=256, d=128, N=8, k=2, f=256, capacity_factor=1.25)
    f = ctypes.c_float

    def call(c, b=0x10000, counts=0x20000, gamma=1e-3):
        return moe.raw_call("moe_bias_update", ctypes.byref(c), b, counts, f(gamma), None)

    assert call(cfg, b=None) == INVALID
    assert call(cfg, counts=None) == INVALID
    assert call(cfg, gamma=float("nan")) == INVALID
    assert call(cfg, gamma=float("inf")) == INVALID
    assert call(moe.make_config(T=256, d=128, N=8, k=9, f=256)) == INVALID


def test_other_entry_points_validate():
    cfg = moe.make_config(T=64, d=128, N=8, k=2, f=128, capacity_factor=1.0, dtype="bf16")
    lb, ob, mr = moe.moe_workspace_size(cfg)
    c = ctypes.byref(cfg)
    sz = ctypes.c_size_t
    # dispatch: seg arrays required
    assert moe.raw_call("moe_dispatch", c, 0x1000, 0x2000, 0x3000, None, 0x5000, 0x6000, None,
                        0x7000, sz(ob), None) == INVALID
    assert moe.raw_call("moe_dispatch", c, 0x1008, 0x2000, 0x3000, 0x4000, 0x5000, 0x6000, None,
                        0x7000, sz(ob), None) == MISAL
    # expert ffn: weights required and aligned
    w = moe.moe_weights_t(0x100, None, 0x1000, 0x2000, None, None, None, None)
    assert moe.raw_call("moe_expert_ffn", c, 0x1000, 0x2000, 0x3000, ctypes.byref(w), 0x4000,
                        0x5000, 0x7000, sz(ob), None) == INVALID
    w = moe.moe_weights_t(0x100, None, 0x1000, 0x2008, 0x3000, None, None, None)
    assert moe.raw_call("moe_expert_ffn", c, 0x1000, 0x2000, 0x3000, ctypes.byref(w), 0x4000,
                        0x5000, 0x7000, sz(ob), None) == MISAL
    # shared expert needs f_shared > 0
    w = moe.moe_weights_t(0x100, None, 0x1000, 0x2000, 0x3000, 0x4000, 0x5000, 0x6000)
    assert moe.raw_call("moe_shared_expert_ffn", c, 0x1000, ctypes.byref(w), 0x4000, 0x5000,
                        0x7000, sz(ob), None) == INVALID
    # combine: y required, workspace checked
    assert moe.raw_call("moe_combine", c, 0x1000, 0x2000, 0x3000, None, None, 0x7000, sz(ob),
                        None) == INVALID
    assert moe.raw_call("moe_combine", c, 0x1000, 0x2000, 0x3000, None, 0x4000, 0x7000, sz(8),
                        None) == WS
    # layer: workspace must cover the layer size, not only the op size
    w = moe.moe_weights_t(0x100, None, 0x1000, 0x2000, 0x3000, None, None, None)
    assert moe.raw_call("moe_layer_fwd", c, ctypes.byref(w), 0x1000, 0x2000, None, 0x7000,
                        sz(ob), None) == WS
    assert moe.raw_call("moe_layer_fwd", c, None, 0x1000, 0x2000, None, 0x7000, sz(lb),
                        None) == INVALID
    # flags query validates its pointers
    assert moe.raw_call("moe_read_flags", None, sz(256), None, None) == INVALID


def test_router_split_alignment_is_checked_by_the_layer_calls():
    # a misaligned w_router_split is refused on the host, forward and backward alike
    cfg = moe.make_config(T=64, d=128, N=128, k=8, f=128, capacity_factor=1.0, dtype="bf16")
    lb, _, _ = moe.moe_workspace_size(cfg)
    bb = moe.moe_backward_workspace_size(cfg)
    c = ctypes.byref(cfg)
    sz = ctypes.c_size_t
    w = moe.make_weights(0x100, w1=0x1000, w3=0x2000, w2=0x3000, w_router_split=0x8008)
    assert moe.raw_call("moe_layer_fwd", c, ctypes.byref(w), 0x1000, 0x2000, None, 0x7000,
                        sz(lb), None) == MISAL
    g = moe.make_grads(dx=0x9000, dw_router=0xa000, dw1=0xb000, dw3=0xc000, dw2=0xd000)
    assert moe.raw_call("moe_layer_bwd", c, ctypes.byref(w), 0x1000, 0x2000, ctypes.c_float(0.01),
                        ctypes.c_float(1e-3), ctypes.byref(g), 0x7000, sz(bb), None) == MISAL


def test_header_documents_every_entry_point():
    text = open(moe.HEADER_PATH).read()
    for f in moe.header_functions():
        assert text.count(f) >= 1
    # each compute entry point cites the page section that defines it
    for f in ("moe_route", "moe_dispatch", "moe_expert_ffn", "moe_combine", "moe_capacity"):
        block = text[text.index(" * " + f + " "):]
        assert "§" in block[:900] or "section" in block[:900], f


def test_mxfp8_config_validation():
    ok = moe.make_config(T=256, d=256, N=8, k=2, f=384, gemm="mxfp8")
    lb_mx, ob_mx, rows = moe.moe_workspace_size(ok)
    lb, ob, rows2 = moe.moe_workspace_size(moe.make_config(T=256, d=256, N=8, k=2, f=384))
    assert rows == rows2 and ob_mx == ob and lb_mx > lb
    for bad in (moe.make_config(T=256, d=320, N=8, k=2, f=384, gemm="mxfp8"),    # d % 128
                moe.make_config(T=256, d=256, N=8, k=2, f=192, gemm="mxfp8"),    # f % 128
                moe.make_config(T=256, d=256, N=8, k=2, f=384, gemm="mxfp8", seg_align=64),
                moe.make_config(T=256, d=256, N=8, k=2, f=384, gemm="mxfp8", dtype="f32")):
        with pytest.raises(moe.MoeError) as ei:
            moe.moe_workspace_size(bad)
        assert ei.value.status == moe.MOE_ERR_UNSUPPORTED
    weird = moe.make_config(T=256, d=256, N=8, k=2, f=384)
    weird.gemm_format = 7
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_workspace_size(weird)
    assert ei.value.status == INVALID


def test_mx_entry_validation():
    q = lambda w=0x1000, G=2, K=256, N=128, c=0x2000, s=0x3000: moe.raw_call(  # noqa: E731
        "moe_mx_quantize_weight", w, ctypes.c_int64(G), K, N, c, s, None)
    assert q(K=100) == moe.MOE_ERR_UNSUPPORTED
    assert q(N=200) == moe.MOE_ERR_UNSUPPORTED
    assert q(w=None) == INVALID
    assert q(G=-1) == INVALID
    assert q(c=0x2008) == MISAL
    assert q(G=0, w=None, c=None, s=None) == moe.MOE_OK   # nothing to do, nothing launched
    plain = moe.make_config(T=256, d=256, N=8, k=2, f=384)
    mx = moe.make_config(T=256, d=256, N=8, k=2, f=384, gemm="mxfp8")
    _, ob, _ = moe.moe_workspace_size(mx)
    sz = ctypes.c_size_t(ob)
    d = lambda c: moe.raw_call("moe_dispatch_mx", ctypes.byref(c), 0x1000, 0x2000, 0x3000, 0x4000,  # noqa: E731
                               0x5000, 0x6000, 0x7000, None, 0x8000, sz, None)
    assert d(plain) == INVALID                              # needs an FP8 config
    w = moe.make_weights(0x100, w1=0x200, w3=0x300, w2=0x400)  # bf16 weights only
    f = lambda c, wt: moe.raw_call("moe_expert_ffn_mx", ctypes.byref(c), 0x1000, 0x2000, 0x3000,  # noqa: E731
                                   0x4000, ctypes.byref(wt), 0x5000, 0x6000, 0x7000, 0x8000, sz, None)
    assert f(mx, w) == INVALID                              # FP8 weights missing
    wmx = moe.make_weights(0x100, w1_mx=0x200, w1_sf=0x300, w3_mx=0x400, w3_sf=0x500, w2_mx=0x600,
                           w2_sf=0x708)
    assert f(mx, wmx) == MISAL
    layer = lambda wt: moe.raw_call("moe_layer_fwd", ctypes.byref(mx), ctypes.byref(wt), 0x1000,  # noqa: E731
                                    0x2000, None, 0x3000, ctypes.c_size_t(1 << 40), None)
    assert layer(w) == INVALID


def test_wait_limit_validation():
    # host only: a bound above the 2 s default is refused, 0 restores the default
    st = moe.raw_call("moe_set_wait_limit_ns", ctypes.c_uint64(2_000_000_001))
    assert st == INVALID
    assert moe.raw_call("moe_set_wait_limit_ns", ctypes.c_uint64(0)) == OK


def test_router_split_validation():
    # host only: sizes, unsupported shapes and a short buffer are refused before any launch
    assert moe.moe_router_split_bytes(4096, 128) == 3 * 4096 * 128 * 2
    assert moe.moe_router_split_bytes(4096, 8) == 3 * 4096 * 64 * 2
    assert moe.moe_router_split_bytes(7168, 256) == 3 * 7168 * 256 * 2
    n = ctypes.c_size_t()
    assert moe.raw_call("moe_router_split_bytes", 64, 257, ctypes.byref(n)) == UNSUP
    assert moe.raw_call("moe_router_split_bytes", 0, 8, ctypes.byref(n)) == INVALID
    fake = ctypes.c_void_p(16)
    assert moe.raw_call("moe_router_split", fake, 64, 8, fake, ctypes.c_size_t(10), None) == WS
    assert moe.raw_call("moe_router_split", fake, 96, 8, fake, ctypes.c_size_t(1 << 20), None) == UNSUP
    assert moe.raw_call("moe_router_split", None, 64, 8, fake, ctypes.c_size_t(1 << 20), None) == INVALID
