"""Pins of the FP8 (block-scaled E4M3) oracle against the format's definition,
library conversions, brute force and closed forms; mutation tests at the end
plant plausible mistakes in the oracle and expect a pin to fail."""
import math

import numpy as np
import pytest
import torch

from oracle import moe_oracle as orc
from oracle import mxfp8 as mx

RNG = np.random.default_rng(4321)


# --------------------------------------------------------------------------
# E4M3 rounding and encoding
# --------------------------------------------------------------------------

def check_e4m3_hand(m=mx):
    r = m.e4m3_round
    assert r(np.array([448.0]))[0] == 448.0                   # largest finite
    assert r(np.array([460.0]))[0] == 448.0                   # saturation
    assert r(np.array([2.0 ** -9]))[0] == 2.0 ** -9           # smallest subnormal
    assert r(np.array([2.0 ** -10]))[0] == 0.0                # tie -> even (0)
    assert r(np.array([3 * 2.0 ** -10]))[0] == 2.0 ** -8      # tie 1 vs 2 quanta -> 2
    assert r(np.array([1.0 + 2.0 ** -4]))[0] == 1.0           # tie -> even mantissa
    assert r(np.array([1.0 + 3 * 2.0 ** -4]))[0] == 1.25      # tie -> even mantissa (up)
    assert r(np.array([-1.0 - 2.0 ** -4 - 1e-9]))[0] == -1.125
    assert r(np.array([15.5]))[0] == 16.0                     # 15 < 15.5 < 16: tie -> 16 (even)
    np.testing.assert_array_equal(m.e4m3_encode(np.array([448.0, -448.0, 1.0, 2.0 ** -9, 0.0, -2.0])),
                                  np.array([0x7E, 0xFE, 0x38, 0x01, 0x00, 0xC0], np.uint8))


def check_e4m3_library(m=mx):
    # torch's float8_e4m3fn cast rounds to nearest even; compare inside the finite range
    v = np.concatenate([RNG.uniform(-448, 448, 20000), RNG.normal(size=20000) * 0.05,
                        RNG.normal(size=2000) * 2.0 ** -8,
                        np.ldexp(1.0, np.arange(-9, 9)) * 1.0625])
    t = torch.from_numpy(v.astype(np.float32)).to(torch.float8_e4m3fn)
    want = t.to(torch.float64).numpy()
    got = m.e4m3_round(v.astype(np.float32).astype(np.float64))
    np.testing.assert_array_equal(got, want)
    np.testing.assert_array_equal(m.e4m3_encode(got), t.view(torch.uint8).numpy())


def test_e4m3_hand():
    check_e4m3_hand()


def test_e4m3_library():
    check_e4m3_library()


# --------------------------------------------------------------------------
# shared exponent
# --------------------------------------------------------------------------

def _brute_exponent(a):
    for e in range(-127, 128):
        if a <= math.ldexp(448.0, e):
            return e
    return 127


def check_scale_exponent(m=mx):
    vals = [0.0, 448.0, 449.0, 1.75, 1.7500001, 1.0, 2.0 ** -130, 3.0e38, 0.875, 0.87500006,
            1.5 * 2.0 ** -120, 7.0 * 2.0 ** 100]
    vals += list(np.abs(RNG.normal(size=300)) * np.ldexp(1.0, RNG.integers(-60, 60, 300)))
    got = m.mx_scale_exponent(np.array(vals))
    want = [_brute_exponent(a) for a in vals]
    np.testing.assert_array_equal(got, want)


def test_scale_exponent():
    check_scale_exponent()


# --------------------------------------------------------------------------
# block quantization
# --------------------------------------------------------------------------

def check_mx_roundtrip_exact(m=mx):
    # blocks whose values are E4M3 values times 2^e, one of them +-448 2^e:
    # the shared exponent is e and the quantization is exact
    R, K = 6, 128
    grid = m.e4m3_round(RNG.uniform(-448, 448, (R, K)))
    grid[:, ::32] = 448.0 * np.where(RNG.random((R, K // 32)) < 0.5, -1, 1)
    e = RNG.integers(-20, 20, (R, K // 32))
    v = grid * np.ldexp(1.0, np.repeat(e, 32, axis=1))
    q = m.mx_quantize(v)
    np.testing.assert_array_equal(q.e, e)
    np.testing.assert_array_equal(q.dequantize(), v)


def check_mx_error_bound_and_axis(m=mx):
    # rows of very different magnitude, and columns of very different magnitude:
    # quantizing along K keeps each element within half a step (2^-4 relative)
    # of its value in the normal range; along the wrong axis it would not
    R, K = 16, 256
    v = RNG.normal(size=(R, K)) * np.ldexp(1.0, RNG.integers(-30, 30, R))[:, None]
    q = m.mx_quantize(v)
    deq = q.dequantize()
    scale = np.ldexp(1.0, np.repeat(q.e, 32, axis=1))
    normal = np.abs(v) >= 2.0 ** -6 * scale
    assert np.all(np.abs(deq - v)[normal] <= 2.0 ** -4 * np.abs(v)[normal])
    assert np.all(np.abs(deq - v)[~normal] <= 2.0 ** -10 * scale[~normal])
    w = RNG.normal(size=(K, 64)) * np.ldexp(1.0, 3 * (np.arange(64) % 8))[None, :]
    wq = m.quantize_weight(w)                      # [64, K], blocks along K per column
    assert wq.q.shape == (64, K)
    rel = np.abs(wq.dequantize().T - w) / np.abs(w)
    assert np.median(rel) < 0.03 and np.max(rel[np.abs(w) > 1e-3 * np.abs(w).max(axis=0)]) <= 2.0 ** -4


def test_mx_roundtrip_exact():
    check_mx_roundtrip_exact()


def test_mx_error_bound_and_axis():
    check_mx_error_bound_and_axis()


# --------------------------------------------------------------------------
# the FP8 layer
# --------------------------------------------------------------------------

def _representable(shape, e_lo=-4, e_hi=0):
    g = mx.e4m3_round(RNG.uniform(-448, 448, shape))
    g[..., ::32] = 448.0
    return g * 2.0 ** RNG.integers(e_lo, e_hi)


def check_layer_h_quantized(m=mx):
    # one expert, k = 1, W2 = identity (f = d): every kept row's output is exactly
    # the block-quantized h = silu(x W1) * (x W3), with x, W1, W3 representable
    T, d = 40, 64
    x = _representable((T, d))
    w1 = _representable((1, d, d), -10, -8)
    w3 = _representable((1, d, d), -10, -8)
    w2 = np.eye(d)[None]
    wr = np.ones((d, 1))
    res = m.layer_forward_mxfp8(x, wr, None, w1, w3, w2, k=1, cap=T)
    h = orc.silu(x @ w1[0]) * (x @ w3[0])
    want = m.mx_quantize(h).dequantize()
    np.testing.assert_allclose(res.y, want, rtol=1e-12, atol=0)
    assert np.any(want != h)                        # the quantization of h is visible


def check_layer_near_bf16(m=mx):
    # the FP8 layer stays within the quantization error of the exact layer
    from expert_router_gemm_b200 import synth
    from expert_router_gemm_b200.configs import Workload
    w = Workload("mx-pin", T=96, d=128, N=4, k=2, f=128, capacity_factor=1.25)
    inp = synth.make_inputs(w)
    ref = orc.layer_forward(inp.x, inp.w_router, inp.bias, inp.w1, inp.w3, inp.w2, k=w.k,
                            capacity_factor=w.capacity_factor, bf16=False)
    res = m.layer_forward_mxfp8(inp.x, inp.w_router, inp.bias, inp.w1, inp.w3, inp.w2, k=w.k,
                                capacity_factor=w.capacity_factor)
    rel = orc.rel_frobenius(res.y, ref.y)
    assert 0.005 < rel < 0.08, rel
    np.testing.assert_array_equal(res.base.idx, ref.idx)


def test_layer_h_quantized():
    check_layer_h_quantized()


def test_layer_near_bf16():
    check_layer_near_bf16()


def check_sf_layout(m=mx):
    # the layout is a bijection of (row, block) onto the bytes of the buffer
    rows, nkb = 256, 12
    r, j = np.meshgrid(np.arange(rows), np.arange(nkb), indexing="ij")
    off = m.sf_atom_offset(r, j, nkb)
    assert sorted(off.reshape(-1).tolist()) == list(range(rows * nkb))
    assert m.sf_atom_offset(np.array([0, 1, 32, 127, 128]), np.array([0, 0, 0, 3, 4]), nkb).tolist() == \
        [0, 16, 4, 16 * 31 + 12 + 3, 3 * 512 + 512]


def test_sf_layout():
    check_sf_layout()


# --------------------------------------------------------------------------
# mutation tests
# --------------------------------------------------------------------------

ALL_CHECKS = [check_e4m3_hand, check_e4m3_library, check_scale_exponent, check_mx_roundtrip_exact,
              check_mx_error_bound_and_axis, check_layer_h_quantized, check_layer_near_bf16,
              check_sf_layout]

_ORIG = {n: getattr(mx, n) for n in ("e4m3_round", "mx_scale_exponent", "mx_quantize", "quantize_weight",
                                     "swiglu_mx")}


def _mut_round_truncate(v):
    v = np.asarray(v, np.float64)
    a = np.abs(v)
    _, ex = np.frexp(a)
    quantum = np.ldexp(1.0, np.maximum(ex - 1, -6) - 3)
    return np.copysign(np.minimum(np.floor(a / quantum) * quantum, 448.0), v)


def _mut_round_half_up(v):
    v = np.asarray(v, np.float64)
    a = np.abs(v)
    _, ex = np.frexp(a)
    quantum = np.ldexp(1.0, np.maximum(ex - 1, -6) - 3)
    return np.copysign(np.minimum(np.floor(a / quantum + 0.5) * quantum, 448.0), v)


def _mut_round_no_subnormals(v):
    v = np.asarray(v, np.float64)
    a = np.abs(v)
    _, ex = np.frexp(a)
    quantum = np.ldexp(1.0, ex - 4)
    q = np.rint(a / quantum) * quantum
    return np.copysign(np.where(a < 2.0 ** -6, 0.0, np.minimum(q, 448.0)), v)


def _mut_exponent_floor(amax):
    # the spec's floor(log2 amax) - 8: may saturate the largest element
    amax = np.asarray(amax, np.float64)
    _, ex = np.frexp(amax)
    return np.clip(np.where(amax == 0, -127, ex - 1 - 8), -127, 127).astype(np.int64)


def _mut_quantize_wrong_axis(v):
    # blocks of 32 rows instead of 32 columns (transposed blocking)
    v = np.asarray(v, np.float64)
    R, K = v.shape
    if R % 32:
        return _ORIG["mx_quantize"](v)
    t = _ORIG["mx_quantize"](v.T)
    deq = t.dequantize().T
    e = mx.mx_scale_exponent(np.abs(v.reshape(R, K // 32, 32)).max(axis=2))
    return mx.MxTensor(deq / np.ldexp(1.0, np.repeat(e, 32, axis=1)), e)


def _mut_weight_along_n(w):
    return _ORIG["mx_quantize"](orc.as_f64(w)).__class__(*_transpose_mx(_ORIG["mx_quantize"](orc.as_f64(w))))


def _transpose_mx(t):
    # blocks formed along N, then presented as [N, K]
    deq = t.dequantize().T
    K = deq.shape[1]
    e = mx.mx_scale_exponent(np.abs(deq.reshape(deq.shape[0], K // 32, 32)).max(axis=2))
    return deq / np.ldexp(1.0, np.repeat(e, 32, axis=1)), e


def _mut_swiglu_no_h_quant(xq, w1q, w3q, w2q):
    xa = xq.dequantize()
    h = orc.silu(xa @ w1q.dequantize().T) * (xa @ w3q.dequantize().T)
    return h @ w2q.dequantize().T


def _mut_swiglu_swap(xq, w1q, w3q, w2q):
    return _ORIG["swiglu_mx"](xq, w3q, w1q, w2q)


MUTANTS = [
    ("e4m3_round", _mut_round_truncate),
    ("e4m3_round", _mut_round_half_up),
    ("e4m3_round", _mut_round_no_subnormals),
    ("mx_scale_exponent", _mut_exponent_floor),
    ("mx_quantize", _mut_quantize_wrong_axis),
    ("quantize_weight", _mut_weight_along_n),
    ("swiglu_mx", _mut_swiglu_no_h_quant),
    ("swiglu_mx", _mut_swiglu_swap),
]


@pytest.mark.parametrize("name,mutant", MUTANTS, ids=[f"{n}:{m.__name__}" for n, m in MUTANTS])
def test_mutant_is_caught(monkeypatch, name, mutant):
    monkeypatch.setattr(mx, name, mutant)
    caught = []
    for chk in ALL_CHECKS:
        try:
            chk(mx)
        except (AssertionError, ValueError, FloatingPointError, IndexError):
            caught.append(chk.__name__)
    assert caught, f"no pin caught the planted mistake in {name}"
