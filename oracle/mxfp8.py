"""fp64 CPU oracle of the FP8 variant of the MoE layer (block-scaled e4m3).

TEST INFRASTRUCTURE, like moe_oracle: only the tests, the smoke check and the
benchmark's CPU legs may use it; it shares no code with the CUDA path.

The pages run the expert GEMMs in FP8 ("MoE 训练加速实战：DeepEP + Grouped GeMM +
Aux-Loss-Free" §9.1, precision row: FP8 forward with bf16 activations; §3.3 and
§6.2: FP8 payloads and FP8-stored experts upcast at use; "ms-swift + Megatron：
MoE模型加速10倍实测" §5.2: FP8 kernels) without fixing a format.  Reading taken
here: the block-scaled FP8 of the OCP Microscaling (MX) specification v1.0 --
E4M3 elements (bias 7, 3 mantissa bits, largest finite 448, no infinities) that
share one power-of-two scale per 32 consecutive elements along the reduction
dimension.  The shared exponent is the smallest e in [-127, 127] with
max|v| <= 448 * 2^e (so no element saturates; the spec's own choice,
floor(log2 max|v|) - 8, can push the largest element past 448), and each element
is v / 2^e rounded to the nearest E4M3 value, ties to even.

The FP8 layer: routing, capacity and combine as in moe_oracle; the permuted rows
and the three expert weights are quantized along K (x rows along d, W1/W3
columns along d, W2 columns along f); GEMM1 and the SwiGLU run in fp64 on the
dequantized operands; h is quantized along f; GEMM2 runs in fp64 on the
dequantized h and W2.  The layer input and output stay bf16 (the shared expert,
when present, is the bf16 one of moe_oracle).
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Optional, Sequence

import numpy as np

from oracle import moe_oracle as orc

E4M3_MAX = 448.0
BLOCK = 32
EXP_MIN, EXP_MAX = -127, 127


def e4m3_round(v: np.ndarray) -> np.ndarray:
    """Round to the nearest E4M3 value, ties to even; finite magnitudes above
    448 become 448 (saturation).  Normal numbers are (1 + m/8) 2^E with
    E in [-6, 8]; below 2^-6 the grid is uniform with step 2^-9 (subnormals)."""
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    _, ex = np.frexp(a)                      # a = f 2^ex, f in [0.5, 1)
    E = np.maximum(ex - 1, -6)               # binade (subnormals share E = -6)
    quantum = np.ldexp(1.0, E - 3)           # 3 mantissa bits
    q = np.rint(a / quantum) * quantum       # rint: round half to even
    q = np.minimum(q, E4M3_MAX)
    return np.copysign(q, v)


def e4m3_encode(q: np.ndarray) -> np.ndarray:
    """Bit patterns (uint8) of values already on the E4M3 grid."""
    q = np.asarray(q, dtype=np.float64)
    sign = (np.signbit(q)).astype(np.uint8) << 7
    a = np.abs(q)
    _, ex = np.frexp(a)
    E = ex - 1
    normal = a >= 2.0 ** -6
    exp_field = np.where(normal, E + 7, 0)
    mant = np.where(normal, a / np.ldexp(1.0, E) - 1.0, a / 2.0 ** -6) * 8.0
    mant = np.where(a == 0, 0.0, mant)
    exp_field = np.where(a == 0, 0, exp_field)
    assert np.all(mant == np.rint(mant)), "value not on the E4M3 grid"
    return (sign | (exp_field.astype(np.uint8) << 3) | mant.astype(np.uint8)).astype(np.uint8)


def mx_scale_exponent(amax: np.ndarray) -> np.ndarray:
    """Smallest integer e in [-127, 127] with amax <= 448 * 2^e (-127 for 0).

    With amax = M 2^E, M in [1, 2): 448 2^e = 1.75 2^(e+8), so e = E - 8 when
    M <= 1.75 and E - 7 otherwise."""
    amax = np.asarray(amax, dtype=np.float64)
    f, ex = np.frexp(amax)
    M, E = 2.0 * f, ex - 1
    e = np.where(M > 1.75, E - 7, E - 8)
    e = np.where(amax == 0, EXP_MIN, e)
    return np.clip(e, EXP_MIN, EXP_MAX).astype(np.int64)


@dataclass
class MxTensor:
    q: np.ndarray      # [R, K] E4M3 values (float64, on the grid)
    e: np.ndarray      # [R, K / 32] shared exponents (int64)

    def dequantize(self) -> np.ndarray:
        return self.q * np.ldexp(1.0, np.repeat(self.e, BLOCK, axis=1))

    def codes(self) -> np.ndarray:
        return e4m3_encode(self.q)

    def scale_bytes(self) -> np.ndarray:
        """E8M0 encodings: e + 127."""
        return (self.e + 127).astype(np.uint8)


def mx_quantize(v: np.ndarray) -> MxTensor:
    """Block-quantize the rows of v [R, K] (K a multiple of 32) along K."""
    v = np.asarray(v, dtype=np.float64)
    R, K = v.shape
    assert K % BLOCK == 0
    blocks = v.reshape(R, K // BLOCK, BLOCK)
    e = mx_scale_exponent(np.abs(blocks).max(axis=2)) if R else np.zeros((0, K // BLOCK), np.int64)
    scaled = blocks / np.ldexp(1.0, e)[:, :, None]
    q = e4m3_round(scaled).reshape(R, K)
    return MxTensor(q, e)


def quantize_weight(w: np.ndarray) -> MxTensor:
    """One expert's weight [K, N] (bf16 bits or floats) quantized along K for each
    output column n: returns the [N, K] (K-major) block-scaled tensor."""
    return mx_quantize(orc.as_f64(w).T)


def swiglu_mx(xq: MxTensor, w1q: MxTensor, w3q: MxTensor, w2q: MxTensor) -> np.ndarray:
    """GEMM1 + SwiGLU on dequantized operands, h quantized along f, GEMM2."""
    xa = xq.dequantize()
    g = xa @ w1q.dequantize().T
    u = xa @ w3q.dequantize().T
    h = orc.silu(g) * u
    hq = mx_quantize(h)
    return hq.dequantize() @ w2q.dequantize().T


@dataclass
class MxLayerResult:
    base: orc.LayerResult         # routing, dispatch and statistics (identical to the bf16 layer)
    tokens: np.ndarray
    y: np.ndarray                 # [len(tokens), d] fp64


def layer_forward_mxfp8(x, w_router, bias, w1, w3, w2, k: int, capacity_factor: float = 1.0,
                        cap: Optional[int] = None, ws1=None, ws3=None, ws2=None, align: int = 128,
                        tokens: Optional[Sequence[int]] = None, logits: Optional[np.ndarray] = None,
                        selection_bias: Optional[np.ndarray] = None) -> MxLayerResult:
    """Forward pass of the FP8 layer; routing is that of moe_oracle.layer_forward
    (the router stays fp32).  Expert e's rows are quantized as the GPU's permuted
    rows are: each kept row x[t] along d."""
    base = orc.layer_forward(x, w_router, bias, w1, w3, w2, k=k, capacity_factor=capacity_factor,
                             cap=cap, bf16=True, align=align, tokens=[], logits=logits,
                             selection_bias=selection_bias)
    T, d = x.shape
    N = w1.shape[0]
    tok = np.arange(T) if tokens is None else np.asarray(tokens, dtype=np.int64)
    y = np.zeros((len(tok), d))
    if len(tok):
        x64 = orc.as_f64(x[tok])
        sub_idx = base.idx[tok]
        sub_kept = base.disp.row_map[tok] >= 0
        o = np.zeros((len(tok), k, d))
        for e in range(N):
            ti, tj = np.nonzero((sub_idx == e) & sub_kept)
            if len(ti):
                o[ti, tj] = swiglu_mx(mx_quantize(x64[ti]), quantize_weight(w1[e]),
                                      quantize_weight(w3[e]), quantize_weight(w2[e]))
        for j in range(k):
            y += np.where(sub_kept[:, j:j + 1], base.w[tok, j:j + 1] * o[:, j], 0.0)
        if ws1 is not None:
            y += orc.swiglu_ffn(x64, ws1, ws3, ws2, True)
    return MxLayerResult(base, tok, y)


def sf_atom_offset(row: np.ndarray, kblock: np.ndarray, n_kblocks: int) -> np.ndarray:
    """Byte offset of the scale of (row, 32-element block) in the tile-interleaved
    scale layout the tensor cores read: 512-byte atoms for 128 rows x 4 blocks,
    atoms ordered (row tile, K tile); inside an atom row m and block j sit at
    16 (m % 32) + 4 (m // 32) + j.  (A storage layout, not arithmetic.)"""
    row = np.asarray(row, dtype=np.int64)
    kblock = np.asarray(kblock, dtype=np.int64)
    ktiles = n_kblocks // 4
    atom = (row // 128) * ktiles + kblock // 4
    m = row % 128
    return atom * 512 + 16 * (m % 32) + 4 * (m // 32) + kblock % 4


def sf_unpack(buf: np.ndarray, rows: int, n_kblocks: int) -> np.ndarray:
    """[rows, n_kblocks] scale bytes read out of a tile-interleaved buffer."""
    r, j = np.meshgrid(np.arange(rows), np.arange(n_kblocks), indexing="ij")
    return np.asarray(buf, dtype=np.uint8).reshape(-1)[sf_atom_offset(r, j, n_kblocks)]
