"""Thin ctypes binding of libmoe.so (include/moe.h).

Argument marshalling only: every step of the MoE layer runs in the library's
CUDA kernels.  PyTorch provides device memory and the current stream.  The
module raises ImportError when the shared library is missing: there is no
fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
import re
from dataclasses import dataclass
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmoe.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "moe.h")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"libmoe.so is not built ({LIB_PATH}); run "
                      "`python -m expert_router_gemm_b200.build`")
_lib = ctypes.CDLL(LIB_PATH)

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_MISALIGNED = 0, 1, 2, 3
MOE_ERR_WORKSPACE, MOE_ERR_CUDA, MOE_ERR_NONFINITE, MOE_ERR_DEVICE = 4, 5, 6, 7
MOE_F32, MOE_BF16 = 0, 1
MOE_GEMM_ACT, MOE_GEMM_MXFP8 = 0, 1
MOE_FLAG_NONFINITE_LOGITS, MOE_FLAG_BAD_EXPERT_INDEX, MOE_FLAG_WAIT_TIMEOUT = 1, 2, 4


class moe_config_t(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int64), ("d", ctypes.c_int32), ("N", ctypes.c_int32),
                ("k", ctypes.c_int32), ("f", ctypes.c_int32), ("f_shared", ctypes.c_int32),
                ("capacity_factor", ctypes.c_double), ("capacity", ctypes.c_int32),
                ("act_dtype", ctypes.c_int), ("seg_align", ctypes.c_int32),
                ("gemm_format", ctypes.c_int32)]


class moe_weights_t(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("w_router", "router_bias", "w1", "w3", "w2", "ws1", "ws3", "ws2",
                 "selection_bias", "w1_mx", "w1_sf", "w3_mx", "w3_sf", "w2_mx", "w2_sf",
                 "w_router_split")]


class moe_stats_t(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("y_frac", "z_mean", "l_aux_p3", "l_aux_switch", "counts", "kept", "num_dropped",
                 "z_loss", "load_std", "top2_ratio", "avg_tokens_per_expert")]


class moe_grads_t(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("dx", "dw_router", "drouter_bias", "dw1", "dw3", "dw2", "dws1", "dws3", "dws2")]


_P = ctypes.c_void_p
_SZ = ctypes.c_size_t
_PROTOS = {
    "moe_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "moe_last_cuda_error": (ctypes.c_char_p, []),
    "moe_version": (ctypes.c_char_p, []),
    "moe_capacity": (ctypes.c_int, [ctypes.POINTER(moe_config_t), ctypes.POINTER(ctypes.c_int32)]),
    "moe_workspace_size": (ctypes.c_int, [ctypes.POINTER(moe_config_t), ctypes.POINTER(_SZ),
                                          ctypes.POINTER(_SZ), ctypes.POINTER(ctypes.c_int64)]),
    "moe_route": (ctypes.c_int, [ctypes.POINTER(moe_config_t), _P, _P, _P, _P, _P, _P, _P,
                                 ctypes.POINTER(moe_stats_t), _P, _SZ, _P]),
    "moe_route_with_split": (ctypes.c_int, [ctypes.POINTER(moe_config_t), _P, _P, _P, _P, _P, _P, _P, _P,
                                            ctypes.POINTER(moe_stats_t), _P, _SZ, _P]),
    "moe_route_from_logits": (ctypes.c_int, [ctypes.POINTER(moe_config_t), _P, _P, _P, _P,
                                             ctypes.POINTER(moe_stats_t), _P, _SZ, _P]),
    "moe_bias_update": (ctypes.c_int, [ctypes.POINTER(moe_config_t), _P, _P, ctypes.c_float, _P]),
    "moe_mx_quantize_weight": (ctypes.c_int, [_P, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, _P, _P,
                                              _P]),
    "moe_dispatch_mx": (ctypes.c_int, [ctypes.POINTER(moe_config_t), _P, _P, _P, _P, _P, _P, _P,
                                       ctypes.POINTER(moe_stats_t), _P, _SZ, _P]),
    "moe_expert_ffn_mx": (ctypes.c_int, [ctypes.POINTER(moe_config_t), _P, _P, _P, _P,
                                         ctypes.POINTER(moe_weights_t), _P, _P, _P, _P, _SZ, _P]),
    "moe_dispatch": (ctypes.c_int, [ctypes.POINTER(moe_config_t), _P, _P, _P, _P, _P, _P,
                                    ctypes.POINTER(moe_stats_t), _P, _SZ, _P]),
    "moe_dispatch_static": (ctypes.c_int, [ctypes.POINTER(moe_config_t), _P, _P, _P, _P, _P, _P,
                                           ctypes.POINTER(moe_stats_t), _P, _P]),
    "moe_expert_ffn": (ctypes.c_int, [ctypes.POINTER(moe_config_t), _P, _P, _P,
                                      ctypes.POINTER(moe_weights_t), _P, _P, _P, _SZ, _P]),
    "moe_shared_expert_ffn": (ctypes.c_int, [ctypes.POINTER(moe_config_t), _P,
                                             ctypes.POINTER(moe_weights_t), _P, _P, _P, _SZ, _P]),
    "moe_combine": (ctypes.c_int, [ctypes.POINTER(moe_config_t), _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "moe_layer_fwd": (ctypes.c_int, [ctypes.POINTER(moe_config_t), ctypes.POINTER(moe_weights_t),
                                     _P, _P, ctypes.POINTER(moe_stats_t), _P, _SZ, _P]),
    "moe_read_flags": (ctypes.c_int, [_P, _SZ, ctypes.POINTER(ctypes.c_uint32), _P]),
    "moe_set_wait_limit_ns": (ctypes.c_int, [ctypes.c_uint64]),
    "moe_router_split_bytes": (ctypes.c_int, [ctypes.c_int32, ctypes.c_int32, ctypes.POINTER(_SZ)]),
    "moe_router_split": (ctypes.c_int, [_P, ctypes.c_int32, ctypes.c_int32, _P, _SZ, _P]),
    "moe_backward_workspace_size": (ctypes.c_int, [ctypes.POINTER(moe_config_t), ctypes.POINTER(_SZ)]),
    "moe_layer_bwd": (ctypes.c_int, [ctypes.POINTER(moe_config_t), ctypes.POINTER(moe_weights_t), _P, _P,
                                     ctypes.c_float, ctypes.c_float, ctypes.POINTER(moe_grads_t), _P, _SZ,
                                     _P]),
}
for _name, (_res, _args) in _PROTOS.items():
    _fn = getattr(_lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args


def header_functions():
    """Names of the functions declared in include/moe.h."""
    with open(HEADER_PATH) as fh:
        text = fh.read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*(moe_[a-z_0-9]+)\s*\(",
                                 text, flags=re.M)))


class MoeError(RuntimeError):
    def __init__(self, status: int, where: str):
        msg = _lib.moe_status_string(status).decode()
        if status == MOE_ERR_CUDA:
            msg += f" ({_lib.moe_last_cuda_error().decode()})"
        super().__init__(f"{where}: {msg}")
        self.status = status


def _check(status: int, where: str):
    if status != MOE_OK:
        raise MoeError(status, where)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        return int(t)
    if t.numel() and not t.is_contiguous():
        raise ValueError("tensors passed to libmoe must be contiguous")
    return t.data_ptr() or None


def _stream(stream) -> Optional[int]:
    if stream is None:
        if not torch.cuda.is_available():
            return None
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def make_config(T: int, d: int, N: int, k: int, f: int, f_shared: int = 0,
                capacity_factor: float = 1.0, capacity: int = -1, dtype: str = "bf16",
                seg_align: int = 0, gemm: str = "act") -> moe_config_t:
    return moe_config_t(T, d, N, k, f, f_shared, capacity_factor, capacity,
                        MOE_BF16 if dtype == "bf16" else MOE_F32, seg_align,
                        MOE_GEMM_MXFP8 if gemm == "mxfp8" else MOE_GEMM_ACT)


def config_from_workload(w, T: Optional[int] = None, **over) -> moe_config_t:
    kw = dict(T=w.T if T is None else T, d=w.d, N=w.N, k=w.k, f=w.f, f_shared=w.f_shared,
              capacity_factor=w.capacity_factor, dtype=w.dtype)
    kw.update(over)
    return make_config(**kw)


def make_weights(w_router, router_bias=None, w1=None, w3=None, w2=None, ws1=None, ws3=None,
                 ws2=None, selection_bias=None, w1_mx=None, w1_sf=None, w3_mx=None, w3_sf=None,
                 w2_mx=None, w2_sf=None, w_router_split=None) -> moe_weights_t:
    return moe_weights_t(*[_ptr(t) for t in (w_router, router_bias, w1, w3, w2, ws1, ws3, ws2,
                                            selection_bias, w1_mx, w1_sf, w3_mx, w3_sf, w2_mx,
                                            w2_sf, w_router_split)])


def make_stats(y_frac=None, z_mean=None, l_aux_p3=None, l_aux_switch=None, counts=None,
               kept=None, num_dropped=None, z_loss=None, load_std=None, top2_ratio=None,
               avg_tokens_per_expert=None) -> moe_stats_t:
    return moe_stats_t(*[_ptr(t) for t in (y_frac, z_mean, l_aux_p3, l_aux_switch, counts, kept,
                                            num_dropped, z_loss, load_std, top2_ratio,
                                            avg_tokens_per_expert)])


# ---------------------------------------------------------------- the C-ABI calls
def moe_version() -> str:
    return _lib.moe_version().decode()


def moe_status_string(status: int) -> str:
    return _lib.moe_status_string(status).decode()


def moe_capacity(cfg: moe_config_t) -> int:
    c = ctypes.c_int32()
    _check(_lib.moe_capacity(ctypes.byref(cfg), ctypes.byref(c)), "moe_capacity")
    return c.value


def moe_workspace_size(cfg: moe_config_t):
    """-> (layer_bytes, op_bytes, max_rows)"""
    lb, ob, mr = _SZ(), _SZ(), ctypes.c_int64()
    _check(_lib.moe_workspace_size(ctypes.byref(cfg), ctypes.byref(lb), ctypes.byref(ob),
                                   ctypes.byref(mr)), "moe_workspace_size")
    return lb.value, ob.value, mr.value


def _stats_ref(stats: Optional[moe_stats_t]):
    return ctypes.byref(stats) if stats is not None else None


def moe_route(cfg, x, w_router, router_bias, selection_bias, logits_out, topk_idx, topk_w, stats,
              ws, stream=None):
    _check(_lib.moe_route(ctypes.byref(cfg), _ptr(x), _ptr(w_router), _ptr(router_bias),
                          _ptr(selection_bias), _ptr(logits_out), _ptr(topk_idx), _ptr(topk_w),
                          _stats_ref(stats), _ptr(ws), ws.numel() if ws is not None else 0,
                          _stream(stream)),
           "moe_route")


def moe_route_with_split(cfg, x, w_router, w_router_split, router_bias, selection_bias, logits_out, topk_idx,
                         topk_w, stats, ws, stream=None):
    _check(_lib.moe_route_with_split(ctypes.byref(cfg), _ptr(x), _ptr(w_router), _ptr(w_router_split),
                                     _ptr(router_bias), _ptr(selection_bias), _ptr(logits_out),
                                     _ptr(topk_idx), _ptr(topk_w), _stats_ref(stats), _ptr(ws),
                                     ws.numel() if ws is not None else 0, _stream(stream)),
           "moe_route_with_split")


def moe_route_from_logits(cfg, logits, selection_bias, topk_idx, topk_w, stats, ws, stream=None):
    _check(_lib.moe_route_from_logits(ctypes.byref(cfg), _ptr(logits), _ptr(selection_bias),
                                      _ptr(topk_idx), _ptr(topk_w), _stats_ref(stats), _ptr(ws),
                                      ws.numel() if ws is not None else 0, _stream(stream)),
           "moe_route_from_logits")


def moe_bias_update(cfg, selection_bias, counts, gamma: float, stream=None):
    _check(_lib.moe_bias_update(ctypes.byref(cfg), _ptr(selection_bias), _ptr(counts),
                                ctypes.c_float(gamma), _stream(stream)), "moe_bias_update")


def moe_dispatch(cfg, x, topk_idx, row_map, seg_off, seg_count, xp, stats, ws, stream=None):
    _check(_lib.moe_dispatch(ctypes.byref(cfg), _ptr(x), _ptr(topk_idx), _ptr(row_map),
                             _ptr(seg_off), _ptr(seg_count), _ptr(xp), _stats_ref(stats),
                             _ptr(ws), ws.numel() if ws is not None else 0, _stream(stream)),
           "moe_dispatch")


def moe_dispatch_static(cfg, x, topk_idx, row_map, seg_off, seg_count, xp, stats,
                        device_flags=None, stream=None):
    _check(_lib.moe_dispatch_static(ctypes.byref(cfg), _ptr(x), _ptr(topk_idx), _ptr(row_map),
                                    _ptr(seg_off), _ptr(seg_count), _ptr(xp), _stats_ref(stats),
                                    _ptr(device_flags), _stream(stream)), "moe_dispatch_static")


MOE_DISPATCH_STATIC_MAX_CELLS = 131072


def moe_mx_quantize_weight(w, G: int, K: int, N: int, codes, sf, stream=None):
    _check(_lib.moe_mx_quantize_weight(_ptr(w), G, K, N, _ptr(codes), _ptr(sf), _stream(stream)),
           "moe_mx_quantize_weight")


def moe_dispatch_mx(cfg, x, topk_idx, row_map, seg_off, seg_count, xp_codes, xp_sf, stats, ws,
                    stream=None):
    _check(_lib.moe_dispatch_mx(ctypes.byref(cfg), _ptr(x), _ptr(topk_idx), _ptr(row_map),
                                _ptr(seg_off), _ptr(seg_count), _ptr(xp_codes), _ptr(xp_sf),
                                _stats_ref(stats), _ptr(ws), ws.numel() if ws is not None else 0,
                                _stream(stream)), "moe_dispatch_mx")


def moe_expert_ffn_mx(cfg, xp_codes, xp_sf, seg_off, seg_count, weights: moe_weights_t, h_codes,
                      h_sf, out_rows, ws, stream=None):
    _check(_lib.moe_expert_ffn_mx(ctypes.byref(cfg), _ptr(xp_codes), _ptr(xp_sf), _ptr(seg_off),
                                  _ptr(seg_count), ctypes.byref(weights), _ptr(h_codes), _ptr(h_sf),
                                  _ptr(out_rows), _ptr(ws), ws.numel() if ws is not None else 0,
                                  _stream(stream)), "moe_expert_ffn_mx")


def mx_sf_bytes(rows: int, K: int) -> int:
    """Bytes of the scales of `rows` rows of K values (tile-interleaved layout)."""
    return (rows + 127) // 128 * 128 * (K // 32)


def moe_expert_ffn(cfg, xp, seg_off, seg_count, weights: moe_weights_t, h, out_rows, ws,
                   stream=None):
    _check(_lib.moe_expert_ffn(ctypes.byref(cfg), _ptr(xp), _ptr(seg_off), _ptr(seg_count),
                               ctypes.byref(weights), _ptr(h), _ptr(out_rows), _ptr(ws),
                               ws.numel() if ws is not None else 0, _stream(stream)),
           "moe_expert_ffn")


def moe_shared_expert_ffn(cfg, x, weights: moe_weights_t, h_shared, shared_out, ws,
                          stream=None):
    _check(_lib.moe_shared_expert_ffn(ctypes.byref(cfg), _ptr(x), ctypes.byref(weights),
                                      _ptr(h_shared), _ptr(shared_out), _ptr(ws),
                                      ws.numel() if ws is not None else 0, _stream(stream)),
           "moe_shared_expert_ffn")


def moe_combine(cfg, out_rows, row_map, topk_w, shared_out, y, ws, stream=None):
    _check(_lib.moe_combine(ctypes.byref(cfg), _ptr(out_rows), _ptr(row_map), _ptr(topk_w),
                            _ptr(shared_out), _ptr(y), _ptr(ws),
                            ws.numel() if ws is not None else 0, _stream(stream)),
           "moe_combine")


def moe_layer_fwd(cfg, weights: moe_weights_t, x, y, stats, ws, stream=None):
    _check(_lib.moe_layer_fwd(ctypes.byref(cfg), ctypes.byref(weights), _ptr(x), _ptr(y),
                              _stats_ref(stats), _ptr(ws), ws.numel() if ws is not None else 0,
                              _stream(stream)), "moe_layer_fwd")


def make_grads(dx=None, dw_router=None, drouter_bias=None, dw1=None, dw3=None, dw2=None, dws1=None,
               dws3=None, dws2=None) -> moe_grads_t:
    return moe_grads_t(*[_ptr(t) for t in (dx, dw_router, drouter_bias, dw1, dw3, dw2, dws1, dws3,
                                           dws2)])


def moe_backward_workspace_size(cfg) -> int:
    b = _SZ()
    _check(_lib.moe_backward_workspace_size(ctypes.byref(cfg), ctypes.byref(b)),
           "moe_backward_workspace_size")
    return b.value


def moe_layer_bwd(cfg, weights: moe_weights_t, x, dy, aux_weight: float, z_weight: float,
                  grads: moe_grads_t, ws, stream=None):
    _check(_lib.moe_layer_bwd(ctypes.byref(cfg), ctypes.byref(weights), _ptr(x), _ptr(dy),
                              ctypes.c_float(aux_weight), ctypes.c_float(z_weight),
                              ctypes.byref(grads), _ptr(ws), ws.numel() if ws is not None else 0,
                              _stream(stream)), "moe_layer_bwd")


def moe_read_flags(ws, stream=None) -> int:
    """Waits for the stream; returns the flags word (raises on a set bit)."""
    v = ctypes.c_uint32()
    st = _lib.moe_read_flags(_ptr(ws), ws.numel(), ctypes.byref(v), _stream(stream))
    if st not in (MOE_OK, MOE_ERR_NONFINITE, MOE_ERR_DEVICE):
        _check(st, "moe_read_flags")
    return v.value


def moe_router_split_bytes(d: int, N: int) -> int:
    b = _SZ()
    _check(_lib.moe_router_split_bytes(d, N, ctypes.byref(b)), "moe_router_split_bytes")
    return b.value


def moe_router_split(w_router, d: int, N: int, split, stream=None) -> None:
    _check(_lib.moe_router_split(_ptr(w_router), d, N, _ptr(split), split.numel() * split.element_size(),
                                 _stream(stream)), "moe_router_split")


def moe_set_wait_limit_ns(ns: int) -> None:
    """Bound of the pipeline waits of later launches of the tensor-core kernels
    (bf16 and FP8 grouped GEMMs, router GEMM); 0: the 2 s default."""
    _check(_lib.moe_set_wait_limit_ns(int(ns)), "moe_set_wait_limit_ns")


def raw_call(name: str, *args) -> int:
    """Call a C-ABI function with raw ctypes arguments; returns its status (tests)."""
    return getattr(_lib, name)(*args)


# ---------------------------------------------------------------- conveniences
@dataclass
class DeviceLayer:
    """Device copies of one layer's inputs (torch tensors on cuda)."""
    cfg: moe_config_t
    x: torch.Tensor
    w_router: torch.Tensor
    bias: Optional[torch.Tensor]
    w1: torch.Tensor
    w3: torch.Tensor
    w2: torch.Tensor
    ws1: Optional[torch.Tensor] = None
    ws3: Optional[torch.Tensor] = None
    ws2: Optional[torch.Tensor] = None
    selection_bias: Optional[torch.Tensor] = None
    mx: Optional[dict] = None      # block-scaled FP8 weights (quantize_mx)
    router_split: Optional[torch.Tensor] = None   # bf16 split of w_router (split_router)

    def weights(self) -> moe_weights_t:
        m = self.mx or {}
        return make_weights(self.w_router, self.bias, self.w1, self.w3, self.w2,
                            self.ws1, self.ws3, self.ws2, self.selection_bias,
                            m.get("w1_mx"), m.get("w1_sf"), m.get("w3_mx"), m.get("w3_sf"),
                            m.get("w2_mx"), m.get("w2_sf"), self.router_split)

    def split_router(self, stream=None) -> torch.Tensor:
        """Make the bf16 split of the router weight once (moe_router_split) and
        pass it to later layer calls through weights()."""
        d, N = self.cfg.d, self.cfg.N
        buf = torch.empty(moe_router_split_bytes(d, N), dtype=torch.uint8, device=self.w_router.device)
        moe_router_split(self.w_router, d, N, buf, stream)
        self.router_split = buf
        return buf

    def quantize_mx(self, stream=None) -> dict:
        """Quantize the routed experts' bf16 weights to block-scaled FP8 on the
        device (moe_mx_quantize_weight) and keep them for weights()."""
        N, d, f = self.cfg.N, self.cfg.d, self.cfg.f
        dev = self.w1.device
        out = {}
        for name, w, K, Nn in (("w1", self.w1, d, f), ("w3", self.w3, d, f), ("w2", self.w2, f, d)):
            codes = torch.empty((N, Nn, K), dtype=torch.uint8, device=dev)
            sf = torch.empty(N * Nn * K // 32, dtype=torch.uint8, device=dev)
            moe_mx_quantize_weight(w, N, K, Nn, codes, sf, stream)
            out[name + "_mx"], out[name + "_sf"] = codes, sf
        self.mx = out
        return out


def to_device(inputs, cfg: moe_config_t, device="cuda") -> DeviceLayer:
    """Upload host arrays (numpy; bf16 as uint16 bits) to device tensors."""
    import numpy as np

    def up(a):
        if a is None:
            return None
        a = np.ascontiguousarray(a)
        t = torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a)
        return t.to(device)

    return DeviceLayer(cfg, up(inputs.x), up(inputs.w_router), up(inputs.bias), up(inputs.w1),
                       up(inputs.w3), up(inputs.w2), up(inputs.ws1), up(inputs.ws3),
                       up(inputs.ws2))


def act_dtype(cfg: moe_config_t):
    return torch.int16 if cfg.act_dtype == MOE_BF16 else torch.float32
