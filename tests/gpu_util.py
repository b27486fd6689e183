"""Helpers of the GPU parity tests: run each C-ABI step on device tensors and
bring the results back as numpy arrays.  (Not a test module.)"""
from __future__ import annotations

import numpy as np
import torch

from expert_router_gemm_b200 import moe

I32, F32, U8 = torch.int32, torch.float32, torch.uint8
NAN = float("nan")


def cuda_tensor(a: np.ndarray) -> torch.Tensor:
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        a = a.view(np.int16)
    return torch.from_numpy(a).cuda()


def host(t: torch.Tensor) -> np.ndarray:
    a = t.cpu().numpy()
    return a.view(np.uint16) if a.dtype == np.int16 else a


def new_stats(N):
    bufs = dict(y_frac=torch.full((N,), NAN, dtype=F32, device="cuda"),
                z_mean=torch.full((N,), NAN, dtype=F32, device="cuda"),
                l_aux_p3=torch.full((1,), NAN, dtype=F32, device="cuda"),
                l_aux_switch=torch.full((1,), NAN, dtype=F32, device="cuda"),
                counts=torch.full((N,), -9, dtype=I32, device="cuda"),
                kept=torch.full((N,), -9, dtype=I32, device="cuda"),
                num_dropped=torch.full((1,), -9, dtype=I32, device="cuda"),
                z_loss=torch.full((1,), NAN, dtype=F32, device="cuda"),
                load_std=torch.full((1,), NAN, dtype=F32, device="cuda"),
                top2_ratio=torch.full((1,), NAN, dtype=F32, device="cuda"),
                avg_tokens_per_expert=torch.full((1,), NAN, dtype=F32, device="cuda"))
    return bufs, moe.make_stats(**bufs)


def stats_host(bufs):
    return {k: host(v) for k, v in bufs.items()}


def op_workspace(cfg):
    _, ob, _ = moe.moe_workspace_size(cfg)
    return torch.zeros(ob, dtype=U8, device="cuda")


def route_from_logits(cfg, logits: np.ndarray, selection_bias=None):
    T, N, k = cfg.T, cfg.N, cfg.k
    lg = cuda_tensor(logits.astype(np.float32))
    idx = torch.full((T, k), -7, dtype=I32, device="cuda")
    w = torch.full((T, k), NAN, dtype=F32, device="cuda")
    ws = op_workspace(cfg)
    bufs, st = new_stats(N)
    sb = None if selection_bias is None else cuda_tensor(np.asarray(selection_bias, np.float32))
    moe.moe_route_from_logits(cfg, lg, sb, idx, w, st, ws)
    flags = moe.moe_read_flags(ws)
    return host(idx), host(w), stats_host(bufs), flags


def dispatch(cfg, x: torch.Tensor, idx: torch.Tensor):
    T, N, k = cfg.T, cfg.N, cfg.k
    _, ob, max_rows = moe.moe_workspace_size(cfg)
    row_map = torch.full((T, k), -7, dtype=I32, device="cuda")
    seg_off = torch.full((N + 1,), -7, dtype=I32, device="cuda")
    seg_count = torch.full((N,), -7, dtype=I32, device="cuda")
    xp = torch.zeros((max_rows, cfg.d), dtype=moe.act_dtype(cfg), device="cuda")
    ws = op_workspace(cfg)
    bufs, st = new_stats(N)
    moe.moe_dispatch(cfg, x, idx, row_map, seg_off, seg_count, xp, st, ws)
    flags = moe.moe_read_flags(ws)
    return dict(row_map=host(row_map), seg_off=host(seg_off), seg_count=host(seg_count),
                xp=host(xp), stats=stats_host(bufs), flags=flags,
                dev=dict(row_map=row_map, seg_off=seg_off, seg_count=seg_count, xp=xp))


def staged_layer(dl: moe.DeviceLayer):
    """Run route -> dispatch -> experts -> (shared) -> combine step by step."""
    cfg = dl.cfg
    T, N, k, d, f = cfg.T, cfg.N, cfg.k, cfg.d, cfg.f
    act = moe.act_dtype(cfg)
    _, ob, max_rows = moe.moe_workspace_size(cfg)
    ws = op_workspace(cfg)
    logits = torch.full((T, N), NAN, dtype=F32, device="cuda")
    idx = torch.full((T, k), -7, dtype=I32, device="cuda")
    w = torch.full((T, k), NAN, dtype=F32, device="cuda")
    bufs, st = new_stats(N)
    moe.moe_route(cfg, dl.x, dl.w_router, dl.bias, dl.selection_bias, logits, idx, w, st, ws)
    row_map = torch.full((T, k), -7, dtype=I32, device="cuda")
    seg_off = torch.full((N + 1,), -7, dtype=I32, device="cuda")
    seg_count = torch.full((N,), -7, dtype=I32, device="cuda")
    xp = torch.zeros((max_rows, d), dtype=act, device="cuda")
    moe.moe_dispatch(cfg, dl.x, idx, row_map, seg_off, seg_count, xp, st, ws)
    h = torch.zeros((max_rows, f), dtype=act, device="cuda")
    out_rows = torch.zeros((max_rows, d), dtype=act, device="cuda")
    wts = dl.weights()
    moe.moe_expert_ffn(cfg, xp, seg_off, seg_count, wts, h, out_rows, ws)
    shared = None
    if cfg.f_shared:
        hs = torch.zeros((T, cfg.f_shared), dtype=act, device="cuda")
        shared = torch.zeros((T, d), dtype=act, device="cuda")
        moe.moe_shared_expert_ffn(cfg, dl.x, wts, hs, shared, ws)
    y = torch.zeros((T, d), dtype=act, device="cuda")
    moe.moe_combine(cfg, out_rows, row_map, w, shared, y, ws)
    flags = moe.moe_read_flags(ws)
    return dict(logits=host(logits), idx=host(idx), w=host(w), row_map=host(row_map),
                seg_off=host(seg_off), seg_count=host(seg_count), y=host(y),
                stats=stats_host(bufs), flags=flags)


def layer_fwd(dl: moe.DeviceLayer, stats=True):
    cfg = dl.cfg
    lb, _, _ = moe.moe_workspace_size(cfg)
    ws = torch.empty(lb, dtype=U8, device="cuda")
    y = torch.zeros((cfg.T, cfg.d), dtype=moe.act_dtype(cfg), device="cuda")
    bufs, st = new_stats(cfg.N) if stats else (None, None)
    moe.moe_layer_fwd(cfg, dl.weights(), dl.x, y, st, ws)
    flags = moe.moe_read_flags(ws)
    return host(y), (stats_host(bufs) if stats else None), flags


def y_as_f64(y: np.ndarray) -> np.ndarray:
    if y.dtype == np.uint16:
        return (y.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    return y.astype(np.float64)
