"""Benchmark of the MoE-layer forward pass on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config qwen3] [--impl ours|reference]

A step is one forward pass of the whole layer (router GEMM + softmax + top-k +
statistics, capacity clip + permutation, grouped SwiGLU GEMMs, combine) over one
synthetic batch of the named workload, through the C ABI of libmoe.so.  The
statistics include L_aux, the router z-loss and the load figures (last step's
values in router_stats).  With --aux-free GAMMA the top-k choice also adds a
per-expert selection bias, and each step ends with its on-device update
(moe_bias_update) on the step's selection counts.

  value     tokens/s of moe_layer_fwd with inputs resident in HBM (K steps,
            CUDA events, max over ranks; every rank runs an independent replica,
            so the work per GPU is fixed: weak scaling)
  e2e       the same call with the batch copied in from pinned host memory and
            the output copied back inside the timed region
  kernels   per-stage times from CUDA events recorded between the C-ABI steps
            (moe_route, moe_dispatch, moe_expert_ffn, moe_combine) of a second
            timed region, with each stage's algorithmic work and roofline
  roofline  the dominant kernel (the grouped GEMM pair of moe_expert_ffn)
  cpu_baseline  the fp64 oracle on the host cores, on a bounded sample

--impl reference times the fp64 oracle (the reference of this method) on the
host cores instead, on the same workload and metric.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from expert_router_gemm_b200 import configs, synth  # noqa: E402

METRIC = "MoE-layer fwd tokens/s on 1 B200; grouped-GEMM % bf16 TC peak; permute GB/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# fp32 FFMA peak of a B200: 148 SMs x 128 FP32 lanes x 2 flop x 1.965 GHz (max SM clock)
FP32_ALU_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


# A timed region at least this long has run into the power limiter's steady
# state; shorter regions run at the burst clock unless their clock record says
# otherwise (below).
SUSTAINED_REGION_S = 2.0
# A region whose sampled SM clock has a median below this fraction of the
# maximum, with the power cap active, ran in the limiter's steady state too.
CAPPED_CLOCK_FRAC = 0.75
MIN_CLOCK_SAMPLES = 5


def choose_tensor_peak(peaks, region_s: float, clocks=None):
    """The measured bf16 tensor-core peak that matches how a kernel was timed:
    the sustained figure (a seconds-long loop under the power cap) when the
    region lasted SUSTAINED_REGION_S seconds or more, or when its clock record
    (`clocks`, a ClockSampler summary: at least MIN_CLOCK_SAMPLES samples) shows
    the power cap active with the median SM clock below CAPPED_CLOCK_FRAC of the
    maximum; the burst figure (a cuBLAS GEMM timed alone) otherwise.
    Returns (peak, key, reason)."""
    if region_s >= SUSTAINED_REGION_S:
        return (peaks["bf16_tflops_sustained"], "bf16_tflops_sustained",
                f"timed region {region_s:.2f} s >= {SUSTAINED_REGION_S:.0f} s: sustained (power-capped) peak")
    c = clocks or {}
    mhz, max_mhz = c.get("sm_mhz"), c.get("sm_max_mhz")
    if (mhz and max_mhz and c.get("samples", 0) >= MIN_CLOCK_SAMPLES and "sw_power_cap" in c.get("reasons", ())
            and mhz < CAPPED_CLOCK_FRAC * max_mhz):
        return (peaks["bf16_tflops_sustained"], "bf16_tflops_sustained",
                f"timed region {region_s:.3f} s ran power-capped (median SM clock {mhz:.0f} of {max_mhz:.0f} MHz, "
                f"sw_power_cap, {c['samples']} samples): sustained peak")
    return (peaks["bf16_tflops"], "bf16_tflops",
            f"timed region {region_s:.3f} s < {SUSTAINED_REGION_S:.0f} s at the burst clock: burst peak")


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as fh:
            for line in fh:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            d = json.load(fh)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def traffic_record(kernel_file: str):
    """DRAM bytes per launch from the committed ncu summary, or None when the
    kernel source changed since the counters were taken."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    src = os.path.join(ROOT, "expert_router_gemm_b200", "csrc", kernel_file)
    if not (os.path.exists(path) and os.path.exists(src)):
        return None
    sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    out = {}
    for line in open(path):
        parts = line.split()
        if len(parts) >= 4 and not line.startswith("#") and parts[1] == sha:
            out[parts[0]] = float(parts[2]) + float(parts[3])
    return out or None


# ----------------------------------------------------------------- clocks (NVML, read only)
class ClockSampler:
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, torch_dev: int, period_s: float = 0.005):
        self.ok = False
        self.samples = []
        self.period = period_s
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(torch_dev)
            bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
            self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # pragma: no cover - depends on the box
            self.err = repr(e)

    def _reasons(self):
        nv = self.nv
        fn = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        return fn(self.h)

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append((nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM),
                                     nv.nvmlDeviceGetPowerUsage(self.h) / 1000.0,
                                     self._reasons()))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self._stop = threading.Event()
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        if self.ok:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        mhz = [s[0] for s in self.samples]
        bits = 0
        for s in self.samples:
            bits |= s[2]
        reasons = [n for b, n in self.REASONS.items() if bits & b and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(mhz), "power_w_max": round(max(s[1] for s in self.samples), 1)}


def wait_gpu(end_event) -> None:
    """Wait for a timed region's end event by polling: the wait sleeps between
    polls, so the clock sampler's thread keeps taking samples while the GPU
    works through the queued region (a blocking synchronize can starve it)."""
    import torch
    while not end_event.query():
        time.sleep(0.0002)
    torch.cuda.synchronize()


# ----------------------------------------------------------------- oracle timing (CPU)
def oracle_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        return max([i.get("num_threads", 1) for i in info if i.get("user_api") == "blas"] or [1])
    except Exception:
        return os.cpu_count() or 1


def oracle_expert_steps(w, inp, n_steps=None, budget_s=None, mx=False):
    """Time the fp64 oracle on a bounded sample of the workload: the routing of
    all T tokens once, then one expert per step (its kept rows through the SwiGLU
    FFN and their weighted contributions to the combine; with mx the oracle's
    block-scaled FP8 expert, quantization included).  Returns a list of
    (token_equivalents, seconds) per step and the routing time."""
    from oracle import moe_oracle as orc
    from oracle import mxfp8 as mxo
    t0 = time.perf_counter()
    g = orc.router_logits(inp.x, inp.w_router, inp.bias)
    s = orc.softmax(g)
    idx = orc.topk(g, w.k)
    wts = orc.topk_weights(s, idx)
    cap = orc.capacity(w.capacity_factor, w.T, w.k, w.N)
    disp = orc.dispatch(idx, w.N, cap, 128)
    orc.aux_stats(idx, s, w.N)
    t_route = time.perf_counter() - t0
    bf16 = w.dtype == "bf16"
    y = np.zeros((w.T, w.d))
    steps = []
    order = np.argsort(-disp.kept, kind="stable")   # busiest experts first: fixed order
    i = 0
    start = time.perf_counter()
    while True:
        if n_steps is not None and i >= n_steps:
            break
        if budget_s is not None and time.perf_counter() - start >= budget_s and i > 0:
            break
        e = int(order[i % w.N])
        ts = time.perf_counter()
        ti, tj = np.nonzero((idx == e) & (disp.row_map >= 0))
        if len(ti) and mx:
            o = mxo.swiglu_mx(mxo.mx_quantize(orc.as_f64(inp.x[ti])), mxo.quantize_weight(inp.w1[e]),
                              mxo.quantize_weight(inp.w3[e]), mxo.quantize_weight(inp.w2[e]))
            np.add.at(y, ti, wts[ti, tj][:, None] * o)
        elif len(ti):
            o = orc.swiglu_ffn(orc.as_f64(inp.x[ti]), inp.w1[e], inp.w3[e], inp.w2[e], bf16)
            np.add.at(y, ti, wts[ti, tj][:, None] * o)
        steps.append((len(ti) / w.k, time.perf_counter() - ts))
        i += 1
    return steps, t_route


# The CPU baseline times the whole layer on these workloads (each well under
# half a minute of fp64 work on 16 host cores); on the larger ones it times the
# routing of every token and the experts on a fixed sample of CPU_SAMPLE_TOKENS
# tokens, scaled to the batch.
FULL_LAYER_WORKLOADS = ("tiny-fp32", "mixtral-8x7b-shaped", "qwen3-moe-shaped")
CPU_SAMPLE_TOKENS = 1024


def oracle_layer_time(w, inp, sample_tokens=None, mx=False):
    """Time the fp64 oracle on one layer pass: routing, capacity clip and
    statistics of all T tokens, then every expert's kept rows through the SwiGLU
    FFN (FP8 oracle with mx) and the weighted combine, plus the shared expert.
    With sample_tokens the experts run only on the kept rows of a fixed sample
    of that many tokens (numpy seed 0).  Returns (route_s, ffn_s, ffn_tokens)."""
    from oracle import moe_oracle as orc
    from oracle import mxfp8 as mxo
    t0 = time.perf_counter()
    g = orc.router_logits(inp.x, inp.w_router, inp.bias)
    s = orc.softmax(g)
    idx = orc.topk(g, w.k)
    wts = orc.topk_weights(s, idx)
    cap = orc.capacity(w.capacity_factor, w.T, w.k, w.N)
    disp = orc.dispatch(idx, w.N, cap, 128)
    orc.aux_stats(idx, s, w.N)
    t_route = time.perf_counter() - t0
    if sample_tokens is None or sample_tokens >= w.T:
        tok = np.arange(w.T)
    else:
        tok = np.sort(np.random.default_rng(0).choice(w.T, sample_tokens, replace=False))
    bf16 = w.dtype == "bf16"
    t1 = time.perf_counter()
    x64 = orc.as_f64(inp.x[tok])
    sub_idx, sub_kept, sub_w = idx[tok], disp.row_map[tok] >= 0, wts[tok]
    y = np.zeros((len(tok), w.d))
    for e in range(w.N):
        ti, tj = np.nonzero((sub_idx == e) & sub_kept)
        if not len(ti):
            continue
        if mx:
            o = mxo.swiglu_mx(mxo.mx_quantize(x64[ti]), mxo.quantize_weight(inp.w1[e]),
                              mxo.quantize_weight(inp.w3[e]), mxo.quantize_weight(inp.w2[e]))
        else:
            o = orc.swiglu_ffn(x64[ti], inp.w1[e], inp.w3[e], inp.w2[e], bf16)
        np.add.at(y, ti, sub_w[ti, tj][:, None] * o)
    if w.f_shared:
        y += orc.swiglu_ffn(x64, inp.ws1, inp.ws3, inp.ws2, bf16)
    return t_route, time.perf_counter() - t1, len(tok)


def cpu_baseline_entry(w, inp, mx=False):
    """The cpu_baseline object of the bench line: the oracle as it stands, on the
    whole layer or on the fixed token sample (then labelled extrapolated)."""
    full = w.name in FULL_LAYER_WORKLOADS
    t_route, t_ffn, n = oracle_layer_time(w, inp, None if full else CPU_SAMPLE_TOKENS, mx=mx)
    sec = t_route + t_ffn * (w.T / n)
    what = "FP8 oracle experts" if mx else "SwiGLU experts"
    if full:
        sample = (f"fp64 oracle, whole layer: routing, capacity clip and statistics of all {w.T} tokens "
                  f"({t_route:.2f} s), then every expert's kept rows through the {what} and the combine "
                  f"({t_ffn:.2f} s)")
    else:
        sample = (f"fp64 oracle, extrapolated: routing of all {w.T} tokens ({t_route:.2f} s) plus the "
                  f"{what}, shared expert and combine on a fixed sample of {n} tokens ({t_ffn:.2f} s), "
                  f"scaled by {w.T}/{n}")
    return {"value": round(w.T / sec, 3), "unit": "tokens/s", "cores": oracle_threads(),
            "cpu_model": cpu_model(), "kind": "oracle", "sample": sample,
            "seconds": round(t_route + t_ffn, 2), "extrapolated": not full}


def cpu_rate(steps, t_route, T):
    tok = sum(s[0] for s in steps)
    sec = sum(s[1] for s in steps) + t_route * tok / T   # routing amortised per token
    return tok / sec if sec > 0 else 0.0, tok, sec


def run_reference(args, w, rank, world):
    """--impl reference: the fp64 oracle on the host cores (rank 0 only)."""
    if rank != 0:
        return
    inp = synth.make_inputs(w)
    warm, _ = oracle_expert_steps(w, inp, n_steps=args.warmup)
    steps, t_route = oracle_expert_steps(w, inp, n_steps=args.steps)
    rate, tok, sec = cpu_rate(steps, t_route, w.T)
    cores = oracle_threads()
    sample = (f"fp64 oracle: routing of all {w.T} tokens once (time amortised per token), "
              f"then per step the kept rows of one expert through the SwiGLU FFN and the "
              f"combine; {args.steps} steps = {tok:.0f} token-equivalents")
    line = {"impl": "reference", "metric": METRIC, "value": round(rate, 3), "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(1e3 * sec / max(1, len(steps)), 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(w),
            "cpu_baseline": {"value": round(rate, 3), "unit": "tokens/s", "cores": cores,
                             "cpu_model": cpu_model(), "kind": "oracle", "sample": sample},
            "e2e": {"value": round(rate, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def calibrate(cfg, w, dl, weights, stream, local, seconds=3.0):
    """Per-clock efficiency of the grouped GEMM pair (moe_expert_ffn) looped
    alone, next to a dense bf16 8192^3 GEMM of the vendor library (torch.matmul,
    a reference measurement only) on the same GPU.  Each runs ~`seconds` so that
    the power limiter settles; efficiency = TFLOP/s / (dense bf16 flops per SM
    clock x 148 SMs x median SM clock)."""
    import torch
    from expert_router_gemm_b200 import moe
    T, N, k, d, f = w.T, w.N, w.k, w.d, w.f
    _, ob, max_rows = moe.moe_workspace_size(cfg)
    ws = torch.empty(ob, dtype=torch.uint8, device="cuda")
    i32 = dict(dtype=torch.int32, device="cuda")
    idx, row_map = torch.empty((T, k), **i32), torch.empty((T, k), **i32)
    wt = torch.empty((T, k), dtype=torch.float32, device="cuda")
    seg_off, seg_count = torch.empty(N + 1, **i32), torch.empty(N, **i32)
    xp = torch.empty((max_rows, d), dtype=dl.x.dtype, device="cuda")
    h = torch.empty((max_rows, f), dtype=dl.x.dtype, device="cuda")
    o = torch.empty((max_rows, d), dtype=dl.x.dtype, device="cuda")
    st = moe.make_stats()
    moe.moe_route(cfg, dl.x, dl.w_router, dl.bias, None, None, idx, wt, st, ws, stream)
    moe.moe_dispatch(cfg, dl.x, idx, row_map, seg_off, seg_count, xp, st, ws, stream)
    torch.cuda.synchronize()
    kept = int(seg_count.sum().item())
    per_mhz = 8192 * 148 * 1e6 / 1e12   # dense bf16 TFLOP/s per MHz of SM clock (148 SMs)

    def loop(fn, flops):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        t0, n = time.time(), 0
        while time.time() - t0 < 0.3:
            fn()
            n += 1
        torch.cuda.synchronize()
        reps = max(5, int(seconds * n / (time.time() - t0)))
        smp = ClockSampler(local, period_s=0.01)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with smp:
            e0.record(stream)
            for _ in range(reps):
                fn()
            e1.record(stream)
            wait_gpu(e1)
        ms = e0.elapsed_time(e1) / reps
        c = smp.summary()
        tf = flops / ms / 1e9
        return {"ms": round(ms, 4), "TFLOP/s": round(tf, 1), "sm_mhz": c.get("sm_mhz"),
                "reasons": c.get("reasons"), "power_w_max": c.get("power_w_max"),
                "per_clock": round(tf / (per_mhz * c["sm_mhz"]), 4) if c.get("sm_mhz") else None}

    out = {"grouped_gemm_pair": loop(
        lambda: moe.moe_expert_ffn(cfg, xp, seg_off, seg_count, weights, h, o, ws, stream), 6.0 * d * f * kept)}
    a = torch.randn(8192, 8192, dtype=torch.bfloat16, device="cuda")
    b = torch.randn(8192, 8192, dtype=torch.bfloat16, device="cuda")
    c = torch.empty(8192, 8192, dtype=torch.bfloat16, device="cuda")
    out["reference_dense_bf16_gemm_8192^3"] = dict(
        loop(lambda: torch.matmul(a, b, out=c), 2.0 * 8192 ** 3), library="cuBLAS via torch.matmul (reference only)")
    return out


def workload_config(w):
    return {"workload": w.name, "T": w.T, "d": w.d, "N": w.N, "k": w.k, "f": w.f,
            "f_shared": w.f_shared, "capacity_factor": w.capacity_factor,
            "capacity": int(np.ceil(w.capacity_factor * w.T * w.k / w.N)),
            "act_dtype": w.dtype, "router_dtype": "f32", "seed": w.seed}


# ----------------------------------------------------------------- our arm
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", default="qwen3")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--quick", action="store_true", help="layer loop only (profiling runs)")
    ap.add_argument("--aux-free", type=float, default=0.0, metavar="GAMMA",
                    help="Aux-Loss-Free routing: a selection bias, updated on the device with "
                         "this step size after every layer call (0 = off)")
    ap.add_argument("--backward", action="store_true",
                    help="also time moe_layer_bwd (forward recompute + backward) and report it")
    ap.add_argument("--gemm", default="act", choices=["act", "mxfp8"],
                    help="number format of the routed experts' GEMMs: the activation dtype, or "
                         "block-scaled FP8 (weights quantized once before the timed region)")
    ap.add_argument("--calibrate", action="store_true",
                    help="also loop the grouped GEMM pair alone and a dense bf16 library GEMM "
                         "(cuBLAS, reference only) for ~3 s each and report their per-clock efficiency")
    ap.add_argument("--shape", default="",
                    help="override workload fields for small profiling cases, e.g. T=2048,N=32")
    args = ap.parse_args()
    if args.warmup < 3 and not args.quick:
        ap.error("--warmup must be >= 3")

    from expert_router_gemm_b200 import replicas
    ranks = replicas.from_env()
    rank, world, local = ranks.rank, ranks.world, ranks.local
    w = configs.get(args.config)
    if args.shape:
        from dataclasses import replace
        kv = dict(item.split("=") for item in args.shape.split(","))
        w = replace(w, name=f"{w.name}[{args.shape}]", **{key: int(v) for key, v in kv.items()})

    if args.impl == "reference":
        run_reference(args, w, rank, world)
        return

    import torch
    torch.cuda.set_device(local)
    replicas.init(ranks, "nccl", torch.device("cuda", local))

    from expert_router_gemm_b200 import moe

    inp = synth.make_inputs(w)
    mx = args.gemm == "mxfp8"
    cfg = moe.config_from_workload(w, gemm=args.gemm)
    dl = moe.to_device(inp, cfg)
    if mx:
        dl.quantize_mx()
        torch.cuda.synchronize()
        dl.w1 = dl.w3 = dl.w2 = None   # the FP8 layer reads only the quantized experts
        torch.cuda.empty_cache()
    # the router weight is constant across calls: its exact bf16 split (what the
    # tensor-core router multiplies) is made once, like the FP8 weights above
    if w.dtype == "bf16":
        dl.split_router()
    aux_free = args.aux_free > 0
    if aux_free:
        dl.selection_bias = torch.zeros(w.N, dtype=torch.float32, device="cuda")
    act = moe.act_dtype(cfg)
    elem = 2 if w.dtype == "bf16" else 4
    lb, ob, max_rows = moe.moe_workspace_size(cfg)
    ws = torch.empty(lb, dtype=torch.uint8, device="cuda")
    y = torch.empty((w.T, w.d), dtype=act, device="cuda")
    sbuf = dict(y_frac=torch.empty(w.N, device="cuda"), z_mean=torch.empty(w.N, device="cuda"),
                l_aux_p3=torch.empty(1, device="cuda"), l_aux_switch=torch.empty(1, device="cuda"),
                counts=torch.empty(w.N, dtype=torch.int32, device="cuda"),
                kept=torch.empty(w.N, dtype=torch.int32, device="cuda"),
                num_dropped=torch.empty(1, dtype=torch.int32, device="cuda"),
                z_loss=torch.empty(1, device="cuda"), load_std=torch.empty(1, device="cuda"),
                top2_ratio=torch.empty(1, device="cuda"),
                avg_tokens_per_expert=torch.empty(1, device="cuda"))
    stats = moe.make_stats(**sbuf)
    weights = dl.weights()
    stream = torch.cuda.current_stream()

    def layer_call(x_, y_):
        moe.moe_layer_fwd(cfg, weights, x_, y_, stats, ws, stream)
        if aux_free:
            moe.moe_bias_update(cfg, dl.selection_bias, sbuf["counts"], args.aux_free, stream)

    def layer():
        layer_call(dl.x, y)

    barrier = replicas.barrier

    def max_over_ranks(v: float) -> float:
        return replicas.max_over_ranks(v, torch.device("cuda", local))

    for _ in range(args.warmup):
        layer()
    torch.cuda.synchronize()
    flags = moe.moe_read_flags(ws)
    dropped = int(sbuf["num_dropped"].item())
    a_kept = w.T * w.k - dropped

    # ------------------------------------------------ region A: the layer call
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local)
    barrier()
    torch.cuda.synchronize()
    with sampler:
        ev0.record(stream)
        for _ in range(args.steps):
            layer()
        ev1.record(stream)
        wait_gpu(ev1)
    barrier()
    ms = max_over_ranks(ev0.elapsed_time(ev1)) / args.steps
    value = replicas.job_throughput(w.T, world, ms / 1e3)
    clocks = sampler.summary()

    # route: bf16 runs the tensor-core router GEMM (on the split made once) and
    # the softmax / top-k kernel (fp32: one fused kernel); dispatch: mask, scan,
    # scatter; two grouped GEMMs (+ two for the shared expert); combine; the bias
    # update
    per_step_launches = ((2 if w.dtype == "bf16" else 1) + 3 + 2 + (2 if w.f_shared else 0) + 1
                         + (1 if aux_free else 0))
    router_stats = {key: round(float(sbuf[key].item()), 6) for key in
                    ("l_aux_p3", "l_aux_switch", "z_loss", "load_std", "top2_ratio",
                     "avg_tokens_per_expert")}
    line = {"metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "mxfp8 experts (e4m3, bf16 in/out)" if mx else w.dtype,
            "data": "synthetic",
            "config": dict(workload_config(w), expert_gemm=args.gemm, parallelism=f"replicas x{world}",
                           router_split=("made once before the loop (moe_router_split)"
                                         if w.dtype == "bf16" else None),
                           l2="inputs larger than L2: the expert weights read every step "
                              f"({(inp.w1.nbytes + inp.w3.nbytes + inp.w2.nbytes) / 1e9:.2f} GB) "
                              "exceed the 126 MB L2; no flush"),
            "gpu_launches": per_step_launches * args.steps, "clocks": clocks,
            "device_flags": flags, "dropped": dropped, "router_stats": router_stats}
    if aux_free:
        line["config"]["aux_loss_free_gamma"] = args.aux_free
        b_last = dl.selection_bias.cpu()
        line["selection_bias_range"] = [round(float(b_last.min()), 6), round(float(b_last.max()), 6)]

    if not args.quick:
        # -------------------------------------------- region B: per-stage events
        T, N, k, d, f = w.T, w.N, w.k, w.d, w.f
        ws_op = torch.empty(ob, dtype=torch.uint8, device="cuda")
        idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
        wt = torch.empty((T, k), dtype=torch.float32, device="cuda")
        row_map = torch.empty((T, k), dtype=torch.int32, device="cuda")
        seg_off = torch.empty(N + 1, dtype=torch.int32, device="cuda")
        seg_count = torch.empty(N, dtype=torch.int32, device="cuda")
        xp = torch.empty((max_rows, d), dtype=act, device="cuda")
        h = torch.empty((max_rows, f), dtype=act, device="cuda")
        if mx:
            x8 = torch.empty((max_rows, d), dtype=torch.uint8, device="cuda")
            x8sf = torch.empty(moe.mx_sf_bytes(max_rows, d), dtype=torch.uint8, device="cuda")
            h8sf = torch.empty(moe.mx_sf_bytes(max_rows, f), dtype=torch.uint8, device="cuda")
        hs = torch.empty((T, w.f_shared), dtype=act, device="cuda") if w.f_shared else None
        sh = torch.empty((T, d), dtype=act, device="cuda") if w.f_shared else None
        names = ["route", "dispatch", "expert_ffn", "shared_ffn", "combine"] + (
            ["bias_update"] if aux_free else [])

        def staged(evs):
            evs[0].record(stream)
            # the layer's routing as moe_layer_fwd runs it: with the split made once
            moe.moe_route_with_split(cfg, dl.x, dl.w_router, dl.router_split, dl.bias, dl.selection_bias, None,
                                     idx, wt, stats, ws_op, stream)
            evs[1].record(stream)
            if mx:
                moe.moe_dispatch_mx(cfg, dl.x, idx, row_map, seg_off, seg_count, x8, x8sf, stats, ws_op,
                                    stream)
            else:
                moe.moe_dispatch(cfg, dl.x, idx, row_map, seg_off, seg_count, xp, stats, ws_op, stream)
            evs[2].record(stream)
            if mx:
                moe.moe_expert_ffn_mx(cfg, x8, x8sf, seg_off, seg_count, weights, h, h8sf, xp, ws_op,
                                      stream)
            else:
                moe.moe_expert_ffn(cfg, xp, seg_off, seg_count, weights, h, xp, ws_op, stream)
            evs[3].record(stream)
            if w.f_shared:
                moe.moe_shared_expert_ffn(cfg, dl.x, weights, hs, sh, ws_op, stream)
            evs[4].record(stream)
            moe.moe_combine(cfg, xp, row_map, wt, sh, y, ws_op, stream)
            evs[5].record(stream)
            if aux_free:
                moe.moe_bias_update(cfg, dl.selection_bias, sbuf["counts"], args.aux_free, stream)
                evs[6].record(stream)

        n_ev = len(names) + 1
        for _ in range(3):
            staged([torch.cuda.Event(enable_timing=True) for _ in range(n_ev)])
        all_evs = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(args.steps)]
        rb0, rb1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        bsampler = ClockSampler(local)
        barrier()
        torch.cuda.synchronize()
        with bsampler:
            rb0.record(stream)
            for evs in all_evs:
                staged(evs)
            rb1.record(stream)
            wait_gpu(rb1)
        region_b_s = max_over_ranks(rb0.elapsed_time(rb1)) / 1e3
        clocks_b = bsampler.summary()
        stage_ms = {n: 0.0 for n in names}
        for evs in all_evs:
            for i, n in enumerate(names):
                stage_ms[n] += evs[i].elapsed_time(evs[i + 1])
        stage_ms = {n: max_over_ranks(v) / args.steps for n, v in stage_ms.items()}

        peaks, peak_src = load_peaks()
        hbm = peaks["hbm_gbs"]
        # the stage times come from region B: its length and clocks decide burst vs sustained
        tc_peak, tc_key, tc_reason = choose_tensor_peak(peaks, region_b_s, clocks_b)
        # the FP8 GEMM's peak: the measured bf16 figure times the nominal FP8 : bf16
        # dense ratio (4.5 : 2.25 PFLOP/s)
        gemm_peak = 2.0 * tc_peak if mx else tc_peak
        x_bytes = T * d * elem
        route_bytes = x_bytes + d * N * 4 + T * k * 8
        route_flops = 2.0 * T * d * N
        if mx:   # rows written as 1-byte codes plus one scale byte per 32 values
            disp_bytes = x_bytes + a_kept * d * (1 + 1 / 32) + T * k * 8
        else:
            disp_bytes = x_bytes + a_kept * d * elem + T * k * 8
        ffn_flops = 6.0 * d * f * a_kept
        ffn_wbytes = 3.0 * N * d * f * ((1 + 1 / 32) if mx else elem)
        comb_bytes = a_kept * d * elem + T * k * 8 + x_bytes + (x_bytes if w.f_shared else 0)
        sh_flops = 6.0 * T * d * w.f_shared

        def gbs(b, ms_):
            return b / (ms_ / 1e3) / 1e9 if ms_ > 0 else None

        def tfs(fl, ms_):
            return fl / (ms_ / 1e3) / 1e12 if ms_ > 0 else None

        tc_router = w.dtype == "bf16"
        route_entry = {"ms": round(stage_ms["route"], 4), "bytes": route_bytes, "flops": route_flops,
                       "GB/s": round(gbs(route_bytes, stage_ms["route"]), 1),
                       "frac_hbm": round(gbs(route_bytes, stage_ms["route"]) / hbm, 4),
                       "TFLOP/s_fp32_equiv": round(tfs(route_flops, stage_ms["route"]), 2)}
        if tc_router:
            # tensor cores: three bf16 MMAs per fp32 weight (exact split)
            route_entry["engine"] = "tcgen05, 3-part bf16 split"
            route_entry["frac_tensor_executed"] = round(
                tfs(3 * route_flops, stage_ms["route"]) / tc_peak, 4)
        else:
            route_entry["engine"] = "CUDA-core FFMA"
            route_entry["frac_fp32_alu"] = round(tfs(route_flops, stage_ms["route"]) / FP32_ALU_TFLOPS, 4)
        kern = {
            "route": route_entry,
            "dispatch": {"ms": round(stage_ms["dispatch"], 4), "bytes": disp_bytes,
                         "GB/s": round(gbs(disp_bytes, stage_ms["dispatch"]), 1),
                         "frac_hbm": round(gbs(disp_bytes, stage_ms["dispatch"]) / hbm, 4)},
            "expert_ffn": {"ms": round(stage_ms["expert_ffn"], 4), "flops": ffn_flops,
                           "TFLOP/s": round(tfs(ffn_flops, stage_ms["expert_ffn"]), 1),
                           "frac_tensor": round(tfs(ffn_flops, stage_ms["expert_ffn"]) / gemm_peak, 4),
                           "weight_bytes": ffn_wbytes,
                           "weight_GB/s": round(gbs(ffn_wbytes, stage_ms["expert_ffn"]), 1)},
            "combine": {"ms": round(stage_ms["combine"], 4), "bytes": comb_bytes,
                        "GB/s": round(gbs(comb_bytes, stage_ms["combine"]), 1),
                        "frac_hbm": round(gbs(comb_bytes, stage_ms["combine"]) / hbm, 4)},
        }
        if aux_free:
            kern["bias_update"] = {"ms": round(stage_ms["bias_update"], 5)}
        if w.f_shared:
            kern["shared_ffn"] = {"ms": round(stage_ms["shared_ffn"], 4), "flops": sh_flops,
                                  "TFLOP/s": round(tfs(sh_flops, stage_ms["shared_ffn"]), 1)}
        line["kernels"] = kern
        line["stage_sum_ms"] = round(sum(stage_ms.values()), 4)
        ffn_tf = tfs(ffn_flops, stage_ms["expert_ffn"])
        # the DRAM records were captured on the Qwen3-shaped workload's per-expert shapes
        tr = (traffic_record("ffn_mx.cu" if mx else "ffn_tc.cu")
              if w.name == configs.QWEN3.name and not args.shape else None)
        fp8x = 2.0 if mx else 1.0
        line["roofline"] = {
            "kernel": ("tc_mx_gemm_kernel (block-scaled FP8 grouped SwiGLU GEMM + down GEMM, the two "
                       "launches of moe_expert_ffn_mx)") if mx else
                      ("tc_ffn_gemm_kernel (grouped SwiGLU GEMM + down GEMM, the two launches of "
                       "moe_expert_ffn)"),
            "bound": "tensor", "achieved": round(ffn_tf, 1), "peak": gemm_peak, "unit": "TFLOP/s",
            "frac": round(ffn_tf / gemm_peak, 4),
            "peak_source": (f"{peak_src} {tc_key} x 2 (nominal FP8 : bf16 dense ratio); {tc_reason}" if mx
                            else f"{peak_src} {tc_key}; {tc_reason}"),
            "frac_of_burst_peak": round(ffn_tf / (peaks["bf16_tflops"] * fp8x), 4),
            "frac_of_sustained_peak": round(ffn_tf / (peaks["bf16_tflops_sustained"] * fp8x), 4),
            "region_s": round(region_b_s, 4), "region_clocks": clocks_b,
            # kernel time x median SM clock of its region = thousands of SM cycles per step
            "kcycles_per_step": (round(stage_ms["expert_ffn"] * clocks_b["sm_mhz"], 1)
                                 if clocks_b.get("sm_mhz") else None),
            "algorithmic_flops_per_step": ffn_flops,
            # the other roofline of the same kernel: its expert weights stream from HBM
            # once per call (the bound on layers with few rows per expert)
            "weight_stream": {"bytes_per_step": ffn_wbytes,
                              "GB/s": round(gbs(ffn_wbytes, stage_ms["expert_ffn"]), 1),
                              "frac_hbm": round(gbs(ffn_wbytes, stage_ms["expert_ffn"]) / hbm, 4),
                              "hbm_peak_gbs": hbm},
            "traffic": (tr["expert_ffn_per_step"] * 1.0 if tr and "expert_ffn_per_step" in tr else None)}

        # -------------------------------------------- e2e: host buffers through the C ABI
        # Every step copies its batch in from pinned host memory and its output
        # back out.  Two buffers per side and two copy streams let the copy-in of
        # step i+1 and the copy-out of step i-1 run while step i computes (the
        # usual way to drive the layer from the host); the serial variant, with
        # copy-in, layer and copy-out back to back, is reported as well.
        x_host = [torch.empty_like(dl.x, device="cpu").pin_memory() for _ in range(2)]
        for xh in x_host:
            xh.copy_(dl.x.cpu())
        y_host = [torch.empty((T, d), dtype=act).pin_memory() for _ in range(2)]
        x_in = [torch.empty_like(dl.x) for _ in range(2)]
        y_dev = [y, torch.empty_like(y)]
        h2d, d2h = torch.cuda.Stream(), torch.cuda.Stream()
        ev = lambda: torch.cuda.Event(enable_timing=False)  # noqa: E731
        h2d_done, comp_done, d2h_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]
        for b in range(2):
            for e_ in (h2d_done[b], comp_done[b], d2h_done[b]):
                e_.record(stream)

        def e2e_step(i):
            b = i % 2
            h2d.wait_event(comp_done[b])          # step i-2 has finished reading x_in[b]
            with torch.cuda.stream(h2d):
                x_in[b].copy_(x_host[b], non_blocking=True)
            h2d_done[b].record(h2d)
            stream.wait_event(h2d_done[b])
            stream.wait_event(d2h_done[b])        # step i-2's output has left y_dev[b]
            layer_call(x_in[b], y_dev[b])
            comp_done[b].record(stream)
            d2h.wait_event(comp_done[b])
            with torch.cuda.stream(d2h):
                y_host[b].copy_(y_dev[b], non_blocking=True)
            d2h_done[b].record(d2h)

        def timed(body, n):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            barrier()
            torch.cuda.synchronize()
            e0.record(stream)
            h2d.wait_stream(stream)
            d2h.wait_stream(stream)
            for i in range(n):
                body(i)
            stream.wait_stream(h2d)
            stream.wait_stream(d2h)
            e1.record(stream)
            torch.cuda.synchronize()
            return max_over_ranks(e0.elapsed_time(e1)) / n

        def serial_step(i):
            with torch.cuda.stream(stream):
                x_in[0].copy_(x_host[0], non_blocking=True)
            layer_call(x_in[0], y_dev[0])
            with torch.cuda.stream(stream):
                y_host[0].copy_(y_dev[0], non_blocking=True)

        for i in range(3):
            e2e_step(i)
        e2e_ms = timed(e2e_step, args.steps)
        serial_ms = timed(serial_step, args.steps)
        line["e2e"] = {"value": round(world * T / (e2e_ms / 1e3), 1), "unit": "tokens/s",
                       "h2d_bytes_per_step": x_host[0].numel() * x_host[0].element_size(),
                       "d2h_bytes_per_step": y_host[0].numel() * y_host[0].element_size(),
                       "ms_per_step": round(e2e_ms, 4),
                       "copies": "overlapped with the neighbouring steps' compute (2 copy streams)",
                       "serial_value": round(world * T / (serial_ms / 1e3), 1),
                       "serial_ms_per_step": round(serial_ms, 4)}

    if not args.quick:
        # -------------------------------------------- steady state: the layer loop run for
        # >= 3 s, long enough for the power limiter to settle (the SM clock a user gets
        # from back-to-back layers; the short region A above runs at the burst clock)
        reps = max(args.steps, int(np.ceil(3000.0 / max(ms, 1e-3))))
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ssampler = ClockSampler(local)
        barrier()
        torch.cuda.synchronize()
        with ssampler:
            s0.record(stream)
            for _ in range(reps):
                layer()
            s1.record(stream)
            wait_gpu(s1)
        barrier()
        s_ms = max_over_ranks(s0.elapsed_time(s1)) / reps
        line["steady_state"] = {"steps": reps, "seconds": round(s_ms * reps / 1e3, 2),
                                "ms_per_step": round(s_ms, 4),
                                "tokens/s": round(replicas.job_throughput(w.T, world, s_ms / 1e3), 1),
                                "clocks": ssampler.summary()}

    if args.backward and not mx:
        # -------------------------------------------- the layer backward
        # One step = moe_layer_bwd: the forward recomputed from x (routing, permutation,
        # GEMM1 saving g and u, GEMM2), then the gradients of every input and weight.
        T, N, k, d, f, fs = w.T, w.N, w.k, w.d, w.f, w.f_shared
        gb = dict(dx=torch.empty((T, d), dtype=act, device="cuda"),
                  dw_router=torch.empty((d, N), device="cuda"),
                  drouter_bias=torch.empty(N, device="cuda") if dl.bias is not None else None,
                  dw1=torch.empty((N, d, f), device="cuda"), dw3=torch.empty((N, d, f), device="cuda"),
                  dw2=torch.empty((N, f, d), device="cuda"))
        if fs:
            gb.update(dws1=torch.empty((d, fs), device="cuda"), dws3=torch.empty((d, fs), device="cuda"),
                      dws2=torch.empty((fs, d), device="cuda"))
        grads = moe.make_grads(**gb)
        ws_b = torch.empty(moe.moe_backward_workspace_size(cfg), dtype=torch.uint8, device="cuda")
        dy = torch.randn((T, d), generator=torch.Generator().manual_seed(5)).to(torch.bfloat16).view(
            torch.int16).cuda()

        def bwd_step():
            moe.moe_layer_bwd(cfg, weights, dl.x, dy, 0.01, 1e-3, grads, ws_b, stream)

        for _ in range(max(3, args.warmup)):
            bwd_step()
        torch.cuda.synchronize()
        bflags = moe.moe_read_flags(ws_b)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n_b = max(1, args.steps // 2)
        bsampler = ClockSampler(local)
        barrier()
        torch.cuda.synchronize()
        with bsampler:
            e0.record(stream)
            for _ in range(n_b):
                bwd_step()
            e1.record(stream)
            wait_gpu(e1)
        barrier()
        bms = max_over_ranks(e0.elapsed_time(e1)) / n_b
        # GEMM work of one step: forward recompute (6 d f per kept row), dgrad (6 d f)
        # and weight gradients (6 d f), plus the shared expert's 2 + 4 + 6 d fs per token
        gemm_fl = 18.0 * d * f * a_kept + (12.0 + 6.0) * T * d * fs
        peaks, peak_src = load_peaks()
        b_clocks = bsampler.summary()
        b_peak, b_key, b_reason = choose_tensor_peak(peaks, bms * n_b / 1e3, b_clocks)
        line["backward"] = {
            "what": "moe_layer_bwd: forward recomputed from x, then dx and every weight gradient (fp32)",
            "steps": n_b, "ms_per_step": round(bms, 4), "tokens/s": round(world * T / (bms / 1e3), 1),
            "gemm_flops_per_step": gemm_fl, "gemm_TFLOP/s": round(gemm_fl / (bms / 1e3) / 1e12, 1),
            "frac_of_bf16_peak": round(gemm_fl / (bms / 1e3) / 1e12 / b_peak, 4),
            "peak_source": f"{peak_src} {b_key}; {b_reason}", "device_flags": bflags,
            "clocks": b_clocks}

    if args.calibrate and world == 1 and not mx and w.dtype == "bf16":
        line["calibration"] = calibrate(cfg, w, dl, weights, stream, local)

    if rank == 0 and world == 1 and not args.no_cpu_baseline and not args.quick:
        line["cpu_baseline"] = cpu_baseline_entry(w, inp, mx=mx)

    if rank == 0:
        print(json.dumps(line), flush=True)
    replicas.finish()


if __name__ == "__main__":
    main()
