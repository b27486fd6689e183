"""Host logic of bench.py on the CPU: the DRAM-traffic records keyed to kernel
sources, the peak table and its fallback, the CPU-rate arithmetic, and the JSON
line of the reference arm (the fp64 oracle, which needs no GPU)."""
import hashlib
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _fake_root(tmp_path, kernel_src: bytes, records: str):
    (tmp_path / "profiles").mkdir()
    (tmp_path / "expert_router_gemm_b200" / "csrc").mkdir(parents=True)
    (tmp_path / "expert_router_gemm_b200" / "csrc" / "k.cu").write_bytes(kernel_src)
    (tmp_path / "profiles" / "dram_traffic.txt").write_text(records)
    return hashlib.sha256(kernel_src).hexdigest()[:16]


def test_traffic_record_applies_only_to_the_captured_source(tmp_path, monkeypatch):
    sha = _fake_root(tmp_path, b"kernel v1", "")
    (tmp_path / "profiles" / "dram_traffic.txt").write_text(
        "# comment line " + sha + " 1 2\n"
        f"expert_ffn_per_step {sha} 100.5e6 20e6\n"
        "expert_ffn_per_step 0123456789abcdef 7e6 8e6\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.traffic_record("k.cu") == {"expert_ffn_per_step": pytest.approx(120.5e6)}
    # the source changes: the counters no longer describe it
    (tmp_path / "expert_router_gemm_b200" / "csrc" / "k.cu").write_bytes(b"kernel v2")
    assert bench.traffic_record("k.cu") is None
    assert bench.traffic_record("missing.cu") is None


def test_committed_traffic_records_are_well_formed():
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    lines = [ln.split() for ln in open(path) if ln.strip() and not ln.startswith("#")]
    assert lines
    for unit, sha, rd, wr in lines:
        assert unit == "expert_ffn_per_step"
        assert len(sha) == 16 and int(sha, 16) >= 0
        assert float(rd) > 0 and float(wr) > 0


def test_peaks_fall_back_when_the_measured_file_is_absent(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    peaks, src = bench.load_peaks()
    assert src == "fallback" and peaks == bench.FALLBACK_PEAKS
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 1.0, "bf16_tflops": 2.0,
                                                             "bf16_tflops_sustained": 3.0}))
    peaks, src = bench.load_peaks()
    assert src == "measured" and peaks["bf16_tflops_sustained"] == 3.0


def test_cpu_rate_amortises_the_routing_per_token():
    # two steps of 100 and 300 token-equivalents in 1 s and 3 s, routing of
    # T = 1000 tokens in 2 s: 400 tokens cost 4 s + 2 * 400 / 1000 s
    rate, tok, sec = bench.cpu_rate([(100, 1.0), (300, 3.0)], 2.0, 1000)
    assert tok == 400 and sec == pytest.approx(4.8)
    assert rate == pytest.approx(400 / 4.8)
    assert bench.cpu_rate([], 0.0, 10)[0] == 0.0


def test_reference_arm_json_line():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--config", "tiny", "--steps", "2",
                        "--warmup", "3"], cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-2000:]
    lines = [json.loads(x) for x in r.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1
    line = lines[0]
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC
    assert line["n_gpus"] == 1 and line["steps"] == 2 and line["warmup"] == 3
    assert line["value"] > 0 and line["unit"] == "tokens/s" and line["higher_is_better"] is True
    assert line["config"]["workload"] == "tiny-fp32"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["cpu_baseline"]["cpu_model"]
    assert line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"] == {"value": line["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}


def test_clock_summary_decodes_reasons_and_takes_the_median():
    s = bench.ClockSampler.__new__(bench.ClockSampler)
    s.ok, s.max_mhz = True, 1965
    # (SM MHz, watts, clocks-event-reason bits): idle is not reported, the others are
    s.samples = [(1200, 700.0, 0x1), (1100, 990.0, 0x4), (1300, 650.0, 0x4 | 0x40)]
    c = s.summary()
    assert c["sm_mhz"] == 1200 and c["sm_max_mhz"] == 1965 and c["samples"] == 3
    assert c["power_w_max"] == 990.0
    assert c["reasons"] == ["sw_power_cap", "hw_thermal_slowdown"]
    s.samples = []
    assert s.summary()["samples"] == 0
    s.ok = False
    assert s.summary()["sm_mhz"] is None


def test_workload_config_names_the_workload_and_its_sizes():
    from expert_router_gemm_b200 import configs
    w = configs.get("qwen3")
    c = bench.workload_config(w)
    assert c["workload"] == "qwen3-moe-shaped"
    assert (c["T"], c["d"], c["N"], c["k"], c["f"]) == (8192, 4096, 128, 8, 1536)
    assert c["capacity"] == 512 and c["act_dtype"] == "bf16" and c["router_dtype"] == "f32"
    assert "model" not in c


def test_tensor_peak_follows_the_length_and_clocks_of_the_timed_region():
    peaks = {"hbm_gbs": 6538.0, "bf16_tflops": 1674.7, "bf16_tflops_sustained": 1364.1}
    p, key, why = bench.choose_tensor_peak(peaks, 0.042)     # 20 layer steps: a burst
    assert (p, key) == (1674.7, "bf16_tflops") and "burst" in why
    p, key, why = bench.choose_tensor_peak(peaks, bench.SUSTAINED_REGION_S)
    assert (p, key) == (1364.1, "bf16_tflops_sustained") and "sustained" in why
    p, key, _ = bench.choose_tensor_peak(peaks, 12.0)
    assert key == "bf16_tflops_sustained"
    # a short region decides by its clock record: capped and slow -> sustained
    capped = {"sm_mhz": 990.0, "sm_max_mhz": 1965, "reasons": ["sw_power_cap"], "samples": 106}
    p, key, why = bench.choose_tensor_peak(peaks, 0.53, capped)
    assert key == "bf16_tflops_sustained" and "990" in why
    # at the burst clock, with too few samples, or without the cap: burst
    for c in (dict(capped, sm_mhz=1965.0), dict(capped, samples=2), dict(capped, reasons=[]), None,
              {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}):
        assert bench.choose_tensor_peak(peaks, 0.53, c)[1] == "bf16_tflops", c


def test_cpu_model_is_named():
    m = bench.cpu_model()
    assert isinstance(m, str) and m and m != "unknown"


def test_cpu_baseline_covers_the_whole_small_layer():
    from expert_router_gemm_b200 import configs, synth
    w = configs.get("tiny")
    e = bench.cpu_baseline_entry(w, synth.make_inputs(w))
    assert e["kind"] == "oracle" and e["extrapolated"] is False and e["value"] > 0
    assert e["cores"] >= 1 and e["cpu_model"] and "whole layer" in e["sample"]
    assert "tiny-fp32" in bench.FULL_LAYER_WORKLOADS and "qwen3-moe-shaped" in bench.FULL_LAYER_WORKLOADS


def test_waiting_for_a_timed_region_polls_and_lets_other_threads_run(monkeypatch):
    """wait_gpu polls the region's end event with short sleeps (a blocking
    synchronize kept the clock sampler's thread from running), then
    synchronises once the event has completed."""
    import threading
    import torch

    calls = {"sync": 0}
    monkeypatch.setattr(torch.cuda, "synchronize", lambda *a, **k: calls.__setitem__("sync", calls["sync"] + 1))

    class Event:
        def __init__(self):
            self.n = 0

        def query(self):
            self.n += 1
            return self.n >= 50

    ticks = []
    stop = threading.Event()

    def sampler():
        while not stop.is_set():
            ticks.append(1)
            stop.wait(0.0005)

    t = threading.Thread(target=sampler)
    t.start()
    ev = Event()
    bench.wait_gpu(ev)
    stop.set()
    t.join()
    assert ev.n == 50 and calls["sync"] == 1
    assert len(ticks) > 1          # the other thread ran while the wait polled
