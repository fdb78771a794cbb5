"""Host-side parts of bench.py, on CPU: the reference arm (which runs the oracle
on the host) prints one JSON line of the contract's shape, stops at its
wall-clock budget and runs on rank 0 only; the oracle's layer time is
extrapolated per kept assignment; the tensor peak follows the run's clock; the
DRAM-traffic lookup reports the committed capture only while the kernel
sources hash to the captured version; the per-clock figure is the rate against
8192 FLOP per SM clock."""
from __future__ import annotations

import hashlib
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench(args, env_extra=None, timeout=300):
    env = dict(os.environ)
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        env.pop(k, None)
    env.update(env_extra or {})
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], capture_output=True, text=True,
                       timeout=timeout, env=env, cwd=ROOT)
    lines = [ln for ln in p.stdout.splitlines() if ln.startswith("{")]
    return p, lines


def test_reference_arm_prints_one_contract_line():
    p, lines = _bench(["--impl", "reference", "--workload", "tiny_f32", "--steps", "3", "--warmup", "1"])
    assert p.returncode == 0, p.stderr[-2000:]
    assert len(lines) == 1
    j = json.loads(lines[0])
    assert j["impl"] == "reference" and j["metric"] == "MoE-layer tokens/s" and j["unit"] == "tokens/s"
    assert j["value"] > 0 and j["higher_is_better"] is True and j["n_gpus"] == 1
    assert j["steps"] == 3 and j["steps_requested"] == 3 and j["warmup"] == 1
    # value = the layer's T tokens over the oracle's (extrapolated) layer time per step
    assert abs(j["value"] - 64 * 1000.0 / j["ms_per_step"]) <= 1e-9 * j["value"]
    cb = j["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == j["value"] and cb["unit"] == "tokens/s" and cb["cores"] >= 1
    assert cb["nproc"] >= 1
    assert j["e2e"] == {"value": j["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert j["config"]["workload"] == "tiny_f32" and j["config"]["T"] == 64


def test_oracle_layer_time_extrapolates_per_kept_assignment():
    sys.path.insert(0, ROOT)
    import bench
    from synth import configs

    w = configs.scaled(configs.WORKLOADS["mid_bf16"], name="small", T=96, d=64, f=128)
    host = dict(wr=configs.make_router(w), wg=configs.make_w_gate(w), wu=configs.make_w_up(w),
                wd=configs.make_w_down(w))
    r = bench.oracle_layer_time(w, host, configs.make_x(w), 16, 3, threads=1)
    assert r["sample_tokens"] == 16 and 0 < r["kept_in_sample"] <= 32 and r["threads"] == 1
    assert r["extrapolation"] == r["n_kept"] / r["kept_in_sample"]
    assert abs(r["layer_s"] - (r["route_s"] + r["ffn_sample_s"] * r["extrapolation"])) <= 1e-12
    assert abs(r["tokens_per_s"] - w.T / r["layer_s"]) <= 1e-9 * r["tokens_per_s"]


def test_tensor_peak_follows_the_run_clock():
    sys.path.insert(0, ROOT)
    import bench

    peaks = {"bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0, "clocks_under_load": {"sm_mhz_median": 1400}}
    p, rule = bench.tensor_peak(peaks, "measured", {"sm_mhz": 1940.0, "sm_max_mhz": 1965.0})
    assert p == 1600.0 and "burst" in rule
    p, rule = bench.tensor_peak(peaks, "measured", {"sm_mhz": 1200.0, "sm_max_mhz": 1965.0})
    assert p == 1400.0 * 1200.0 / 1400.0 and "sustained" in rule
    # never above the burst figure
    p, _ = bench.tensor_peak(peaks, "measured", {"sm_mhz": 1800.0, "sm_max_mhz": 1965.0})
    assert p == 1600.0
    p, _ = bench.tensor_peak({"bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0}, "measured", {})
    assert p == 1400.0


def test_reference_arm_stops_at_its_budget():
    p, lines = _bench(["--impl", "reference", "--workload", "tiny_f32", "--steps", "1000000", "--warmup", "0",
                       "--ref-budget-s", "0.5"])
    assert p.returncode == 0, p.stderr[-2000:]
    j = json.loads(lines[-1])
    assert 1 <= j["steps"] < 1000000 and j["steps_requested"] == 1000000
    # the budget bounds the timed work: the next step would have passed it
    assert j["steps"] * j["ms_per_step"] / 1000.0 <= 0.5 + 2 * j["ms_per_step"] / 1000.0


def test_reference_arm_runs_on_rank_zero_only():
    p, lines = _bench(["--impl", "reference", "--workload", "tiny_f32", "--steps", "2", "--warmup", "0"],
                      env_extra={"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert p.returncode == 0, p.stderr[-2000:]
    assert lines == []


def test_traffic_lookup_follows_the_kernel_sources(tmp_path, monkeypatch):
    sys.path.insert(0, ROOT)
    import bench

    h = hashlib.sha256()
    for src in bench.KERNEL_SOURCES:
        with open(src, "rb") as fh:
            h.update(fh.read())
    body = {"workloads": {"grok_prefill": {"gate_up": {"dram_bytes_per_launch": 123456}}}}
    good = tmp_path / "good.json"
    good.write_text(json.dumps(dict(body, kernel_sources_sha256=h.hexdigest())))
    stale = tmp_path / "stale.json"
    stale.write_text(json.dumps(dict(body, kernel_sources_sha256="0" * 64)))
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(good))
    assert bench.measured_traffic("grok_prefill") == 123456.0
    assert bench.measured_traffic("grok_prefill", "down") is None
    assert bench.measured_traffic("mid_bf16") is None  # no capture of that workload
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(stale))
    assert bench.measured_traffic("grok_prefill") is None
    # every header the grouped GEMM kernel includes is hashed
    names = {os.path.basename(p) for p in bench.KERNEL_SOURCES}
    assert {"ffn_tc.cu", "tc_ptx.cuh", "common.cuh", "internal.h"} <= names


def test_clock_sampler_parses_and_filters_by_gpu(tmp_path, monkeypatch):
    """A stand-in nvidia-smi on PATH prints samples of two GPUs; the sampler keeps
    the named GPU's, takes the median SM clock and collects the active reasons."""
    sys.path.insert(0, ROOT)
    import bench

    fake = tmp_path / "nvidia-smi"
    fake.write_text(
        "#!/bin/sh\n"
        "echo 'GPU-a, 1200, 1965, 900.5, Not Active, Not Active, Not Active, Active'\n"
        "echo 'GPU-b, 300, 1965, 100.0, Active, Not Active, Not Active, Not Active'\n"
        "echo 'GPU-a, 1300, 1965, 1001.0, Not Active, Not Active, Not Active, Active'\n"
        "echo 'GPU-a, 1250, 1965, 950.0, Not Active, Not Active, Not Active, Not Active'\n"
        "sleep 30\n")
    fake.chmod(0o755)
    monkeypatch.setenv("PATH", str(tmp_path) + os.pathsep + os.environ.get("PATH", ""))
    s = bench.ClockSampler("GPU-a")
    s.start()
    import time

    for _ in range(100):
        if len(s.rows) >= 3:
            break
        time.sleep(0.05)
    r = s.stop(window=(0.0, time.monotonic()))
    assert r["samples"] == 3 and r["sm_mhz"] == 1250.0 and r["sm_max_mhz"] == 1965.0
    assert r["reasons"] == ["sw_power_cap"] and r["power_w_max"] == 1001.0


def test_per_clock_rate_against_the_nominal_sm_rate():
    sys.path.insert(0, ROOT)
    import bench

    # 148 SMs x 8192 FLOP per clock at 1300 MHz is 1576 TFLOP/s: that rate is 1.0 of nominal
    full = 148 * 8192 * 1300e6 / 1e12
    r = bench.per_clock(full, {"sm_mhz": 1300.0})
    assert abs(r["frac_of_nominal"] - 1.0) < 1e-12 and abs(r["flop_per_clock_per_sm"] - 8192.0) < 1e-9
    r = bench.per_clock(full / 2, {"sm_mhz": 1300.0})
    assert abs(r["frac_of_nominal"] - 0.5) < 1e-12
    # the same rate at a higher clock is a smaller fraction per clock
    assert bench.per_clock(full, {"sm_mhz": 2600.0})["frac_of_nominal"] == 0.5
    # no clock record, no figure
    assert bench.per_clock(full, {"sm_mhz": None}) is None and bench.per_clock(full, None) is None
