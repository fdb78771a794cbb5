"""Host-side parts of bench.py, on CPU: the reference arm (which runs the oracle
on the host) prints one JSON line of the contract's shape, stops at its
wall-clock budget and runs on rank 0 only; the DRAM-traffic lookup reports the
committed capture only while the kernel sources hash to the captured version."""
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
    # value = tokens timed / time timed, with --ref-tokens (2) tokens per step
    assert abs(j["value"] - 2 * 1000.0 / j["ms_per_step"]) <= 1e-9 * j["value"]
    cb = j["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == j["value"] and cb["unit"] == "tokens/s" and cb["cores"] >= 1
    assert j["e2e"] == {"value": j["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert j["config"]["workload"] == "tiny_f32" and j["config"]["T"] == 64


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
    good = tmp_path / "good.md"
    good.write_text(f"capture\n    kernel_sources_sha256: {h.hexdigest()}\n    gate_up_dram_bytes_per_launch: 123456\n")
    stale = tmp_path / "stale.md"
    stale.write_text("capture\n    kernel_sources_sha256: " + "0" * 64 + "\n    gate_up_dram_bytes_per_launch: 123456\n")
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(good))
    assert bench.measured_traffic("grok_prefill") == 123456.0
    assert bench.measured_traffic("mid_bf16") is None  # captured on the Grok prefill workload only
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(stale))
    assert bench.measured_traffic("grok_prefill") is None


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
    r = s.stop()
    assert r["samples"] == 3 and r["sm_mhz"] == 1250.0 and r["sm_max_mhz"] == 1965.0
    assert r["reasons"] == ["sw_power_cap"] and r["power_w_max"] == 1001.0
