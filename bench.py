"""Benchmark of the MoE layer forward pass on B200.

One step = one pass of the whole layer (router + top-2, dispatch, gather,
gate/up + SwiGLU, down, combine) over one batch of the workload, through the
C ABI.  Prints one JSON line on rank 0.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

Workload default: the Grok-1-shape prefill layer (T=8192, d=6144, f=32768,
E=8, top-2, no drop).  Under torchrun every rank runs its own batch (distinct
x, same weights): the layer shards by token batch with no collective on the
data path ("weak" scaling); timing is the max over ranks.  On one GPU the line
also carries a per-configuration block (the mid bf16 layer, the skewed Grok
layer, the Grok decode calls and the tiny fp32 layer), each entry timed with
its own clock record.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from synth import configs  # noqa: E402

# the pool's earlier measurement: burst cuBLAS bf16, and the sustained figure with
# the SM clock it settled at under the power cap
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "bf16_tflops_sustained_sm_mhz": 1300.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            d = json.load(fh)
        return d, "measured"
    return PEAKS_FALLBACK, "fallback"


def _num(v):
    try:
        return float(v)
    except (TypeError, ValueError):
        return None


def _sustained_clock_mhz(peaks):
    """SM clock (MHz) at which the sustained tensor peak was measured, when recorded:
    a key of its own, or the median of the clock record taken under load."""
    for key in ("bf16_tflops_sustained_sm_mhz", "bf16_tflops_sustained_clock_mhz"):
        if _num(peaks.get(key)):
            return _num(peaks[key])
    sect = peaks.get("clocks_under_load")
    if _num(sect):
        return _num(sect)
    if isinstance(sect, dict):
        for key in ("sm_mhz_median", "median_sm_mhz", "sm_mhz", "median", "clocks.sm"):
            if _num(sect.get(key)):
                return _num(sect[key])
    return None


def tensor_peak(peaks, src, clk):
    """The dense bf16 tensor peak that matches the clock the run actually had.

    The burst figure (a GEMM timed alone, at full clock) applies when the run's
    median SM clock is within 5% of the maximum.  Below that the run was held
    down by the power cap: the sustained figure is scaled by (the run's median
    SM MHz / the MHz it was measured at), and never taken above the burst
    figure; without a record of that clock the sustained figure is used as it
    is.  Returns (peak TFLOP/s, the rule used)."""
    burst = _num(peaks.get("bf16_tflops")) or PEAKS_FALLBACK["bf16_tflops"]
    sm = _num((clk or {}).get("sm_mhz"))
    smax = _num((clk or {}).get("sm_max_mhz"))
    if sm and smax and sm >= 0.95 * smax:
        return burst, f"{src} bf16_tflops (burst): run median SM clock {sm:.0f} MHz within 5% of max {smax:.0f}"
    sus = _num(peaks.get("bf16_tflops_sustained"))
    at = _sustained_clock_mhz(peaks)
    if sm and sus and at:
        p = min(burst, sus * sm / at)
        return p, (f"{src} bf16_tflops_sustained x run median SM clock {sm:.0f} MHz / {at:.0f} MHz at which it "
                   f"was measured (capped at the burst figure)")
    if sus:
        return sus, f"{src} bf16_tflops_sustained: run SM clock below 95% of max or not recorded"
    return burst, f"{src} bf16_tflops (burst): no clock record"


# DRAM traffic per launch of the roofline kernel, from a committed ncu capture
# (machine-readable; the summary beside it in profiles/ gives the command).
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "dram_traffic.json")
KERNEL_SOURCES = [os.path.join(ROOT, "sparse_moe_layer_07_b200", "csrc", n)
                  for n in ("ffn_tc.cu", "tc_ptx.cuh", "common.cuh", "internal.h")]


def kernel_sources_sha256():
    import hashlib

    h = hashlib.sha256()
    for p in KERNEL_SOURCES:
        with open(p, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def measured_traffic(workload_name, kernel="gate_up"):
    """DRAM read + write bytes per launch of `kernel` on this workload from the
    committed capture, or None when there is none or the kernel sources changed
    since it was taken."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    with open(TRAFFIC_FILE) as fh:
        d = json.load(fh)
    if d.get("kernel_sources_sha256") != kernel_sources_sha256():
        return None
    entry = d.get("workloads", {}).get(workload_name, {}).get(kernel)
    return _num(entry.get("dram_bytes_per_launch")) if isinstance(entry, dict) else None
def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


# ---------------------------------------------------------------------------- multi-rank plumbing
def rank_x(w, rank):
    """The batch of rank `rank`: rank 0 runs the workload's own x; rank r > 0 a distinct
    seeded batch of the same shape (independent token batches, no exchange)."""
    if rank == 0:
        return configs.make_x(w)
    from synth import normal

    return normal(configs.SEED, configs.TID_X + 1000 * rank, (w.T, w.d), dtype=w.storage)


def share_weights(W, world):
    """Rank 0 generated the weights; every other rank receives them once at set-up."""
    import torch.distributed as dist

    if world > 1:
        for k in sorted(W):
            dist.broadcast(W[k], src=0)
    return W


def max_over_ranks(value, device, world):
    """The slowest rank's time (every rank gets the same number)."""
    if world == 1:
        return float(value)
    import torch
    import torch.distributed as dist

    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def throughput(world, tokens_per_rank_step, steps, ms_total):
    """Whole-job tokens/s: the tokens of all ranks over the slowest rank's time."""
    return world * tokens_per_rank_step * steps / (ms_total / 1000.0)


# ---------------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples nvidia-smi clocks/throttle reasons for one GPU while running."""

    FIELDS = ("uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str):
        self.uuid = uuid
        self.rows = []
        self.times = []
        self.proc = None
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) == 8 and (not self.uuid or parts[0] == self.uuid):
                self.rows.append(parts)
                self.times.append(time.monotonic())

    def stop(self, window=None):
        """Stops sampling; `window` = (t0, t1) in time.monotonic() keeps the
        samples taken inside it (the nearest later one when none falls inside)."""
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=5)
        if window is not None and self.rows:
            t0, t1 = window
            keep = [r for r, t in zip(self.rows, self.times) if t0 <= t <= t1 + 0.15]
            if not keep:
                later = [r for r, t in zip(self.rows, self.times) if t >= t0]
                keep = later[:1]
            self.rows = keep
        sm = [float(r[1]) for r in self.rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in self.rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in self.rows for i in range(4) if r[4 + i] == "Active"})
        pw = [float(r[3]) for r in self.rows if r[3].replace(".", "").isdigit()]
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(self.rows), "power_w_max": max(pw) if pw else None}


# ---------------------------------------------------------------------------- CPU baseline (oracle)
def blas_threads():
    try:
        from threadpoolctl import threadpool_info

        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def oracle_layer_time(w, host, x, n_sample, seed, threads=None):
    """The oracle's time for the whole layer, by the recipe of the measurement plan:
    router, top-2 and dispatch timed over all T tokens; the expert FFN and the
    combine timed on a seeded sample of tokens and extrapolated per kept
    assignment (x N_kept / kept assignments in the sample).  `threads` limits
    the BLAS threads (None: the library's default, all cores)."""
    import contextlib

    import oracle

    limit = contextlib.nullcontext()
    if threads is not None:
        from threadpoolctl import threadpool_limits

        limit = threadpool_limits(limits=threads, user_api="blas")
    rng = np.random.default_rng(seed)
    tok = np.sort(rng.choice(w.T, size=min(n_sample, w.T), replace=False))
    bias = configs.make_bias(w)
    with limit:
        used = blas_threads()
        t0 = time.perf_counter()
        lg = oracle.router_logits(x, host["wr"], bias)
        idx, wt = oracle.top2_softmax(lg)
        disp = oracle.dispatch(idx, wt, w.E, oracle.capacity(w.T, w.top_k, w.E, w.capacity_factor))
        t_route = time.perf_counter() - t0
        t0 = time.perf_counter()
        oracle.layer_forward(x, host["wr"], host["wg"], host["wu"], host["wd"], w.capacity_factor, logit_bias=bias,
                             tokens=tok)
        t_sample = time.perf_counter() - t0
    # layer_forward routes all T again before the sampled FFN: that share is t_route
    t_ffn = max(t_sample - t_route, 0.0)
    kept_sample = int((disp["slot_of"][tok] >= 0).sum())
    n_kept = int(disp["n_kept"])
    scale = n_kept / kept_sample if kept_sample else 0.0
    t_layer = t_route + t_ffn * scale
    return {"layer_s": t_layer, "tokens_per_s": w.T / t_layer, "route_s": t_route, "ffn_sample_s": t_ffn,
            "sample_tokens": int(tok.size), "kept_in_sample": kept_sample, "n_kept": n_kept,
            "extrapolation": scale, "threads": used}


def cpu_baseline(w, host, x, n_sample):
    """The oracle on this host's cores, single-threaded and on all cores."""
    one = oracle_layer_time(w, host, x, n_sample, 7, threads=1)
    allc = oracle_layer_time(w, host, x, n_sample, 7)
    return {"value": allc["tokens_per_s"], "unit": "tokens/s", "cores": allc["threads"], "kind": "oracle",
            "nproc": host_cores(),
            "sample": (f"oracle (fp64 numpy): router, top-2 and dispatch over all T={w.T} tokens "
                       f"({allc['route_s']:.2f} s); expert FFN and combine on {allc['sample_tokens']} seeded tokens "
                       f"({allc['kept_in_sample']} kept assignments, {allc['ffn_sample_s']:.2f} s) extrapolated "
                       f"x{allc['extrapolation']:.1f} to the {allc['n_kept']} kept assignments of the layer"),
            "layer_s": allc["layer_s"],
            "single_thread": {"value": one["tokens_per_s"], "cores": one["threads"], "layer_s": one["layer_s"],
                              "route_s": one["route_s"], "ffn_sample_s": one["ffn_sample_s"]}}


def reference_arm(args, w):
    ws, rank, _ = dist_env()
    if rank != 0:
        return
    host = dict(wr=configs.make_router(w), wg=configs.make_w_gate(w), wu=configs.make_w_up(w),
                wd=configs.make_w_down(w))
    x = configs.make_x(w)
    n = args.ref_tokens
    # Each step is one oracle measurement of the whole layer (routing over all T,
    # the FFN on an n-token sample extrapolated per kept assignment); steps stop
    # once the next one would pass the wall-clock budget, so a long --steps
    # still ends within a few minutes.  Warm-up steps stop at a third of it.
    t_w, warm = 0.0, 0
    for i in range(args.warmup):
        if warm and t_w + t_w / warm > args.ref_budget_s / 3:
            break
        t0 = time.perf_counter()
        oracle_layer_time(w, host, x, n, 1000 + i)
        t_w += time.perf_counter() - t0
        warm += 1
    layer_s, wall, done, r = [], 0.0, 0, None
    for i in range(args.steps):
        if done and wall + wall / done > args.ref_budget_s:
            break
        t0 = time.perf_counter()
        r = oracle_layer_time(w, host, x, n, i)
        wall += time.perf_counter() - t0
        layer_s.append(r["layer_s"])
        done += 1
    ms = 1000.0 * statistics.fmean(layer_s)
    value = w.T / (ms / 1000.0)
    sample = (f"oracle (fp64 numpy) per step: router, top-2 and dispatch over all T={w.T} tokens, expert FFN and "
              f"combine on {n} seeded tokens extrapolated per kept assignment to the whole layer; {done} of "
              f"{args.steps} requested steps timed (wall-clock budget {args.ref_budget_s:.0f} s), {warm} warm-up")
    line = {"impl": "reference", "metric": "MoE-layer tokens/s", "value": value, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": done, "steps_requested": args.steps, "warmup": warm,
            "warmup_requested": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(w),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": r["threads"], "nproc": host_cores(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def hbm_steps(w, n_kept, per_kernel, fused, peaks):
    """Achieved bandwidth of the memory-bound steps from their algorithmic bytes:
    router T*d*b + E*d*b + 16*T; dispatch (3 kernels) + gather 8*T + 12*N + 2*N*d*b;
    combine 4*N*d + 8*T + T*d*b (in the fused path the combine is inside the down pass)."""
    b = 2 if w.storage == "bf16" else 4
    hbm = peaks.get("hbm_gbs", 6650.0)
    out = {}
    items = {"router": w.T * w.d * b + w.E * w.d * b + 16 * w.T,
             "dispatch": 8 * w.T + 12 * n_kept + 2 * n_kept * w.d * b}
    if not fused:
        items["combine"] = 4 * n_kept * w.d + 8 * w.T + w.T * w.d * b
    for name, nbytes in items.items():
        ms = per_kernel.get(name, 0.0)
        if ms > 0:
            gbs = nbytes / (ms / 1000.0) / 1e9
            out[name] = {"bytes": nbytes, "ms": ms, "gbs": gbs, "frac_hbm": gbs / hbm}
    return out


def workload_config(w):
    return {"workload": w.name, "T": w.T, "d": w.d, "f": w.f, "E": w.E, "top_k": w.top_k,
            "capacity_factor": w.capacity_factor, "logit_bias": list(w.logit_bias) if w.logit_bias else None,
            "l2": "inputs larger than L2 (expert weights %.2f GB per step)" % (3 * w.E * w.d * w.f * 2 / 1e9),
            "description": w.description}


# ---------------------------------------------------------------------------- our arm
class LayerRun:
    """Device buffers of one workload and one step of the layer through the
    separate entry points (router -> dispatch -> gate/up -> down + combine),
    with CUDA events between the calls."""

    NAMES = ["router", "dispatch", "gate_up", "down", "combine"]

    def __init__(self, moe, w, W, x, bias_d, dev, stream, int8=False, unfused=False):
        import torch

        self.moe, self.w, self.W, self.x, self.bias_d, self.dev, self.stream = moe, w, W, x, bias_d, dev, stream
        self.cfg = cfg = moe.Config(w.T, w.d, w.f, capacity_factor=w.capacity_factor, dtype=w.storage)
        rows = w.T * w.top_k
        tdt = cfg.torch_dtype
        self.buf = {
            "idx": torch.empty((w.T, 2), dtype=torch.int32, device=dev),
            "w": torch.empty((w.T, 2), dtype=torch.float32, device=dev),
            "h": torch.empty((rows, w.f), dtype=tdt, device=dev),
            "out": torch.empty((w.T, w.d), dtype=tdt, device=dev),
            "ws": torch.empty((max(moe.dispatch_workspace_size(cfg), 16),), dtype=torch.uint8, device=dev),
        }
        self.disp = {"counts_raw": torch.empty(8, dtype=torch.int32, device=dev),
                     "counts_kept": torch.empty(8, dtype=torch.int32, device=dev),
                     "offsets": torch.empty(9, dtype=torch.int32, device=dev),
                     "perm": torch.empty(rows, dtype=torch.int32, device=dev),
                     "slot_of": torch.empty((w.T, 2), dtype=torch.int32, device=dev),
                     "row_scale": torch.empty(rows, dtype=torch.float32, device=dev),
                     "x_perm": torch.empty((rows, w.d), dtype=tdt, device=dev)}
        self.qw = moe.QuantizedExperts(cfg, W["wg"], W["wu"], W["wd"]) if int8 else None
        self.ws8 = (torch.empty((max(moe.lib.moe_expert_ffn_w8_workspace_size(cfg.ref), 16),), dtype=torch.uint8,
                                device=dev) if int8 else None)
        # bf16 tensor-core batches sum the down outputs into token order (zero + down
        # + rounding pass, no y buffer, no separate combine)
        self.fused = (not int8 and not unfused and w.storage == "bf16" and w.T * 2 > 64 * w.E and w.d % 256 == 0)
        if self.fused:
            self.buf["dc_ws"] = torch.empty(moe.lib.moe_expert_down_combine_workspace_size(cfg.ref),
                                            dtype=torch.uint8, device=dev)
        else:
            self.buf["y"] = torch.empty((rows, w.d), dtype=torch.float32, device=dev)
        # router 1, dispatch 3 + gather 1, gate/up 1, down 1, combine 1 (int8 experts: + 2 row-code
        # passes and the partial sum); fused: router 1, dispatch 3 + gather 1, gate/up 1, zero + down +
        # rounding 3
        self.launches_per_step = 11 if int8 else (9 if self.fused else 8)

    def step(self, ev=None):
        moe, cfg, W, buf, disp, s = self.moe, self.cfg, self.W, self.buf, self.disp, self.stream

        def mark(i):
            if ev:
                ev[i].record(s)

        mark(0)
        moe.router_topk(cfg, self.x, W["wr"], self.bias_d, topk_idx=buf["idx"], topk_w=buf["w"])
        mark(1)
        moe.dispatch(cfg, self.x, buf["idx"], buf["w"], out=disp, ws=buf["ws"])
        mark(2)
        if self.qw is not None:
            # int8 experts: gate/up and down in one call (both timed under "gate_up")
            moe.expert_ffn_w8(cfg, disp["x_perm"], disp["offsets"], self.qw, disp["row_scale"], y=buf["y"],
                              ws=self.ws8)
        else:
            moe.expert_gate_up(cfg, disp["x_perm"], disp["offsets"], W["wg"], W["wu"], h=buf["h"])
        mark(3)
        if self.fused:
            moe.expert_down_combine(cfg, buf["h"], disp["offsets"], W["wd"], disp["row_scale"], disp["perm"],
                                    out=buf["out"], ws=buf["dc_ws"])
            mark(4)
            mark(5)
            return
        if self.qw is None:
            moe.expert_down(cfg, buf["h"], disp["offsets"], W["wd"], disp["row_scale"], y=buf["y"])
        mark(4)
        moe.combine(cfg, buf["y"], disp["slot_of"], buf["w"], weights_applied=True, out=buf["out"])
        mark(5)

    def graph_replay(self, steps):
        """The same step (separate entry points, no events) captured once in a
        CUDA graph and replayed `steps` times: ms per step without host launch
        overhead."""
        import torch

        cap = torch.cuda.Stream(self.dev)
        cap.wait_stream(torch.cuda.current_stream(self.dev))
        with torch.cuda.stream(cap):
            for _ in range(3):
                self.step()
        torch.cuda.synchronize(self.dev)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cap, capture_error_mode="relaxed"):
            self.step()
        torch.cuda.synchronize(self.dev)
        for _ in range(3):
            g.replay()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(self.dev)
        a.record(self.stream)
        for _ in range(steps):
            g.replay()
        b.record(self.stream)
        torch.cuda.synchronize(self.dev)
        ms = a.elapsed_time(b) / steps
        del g
        return ms

    def router_alone(self, reps=30):
        """The router kernel timed on its own, each launch after a plain read of a
        256 MB buffer has replaced L2's contents with clean lines (in the step the
        router starts with the previous step's output dirty in L2, whose
        write-back shares the HBM bandwidth).  Median ms over `reps` launches."""
        import torch

        scratch = torch.ones(256 << 20, dtype=torch.uint8, device=self.dev)
        times = []
        for _ in range(reps + 3):
            scratch.max()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(self.stream)
            self.moe.router_topk(self.cfg, self.x, self.W["wr"], self.bias_d, topk_idx=self.buf["idx"],
                                 topk_w=self.buf["w"])
            e1.record(self.stream)
            times.append((e0, e1))
        torch.cuda.synchronize(self.dev)
        del scratch
        return float(sorted(a.elapsed_time(b) for a, b in times[3:])[reps // 2])

    def time(self, steps, warmup, world=1):
        """W untimed steps, then K steps between a barrier + synchronize on both
        sides, clocks sampled during the timed region; the max over ranks.
        Per-kernel times come from up to 100 further steps with CUDA events
        between the calls (kept out of the timed steps, where they would
        serialise the launches)."""
        import torch
        import torch.distributed as dist

        dev, stream = self.dev, self.stream
        for _ in range(warmup):
            self.step()
        torch.cuda.synchronize(dev)
        n_kept = int(self.disp["offsets"][-1].item())
        counts_kept = self.disp["counts_kept"].cpu().tolist()
        counts_raw = self.disp["counts_raw"].cpu().tolist()
        uuid = ""
        try:
            uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
        except Exception:
            pass
        clocks = ClockSampler(uuid)
        clocks.start()
        time.sleep(0.5)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        t_start = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        w0 = time.monotonic()
        # no events between the calls inside the timed steps: an event between two
        # launches would stop the next kernel's launch from overlapping the
        # previous kernel's exit (programmatic dependent launch)
        t_start.record(stream)
        for i in range(steps):
            self.step()
        t_end.record(stream)
        torch.cuda.synchronize(dev)
        w1 = time.monotonic()
        # a pipeline wait that ran out of time sets the device error word: such a run is invalid
        device_error = self.moe.get_device_error()
        if world > 1:
            dist.barrier()
        clk = clocks.stop(window=(w0, w1))
        ms_total = max_over_ranks(t_start.elapsed_time(t_end), dev, world)
        # per-kernel times on separate steps, with events between the calls
        n_k = min(steps, 100)
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(n_k)]
        for i in range(n_k):
            self.step(evs[i])
        torch.cuda.synchronize(dev)
        per_kernel = {n: 0.0 for n in self.NAMES}
        for e in evs:
            for j, n in enumerate(self.NAMES):
                per_kernel[n] += e[j].elapsed_time(e[j + 1])
        per_kernel = {n: v / n_k for n, v in per_kernel.items()}
        return {"ms_total": ms_total, "ms_step": ms_total / steps, "per_kernel": per_kernel, "n_kept": n_kept,
                "counts_kept": counts_kept, "counts_raw": counts_raw, "device_error": device_error, "clocks": clk}


def gemm_roofline(w, res, peaks, src):
    """Achieved TFLOP/s of the gate/up and down kernels against the clock-matched tensor peak."""
    n = res["n_kept"]
    pk = res["per_kernel"]
    peak, rule = tensor_peak(peaks, src, res["clocks"])
    gu = 4.0 * n * w.d * w.f / (pk["gate_up"] / 1000.0) / 1e12 if pk["gate_up"] > 0 else 0.0
    dn = 2.0 * n * w.d * w.f / (pk["down"] / 1000.0) / 1e12 if pk["down"] > 0 else 0.0
    return peak, rule, gu, dn


def per_clock(tflops, clocks):
    """The kernel's rate per SM clock against the nominal dense bf16 rate of a
    B200 SM (one 128 x 256 x 16 MMA per 128 clocks = 8192 FLOP per clock), at
    the run's median SM clock.  That median covers the whole step, short kernels
    included, so it is an upper bound on the GEMM's clock and the fraction a
    lower bound."""
    mhz = (clocks or {}).get("sm_mhz")
    if not mhz or not tflops:
        return None
    fpc = tflops * 1e12 / (148 * mhz * 1e6)
    return {"flop_per_clock_per_sm": fpc, "frac_of_nominal": fpc / 8192.0, "sm_mhz": mhz}


def layer_summary(w, res, peaks, src, world, steps):
    """tokens/s, TFLOP/s, GEMM roofline fractions, drops and balance of one timed workload."""
    n = res["n_kept"]
    ms = res["ms_total"]
    flops_step = 2.0 * w.T * w.d * w.E + 6.0 * n * w.d * w.f
    peak, rule, gu, dn = gemm_roofline(w, res, peaks, src)
    ck = res["counts_kept"]
    tf = world * flops_step * steps / (ms / 1000.0) / 1e12
    return {"workload": w.name, "T": w.T, "d": w.d, "f": w.f, "capacity_factor": w.capacity_factor,
            "dtype": "bf16" if w.storage == "bf16" else "f32",
            "tokens_per_s": throughput(world, w.T, steps, ms), "ms_per_step": res["ms_step"], "steps": steps,
            "tflops": tf, "tensor_frac_layer": tf / peak,
            "gate_up": {"tflops": gu, "frac": gu / peak}, "down": {"tflops": dn, "frac": dn / peak},
            "peak_tflops": peak, "peak_rule": rule, "kernels_ms": res["per_kernel"],
            "n_kept": n, "dropped": w.top_k * w.T - n, "counts_raw": res["counts_raw"], "counts_kept": ck,
            "expert0_share_raw": res["counts_raw"][0] / max(sum(res["counts_raw"]), 1),
            "imbalance_max_over_mean_kept": max(ck) / (sum(ck) / len(ck)) if sum(ck) else None,
            "device_error": res["device_error"], "clocks": res["clocks"]}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="grok_prefill", choices=sorted(configs.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--ref-tokens", type=int, default=64, help="sampled tokens per reference-arm step")
    ap.add_argument("--ref-budget-s", type=float, default=150.0, help="wall-clock budget of the reference arm's steps")
    ap.add_argument("--cpu-tokens", type=int, default=64, help="tokens in the CPU-baseline sample")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-configs", action="store_true", help="skip the per-configuration block")
    ap.add_argument("--shape", default=None, help="T,d,f override of the workload (profiling cases)")
    ap.add_argument("--int8", action="store_true", help="int8 expert weights (weight-only, per-channel scales)")
    ap.add_argument("--no-train", action="store_true", help="skip the training pair (forward + backward)")
    ap.add_argument("--train-steps", type=int, default=20)
    ap.add_argument("--tiles", default="auto", choices=["auto", "single", "pair"],
                    help="tile shape of the bf16 grouped GEMMs")
    ap.add_argument("--unfused", action="store_true",
                    help="separate down and combine kernels instead of the fused down-combine")
    ap.add_argument("--ep-only", action="store_true",
                    help="only the expert-parallel measurement (8 ranks on this GPU), e.g. for profiling its kernels")
    args = ap.parse_args()
    w = configs.WORKLOADS[args.workload]
    if args.shape:
        T, d, f = (int(v) for v in args.shape.split(","))
        w = configs.scaled(w, name=f"{w.name}_T{T}_d{d}_f{f}", T=T, d=d, f=f)
    if args.impl == "reference":
        return reference_arm(args, w)

    import torch
    import torch.distributed as dist

    import sparse_moe_layer_07_b200 as moe

    moe.set_gemm_tiles(args.tiles)
    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta

        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=dev)

    # ---- inputs: weights generated once (rank 0) and broadcast; x distinct per rank
    host = None
    if rank == 0:
        host = dict(wr=configs.make_router(w), wg=configs.make_w_gate(w), wu=configs.make_w_up(w),
                    wd=configs.make_w_down(w))
        W = {k: to_dev(v, dev) for k, v in host.items()}
    else:
        tdt = torch.bfloat16 if w.storage == "bf16" else torch.float32
        W = {"wr": torch.empty((w.E, w.d), dtype=tdt, device=dev),
             "wg": torch.empty((w.E, w.d, w.f), dtype=tdt, device=dev),
             "wu": torch.empty((w.E, w.d, w.f), dtype=tdt, device=dev),
             "wd": torch.empty((w.E, w.f, w.d), dtype=tdt, device=dev)}
    share_weights(W, world)
    x_np = rank_x(w, rank)
    x = to_dev(x_np, dev)
    bias = configs.make_bias(w)
    bias_d = None if bias is None else to_dev(bias, dev)
    stream = torch.cuda.current_stream(dev)
    if args.ep_only:
        if world > 1 or w.storage != "bf16" or w.T % 8 or w.d % 256:
            raise SystemExit("--ep-only: one GPU, a bf16 workload, T a multiple of 8 and d of 256")
        peaks, peak_src = load_peaks()
        print(json.dumps({"workload": w.name, "ep_peers": ep_peers_bench(moe, w, W, x, bias_d, dev, stream, peaks,
                                                                          peak_src)}), flush=True)
        return
    run = LayerRun(moe, w, W, x, bias_d, dev, stream, int8=args.int8, unfused=args.unfused)
    cfg, tdt = run.cfg, run.cfg.torch_dtype
    res = run.time(args.steps, args.warmup, world)
    peaks, peak_src = load_peaks()
    summ = layer_summary(w, res, peaks, peak_src, world, args.steps)
    n_kept, per_kernel = res["n_kept"], res["per_kernel"]
    gu_flops = 4.0 * n_kept * w.d * w.f
    roofline = {"bound": "tensor", "kernel": "grouped_gemm_tc_kernel<gate_up> (SwiGLU epilogue)",
                "achieved": summ["gate_up"]["tflops"], "peak": summ["peak_tflops"], "unit": "TFLOP/s",
                "frac": summ["gate_up"]["frac"], "peak_source": summ["peak_rule"],
                "traffic": measured_traffic(w.name, "gate_up"),
                "traffic_unit": "bytes per launch (dram read + write, ncu)",
                "per_clock": per_clock(summ["gate_up"]["tflops"], res["clocks"]),
                "algorithmic": f"4*d*f*N_kept = {gu_flops:.4e} FLOP per launch (N_kept={n_kept})",
                "down": dict(summ["down"], kernel="grouped_gemm_tc_kernel<down> (routing-weight scatter epilogue)",
                             traffic=measured_traffic(w.name, "down"))}
    line = {"metric": "MoE-layer tokens/s", "value": summ["tokens_per_s"], "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": res["ms_step"], "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if w.storage == "bf16" else "f32",
            "data": "synthetic (seeded Philox4x32-10 normal inputs, random-init weights)",
            "config": dict(workload_config(w), expert_weights="int8" if args.int8 else w.storage),
            "tflops": summ["tflops"], "tensor_frac_layer": summ["tensor_frac_layer"],
            "kernels_ms": per_kernel, "hbm_steps": hbm_steps(w, n_kept, per_kernel, run.fused, peaks),
            "gemm_tiles": args.tiles, "device_error": res["device_error"],
            "path": ("down-combine fused: down sums into token order (its time includes the zeroing and "
                     "rounding passes; combine 0)") if run.fused else "separate down and combine",
            "counts_kept": res["counts_kept"], "n_kept": n_kept, "dropped": summ["dropped"],
            "imbalance_max_over_mean_kept": summ["imbalance_max_over_mean_kept"],
            "expert_utilization": [c * w.E / max(sum(res["counts_kept"]), 1) for c in res["counts_kept"]],
            "gpu_launches": run.launches_per_step * args.steps, "roofline": roofline, "clocks": res["clocks"]}
    rt = line["hbm_steps"].get("router")
    if rt:
        ms_alone = run.router_alone()
        gbs = rt["bytes"] / (ms_alone / 1000.0) / 1e9
        rt["alone"] = {"ms": ms_alone, "gbs": gbs, "frac_hbm": gbs / peaks.get("hbm_gbs", 6650.0),
                       "note": "the same kernel launched on its own after a 256 MB read has left only clean lines "
                               "in L2 (median of 30); in the step it starts with the previous step's output "
                               "dirty in L2"}
    del run

    if not args.no_e2e:
        line["e2e"] = e2e_bench(moe, w, cfg, W, x_np, bias_d, dev, stream, args, world)
    if not args.no_decode and w.name == "grok_prefill" and not args.shape:
        line["decode"] = decode_bench(moe, W, dev, stream, peaks, peak_src, world)
    if (not args.no_train and w.name.startswith("grok_prefill") and w.storage == "bf16" and w.d % 256 == 0
            and w.f % 256 == 0):
        line["train"] = train_bench(moe, cfg, W, x, bias_d, n_kept, dev, stream, peaks, peak_src, world,
                                    args.train_steps)
    if world == 1 and not args.no_configs and w.name == "grok_prefill" and not args.shape and not args.int8:
        line["per_config"] = per_config(moe, W, dev, stream, peaks, peak_src, summ, line.get("decode"))
    if world == 1 and not args.no_configs and w.name == "grok_prefill" and not args.shape and not args.int8:
        line["ep_peers"] = ep_peers_bench(moe, w, W, x, bias_d, dev, stream, peaks, peak_src)
    if rank == 0 and world == 1 and not args.no_cpu and host is not None:
        line["cpu_baseline"] = cpu_baseline(w, host, x_np, args.cpu_tokens)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def to_dev(a, dev):
    import torch

    t = torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    return t.view(torch.bfloat16) if a.dtype == np.uint16 else t


def _sampler(dev):
    import torch

    uuid = ""
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    s = ClockSampler(uuid)
    s.start()
    time.sleep(0.3)
    return s


def e2e_bench(moe, w, cfg, W, x_np, bias_d, dev, stream, args, world):
    """End to end: host x in, host out, through the C entry points with host buffers.
    Headline: moe_layer_forward_host_batches, one batch per step, every step's x copied
    in and its out copied back inside the timed region (overlapped with the compute of
    the neighbouring steps).  Also reported: the one-batch call, which waits per batch."""
    import torch
    import torch.distributed as dist

    tdt = cfg.torch_dtype
    ws_full = torch.empty(moe.workspace_size_host_batches(cfg), dtype=torch.uint8, device=dev)
    x_host = torch.from_numpy(np.ascontiguousarray(x_np))
    x_host = (x_host.view(torch.bfloat16) if w.storage == "bf16" else x_host).pin_memory()
    out_ring = [torch.empty((w.T, w.d), dtype=tdt).pin_memory() for _ in range(2)]

    def run_batches(n):
        moe.layer_forward_host_batches(cfg, [x_host] * n, W["wr"], W["wg"], W["wu"], W["wd"],
                                       [out_ring[i % 2] for i in range(n)], ws_full, logit_bias=bias_d,
                                       stream=stream)

    run_batches(args.warmup)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    run_batches(args.steps)
    b.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(a.elapsed_time(b), dev, world)
    nbytes = w.T * w.d * (2 if w.storage == "bf16" else 4)
    tokens = world * w.T * args.steps
    # the one-batch entry point (copy in, layer, copy out, wait) for comparison
    single_steps = min(args.steps, 10)
    moe.layer_forward_host(cfg, x_host, W["wr"], W["wg"], W["wu"], W["wd"], out_ring[0], ws_full,
                           logit_bias=bias_d, stream=stream)
    if world > 1:
        dist.barrier()
    a.record(stream)
    for _ in range(single_steps):
        moe.layer_forward_host(cfg, x_host, W["wr"], W["wg"], W["wu"], W["wd"], out_ring[0], ws_full,
                               logit_bias=bias_d, stream=stream)
    b.record(stream)
    torch.cuda.synchronize(dev)
    single_ms = max_over_ranks(a.elapsed_time(b), dev, world) / single_steps
    del ws_full
    return {"value": tokens / (e2e_ms / 1000.0), "unit": "tokens/s", "h2d_bytes_per_step": nbytes,
            "d2h_bytes_per_step": nbytes, "ms_per_step": e2e_ms / args.steps,
            "api": "moe_layer_forward_host_batches (pinned host x/out, one batch per step, copies "
                   "overlapped with the neighbouring steps' compute; device-resident weights)",
            "one_batch_call": {"ms_per_step": single_ms, "value": tokens / args.steps / (single_ms / 1000.0),
                               "api": "moe_layer_forward_host (copy in, layer, copy out, wait)"}}


def per_config(moe, W_grok, dev, stream, peaks, peak_src, grok_summary, decode):
    """Every configuration of the workload list, each timed with its own clock
    record: the mid bf16 layer and the tiny fp32 layer on their own weights, the
    skewed Grok layer on the (identical) Grok weights already resident, the Grok
    prefill headline and the Grok decode calls as measured above."""
    out = {"grok_prefill": {k: grok_summary[k] for k in ("tokens_per_s", "ms_per_step", "tflops", "gate_up",
                                                          "down", "n_kept", "dropped", "expert0_share_raw",
                                                          "imbalance_max_over_mean_kept", "peak_rule")}}
    out["grok_prefill"]["note"] = "the headline workload (value, roofline and clocks of this line)"
    plan = (("mid_bf16", None, 3000, 20), ("grok_skew", W_grok, 30, 3), ("tiny_f32", None, 2000, 20))
    for name, W, steps, warm in plan:
        w = configs.WORKLOADS[name]
        if W is None:
            W = {"wr": to_dev(configs.make_router(w), dev), "wg": to_dev(configs.make_w_gate(w), dev),
                 "wu": to_dev(configs.make_w_up(w), dev), "wd": to_dev(configs.make_w_down(w), dev)}
        bias = configs.make_bias(w)
        run = LayerRun(moe, w, W, to_dev(configs.make_x(w), dev), None if bias is None else to_dev(bias, dev), dev,
                       stream)
        s = layer_summary(w, run.time(steps, warm), peaks, peak_src, 1, steps)
        s["gpu_launches"] = run.launches_per_step * steps
        if name == "mid_bf16":
            ms_g = run.graph_replay(steps)
            s["graph"] = {"ms_per_step": ms_g, "tokens_per_s": w.T * 1000.0 / ms_g,
                          "note": "the same calls captured once in a CUDA graph and replayed (no host launch cost)"}
        if name == "tiny_f32":
            s["note"] = ("parity case: fp32 experts on the CUDA cores (exact FFMA, no tensor cores), so the "
                         "bf16 tensor fractions do not apply")
            for k in ("tensor_frac_layer", "gate_up", "down", "peak_tflops", "peak_rule"):
                s.pop(k, None)
        out[name] = s
        del run
    if decode:
        out["grok_decode"] = {k: decode[k] for k in ("ms_per_call", "tokens_per_s", "achieved_gbs", "frac",
                                                     "peak_gbs", "bound", "clocks") if k in decode}
        out["grok_decode"]["int8_weights"] = {k: decode["int8_weights"][k]
                                              for k in ("ms_per_call", "tokens_per_s", "achieved_gbs", "frac")}
    return out


def ep_peers_bench(moe, w, W, x, bias_d, dev, stream, peaks, peak_src, world=8, steps=100, warmup=3,
                   phase_steps=10):
    """Expert parallelism over peer memory with its `world` ranks held by this
    process on this GPU: the headline batch split into `world` rank batches of
    T / world tokens, rank q owning experts [q E / world, (q + 1) E / world).
    A step runs every rank's routing and dispatch, then every rank's experts,
    then every rank's rounding on one stream (the stream order stands in for
    the barriers), so it is the work all `world` GPUs of a real run share,
    without the NVLink transfers.  The outputs, put back in token order, must
    equal the single-device layer's on the whole batch bit for bit (no token
    is dropped at this capacity factor on either side).  `steps` matches the
    headline's timed steps so that both run under the same power-capped clock."""
    import torch

    from sparse_moe_layer_07_b200.expert_parallel import EpPeerBuffers, ep_route

    Tr = w.T // world
    cfg = moe.Config(Tr, w.d, w.f, capacity_factor=w.capacity_factor, dtype="bf16")
    xs = [x[r * Tr:(r + 1) * Tr] for r in range(world)]
    bufs = [EpPeerBuffers(cfg, world, dev) for _ in range(world)]
    addrs = [b.addrs() for b in bufs]
    peers = [moe.EpPeers(world, r, addrs) for r in range(world)]
    outs = [torch.empty((Tr, w.d), dtype=torch.bfloat16, device=dev) for _ in range(world)]

    def dispatch_all(disps, table):
        for r in range(world):
            moe.ep_dispatch_peers(cfg, peers[r], table, xs[r], disps[r], bufs[r].grp_offsets)

    def step(ev=None):
        def mark(i):
            if ev:
                ev[i].record(stream)

        mark(0)
        disps = [ep_route(cfg, xs[r], W["wr"], bias_d) for r in range(world)]
        table = torch.stack([d["counts_kept"] for d in disps])
        mark(1)
        dispatch_all(disps, table)
        mark(2)
        for r in range(world):
            moe.ep_expert_ffn_peers(cfg, peers[r], bufs[r].grp_offsets, W["wg"], W["wu"], W["wd"], bufs[r].h)
        mark(3)
        for r in range(world):
            moe.ep_combine_peers(cfg, peers[r], outs[r])
        mark(4)
        return disps, table

    with torch.cuda.stream(stream):
        for _ in range(warmup):
            step()
        torch.cuda.synchronize(dev)
        clocks = _sampler(dev)
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        w0 = time.monotonic()
        t0.record(stream)
        for _ in range(steps):
            step()
        t1.record(stream)
        torch.cuda.synchronize(dev)
        clk = clocks.stop(window=(w0, time.monotonic()))
        ms = t0.elapsed_time(t1) / steps
        # phases on further steps, with events between them
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(phase_steps)]
        phase = [0.0] * 4
        for i in range(phase_steps):
            disps, table = step(evs[i])
            torch.cuda.synchronize(dev)
            for j in range(4):
                phase[j] += evs[i][j].elapsed_time(evs[i][j + 1]) / phase_steps
        n_kept = sum(int(d["offsets"][-1].item()) for d in disps)
        recv = [int(b.grp_offsets[-1].item()) for b in bufs]
        single = moe.layer_forward(moe.Config(w.T, w.d, w.f, capacity_factor=w.capacity_factor, dtype="bf16"), x,
                                   W["wr"], W["wg"], W["wu"], W["wd"], logit_bias=bias_d)
        same = bool(torch.equal(torch.cat(outs).view(torch.int16), single.view(torch.int16)))
        # the dispatch kernels as the GPU runs them: called one by one, each call
        # spends more time on the host than its kernel on the GPU, so the calls are
        # captured once in a CUDA graph and replayed back to back (they rewrite the
        # same rows each time)
        g = torch.cuda.CUDAGraph()
        cap = torch.cuda.Stream(dev)
        cap.wait_stream(stream)
        torch.cuda.synchronize(dev)
        with torch.cuda.graph(g, stream=cap, capture_error_mode="relaxed"):
            dispatch_all(disps, table)
        torch.cuda.synchronize(dev)
        stream.wait_stream(cap)
        for _ in range(3):
            g.replay()
        reps = 20
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record(stream)
        for _ in range(reps):
            g.replay()
        g1.record(stream)
        torch.cuda.synchronize(dev)
        disp_ms = g0.elapsed_time(g1) / reps
        del g
    device_error = moe.get_device_error()
    # the dispatch calls: zero the rank's fp32 sums, read each kept row and store
    # it with its 8 bytes of source id and weight (and read perm, row_scale)
    dbytes = world * Tr * w.d * 4 + n_kept * (2 * w.d * 2 + 16)
    dgbs = dbytes / (disp_ms / 1000.0) / 1e9
    flops = 6.0 * n_kept * w.d * w.f
    peak, rule = tensor_peak(peaks, peak_src, clk)
    ex_tf = flops / (phase[2] / 1000.0) / 1e12
    del bufs, outs
    return {"world": world, "tokens_per_rank": Tr, "steps": steps, "ms_per_step": ms,
            "tokens_per_s": w.T * 1000.0 / ms,
            "ms_phases": {"route": phase[0], "dispatch": phase[1], "experts": phase[2], "combine": phase[3]},
            "dispatch": {"ms": disp_ms, "ms_per_rank": disp_ms / world, "bytes": dbytes, "gbs": dgbs,
                         "frac_hbm": dgbs / peaks.get("hbm_gbs", 6650.0),
                         "timing": "the 8 calls (one kernel each) replayed as a CUDA graph, 20 replays"},
            "experts": {"tflops": ex_tf, "frac": ex_tf / peak, "peak_tflops": peak, "peak_rule": rule},
            "rows_received": recv, "n_kept": n_kept, "equals_single_device": same, "device_error": device_error,
            "gpu_launches_per_step": world * 8, "clocks": clk,
            "phases_timing": f"events between the phases of {phase_steps} further steps (the short phases "
                             "include host launch time)",
            "note": "all ranks on one GPU, one after another: a step is the whole job's work without NVLink; "
                    "the dispatch stores go to this GPU's own memory here (HBM-bound), to peers' over NVLink "
                    "in a real run"}


def train_bench(moe, cfg, W, x, bias_d, n_kept, dev, stream, peaks, peak_src, world, steps):
    """Forward-for-training + backward of the layer; backward FLOPs = 12*d*f per kept row
    (dH, dX over gate and up, and the three weight gradients) + 4*T*d*E for the router.
    Per-kernel times come from the library's phase events (moe_profile_phases)."""
    import torch

    from synth import normal

    ws = torch.empty(moe.workspace_size_train(cfg), dtype=torch.uint8, device=dev)
    out = torch.empty((cfg.T, cfg.d), dtype=torch.bfloat16, device=dev)
    dout = torch.from_numpy(normal(configs.SEED, 907, (cfg.T, cfg.d), dtype="bf16")).view(torch.bfloat16).to(dev)
    E, d, f = cfg.E, cfg.d, cfg.f
    grads = {"dx": torch.empty((cfg.T, d), dtype=torch.bfloat16, device=dev),
             "dw_router": torch.empty((E, d), dtype=torch.float32, device=dev),
             "dbias": torch.empty((E,), dtype=torch.float32, device=dev),
             "dw_gate": torch.empty((E, d, f), dtype=torch.float32, device=dev),
             "dw_up": torch.empty((E, d, f), dtype=torch.float32, device=dev),
             "dw_down": torch.empty((E, f, d), dtype=torch.float32, device=dev)}

    def step(ev=None):
        if ev:
            ev[0].record(stream)
        moe.layer_forward_train(cfg, x, W["wr"], W["wg"], W["wu"], W["wd"], ws, logit_bias=bias_d, out=out,
                                stream=stream)
        if ev:
            ev[1].record(stream)
        moe.layer_backward(cfg, x, W["wr"], W["wg"], W["wu"], W["wd"], dout, ws, grads=grads, stream=stream)
        if ev:
            ev[2].record(stream)

    for _ in range(3):
        step()
    torch.cuda.synchronize(dev)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    clocks = _sampler(dev)
    w0 = time.monotonic()
    for i in range(steps):
        step(evs[i])
    torch.cuda.synchronize(dev)
    clk = clocks.stop(window=(w0, time.monotonic()))
    fwd = max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in evs) / steps, dev, world)
    bwd = max_over_ranks(sum(e[1].elapsed_time(e[2]) for e in evs) / steps, dev, world)
    # per-kernel breakdown on separate steps (the phase events add a few us per kernel)
    moe.profile_phases(True)
    moe.profile_read()
    for _ in range(steps):
        step()
    torch.cuda.synchronize(dev)
    ph = moe.profile_read()
    moe.profile_phases(False)
    bwd_flops = 12.0 * n_kept * d * f + 4.0 * cfg.T * d * E
    peak, rule = tensor_peak(peaks, peak_src, clk)
    tf = bwd_flops / (bwd / 1000.0) / 1e12
    unit_flops = {"fwd_gate_up": 4.0 * n_kept * d * f, "fwd_down": 2.0 * n_kept * d * f,
                  "bwd_dh": 2.0 * n_kept * d * f, "bwd_dx": 4.0 * n_kept * d * f, "bwd_wg_down": 2.0 * n_kept * d * f,
                  "bwd_wg_gate": 2.0 * n_kept * d * f, "bwd_wg_up": 2.0 * n_kept * d * f}
    kernels = {}
    for name, (ms, calls) in ph.items():
        if calls:
            k = {"ms": ms / calls}
            if name in unit_flops:
                k["tflops"] = unit_flops[name] / (k["ms"] / 1000.0) / 1e12
                k["frac"] = k["tflops"] / peak
            kernels[name] = k
    res = {"steps": steps, "forward_train_ms": fwd, "backward_ms": bwd,
           "tokens_per_s": world * cfg.T / ((fwd + bwd) / 1000.0),
           "backward_tflops": tf, "backward_frac": tf / peak, "peak_tflops": peak, "peak_rule": rule,
           "backward_algorithmic": "12*d*f*N_kept + 4*T*d*E FLOP", "gpu_launches_per_step": 8 + 10,
           "kernels": kernels, "kernels_note": "per-kernel times from phase events on separate steps",
           "grad_dtype": "fp32 weight gradients, bf16 dx", "clocks": clk}
    del ws, grads
    return res
def graph_decode(moe, cfg, W, xs, out, ws, dev, stream, calls, eager_ms):
    import torch

    x_in = torch.empty_like(xs[0])
    cap = torch.cuda.Stream(dev)
    cap.wait_stream(stream)
    with torch.cuda.stream(cap):
        x_in.copy_(xs[0])
        moe.layer_forward(cfg, x_in, W["wr"], W["wg"], W["wu"], W["wd"], out=out, ws=ws)
    torch.cuda.synchronize(dev)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=cap, capture_error_mode="relaxed"):
        moe.layer_forward(cfg, x_in, W["wr"], W["wg"], W["wu"], W["wd"], out=out, ws=ws)
    torch.cuda.synchronize(dev)
    for i in range(3):
        x_in.copy_(xs[i])
        g.replay()
    torch.cuda.synchronize(dev)
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for i in range(calls):
        x_in.copy_(xs[i])
        g.replay()
    b.record(stream)
    torch.cuda.synchronize(dev)
    ms = a.elapsed_time(b)
    return {"ms_per_call": ms / calls, "tokens_per_s": xs.shape[1] * calls / (ms / 1000.0),
            "speedup_vs_eager": eager_ms / ms,
            "note": "layer launches captured in one CUDA graph; each call = copy of x into the "
                    "captured buffer + replay"}


def decode_bench(moe, W, dev, stream, peaks, peak_src, world):
    import torch

    w = configs.WORKLOADS["grok_decode"]
    cfg = moe.Config(w.T, w.d, w.f, capacity_factor=w.capacity_factor, dtype="bf16")
    xs = torch.stack([torch.from_numpy(configs.make_x(w, call=i)).view(torch.bfloat16) for i in range(w.calls)])
    xs = xs.to(dev)
    ws = torch.empty(moe.workspace_size(cfg), dtype=torch.uint8, device=dev)
    out = torch.empty((w.T, w.d), dtype=torch.bfloat16, device=dev)
    stats = torch.zeros(26, dtype=torch.int32, device=dev)
    used = torch.zeros(8, dtype=torch.int64, device=dev)
    for i in range(3):
        moe.layer_forward(cfg, xs[i], W["wr"], W["wg"], W["wu"], W["wd"], out=out, ws=ws)
    torch.cuda.synchronize(dev)
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    clocks = _sampler(dev)
    w0 = time.monotonic()
    a.record(stream)
    for i in range(w.calls):
        moe.layer_forward(cfg, xs[i], W["wr"], W["wg"], W["wu"], W["wd"], out=out, stats=stats, ws=ws)
    b.record(stream)
    torch.cuda.synchronize(dev)
    clk = clocks.stop(window=(w0, time.monotonic()))
    ms = a.elapsed_time(b)
    # experts used per call (counted after timing, on a second pass)
    n_used = 0
    for i in range(w.calls):
        moe.layer_forward(cfg, xs[i], W["wr"], W["wg"], W["wu"], W["wd"], out=out, stats=stats, ws=ws)
        used += (stats[8:16] > 0).to(torch.int64)
    torch.cuda.synchronize(dev)
    n_used = int(used.sum().item())
    weight_bytes = n_used * 3 * w.d * w.f * 2
    gbs = weight_bytes / (ms / 1000.0) / 1e9
    res = {"workload": w.name, "calls": w.calls, "ms_per_call": ms / w.calls,
           "tokens_per_s": w.T * w.calls / (ms / 1000.0), "expert_weight_gb_per_call": weight_bytes / w.calls / 1e9,
           "achieved_gbs": gbs, "peak_gbs": peaks["hbm_gbs"], "frac": gbs / peaks["hbm_gbs"],
           "peak_source": f"{peak_src} hbm_gbs", "bound": "hbm", "clocks": clk,
           "kernel": "decode_gemm_kernel (weights on the MMA M side)"}
    # the same calls replayed from a CUDA graph: the layer's launches are captured once
    # and each call copies its x into the captured input buffer, then replays
    try:
        res["graph"] = graph_decode(moe, cfg, W, xs, out, ws, dev, stream, w.calls, ms)
    except Exception as exc:  # capture is an optional measurement; report why it is missing
        res["graph"] = {"unavailable": f"{type(exc).__name__}: {exc}"[:200]}
    # the same calls with int8 expert weights (per-channel scales, int8 tensor cores)
    qw = moe.QuantizedExperts(cfg, W["wg"], W["wu"], W["wd"])
    ws8 = torch.empty(moe.lib.moe_workspace_size_w8(cfg.ref), dtype=torch.uint8, device=dev)
    for i in range(3):
        moe.layer_forward_w8(cfg, xs[i], W["wr"], qw, out=out, ws=ws8)
    torch.cuda.synchronize(dev)
    a.record(stream)
    for i in range(w.calls):
        moe.layer_forward_w8(cfg, xs[i], W["wr"], qw, out=out, ws=ws8)
    b.record(stream)
    torch.cuda.synchronize(dev)
    ms8 = a.elapsed_time(b)
    bytes8 = n_used * (3 * w.d * w.f + w.f * 2 * 4 + w.d * 4)  # int8 codes + fp32 scales of the used experts
    gbs8 = bytes8 / (ms8 / 1000.0) / 1e9
    res["int8_weights"] = {"ms_per_call": ms8 / w.calls, "tokens_per_s": w.T * w.calls / (ms8 / 1000.0),
                           "expert_weight_gb_per_call": bytes8 / w.calls / 1e9, "achieved_gbs": gbs8,
                           "frac": gbs8 / peaks["hbm_gbs"], "speedup_vs_bf16": ms / ms8}
    del qw, ws8
    return res


if __name__ == "__main__":
    main()
