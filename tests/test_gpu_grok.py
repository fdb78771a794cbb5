"""Full-size Grok-1-shape parity (d=6144, f=32768, E=8, top-2), in the launch
configuration the benchmark times.

Router logits, top-2, counts, permutation, slot map and drop mask are checked
over every token; the layer output is checked on a seeded sample of tokens
(the oracle evaluates them one by one in fp64).  Set PARITY_REPORT=<path> to
write the measured statistics as JSON.
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from synth import configs

from parity_util import (LayerInputs, check_dispatch, check_layer_out, check_routing, run_steps, run_steps_w8,
                         to_dev)

pytestmark = pytest.mark.gpu

W = configs.WORKLOADS
REPORT = {}


@pytest.fixture(scope="module")
def grok():
    w = W["grok_prefill"]
    host = dict(wr=configs.make_router(w), wg=configs.make_w_gate(w), wu=configs.make_w_up(w),
                wd=configs.make_w_down(w))
    dev = {k: to_dev(v) for k, v in host.items()}
    yield host, dev
    path = os.environ.get("PARITY_REPORT")
    if path:
        with open(path, "w") as fh:
            json.dump(REPORT, fh, indent=1)


def _sample(T, n, seed, extra=()):
    rng = np.random.default_rng(seed)
    s = set(rng.choice(T, size=n, replace=False).tolist()) | {0, T - 1} | set(int(v) for v in extra)
    return np.array(sorted(s))


def _check(L, g, tokens, name):
    ref = oracle.layer_forward(L.x, L.wr, L.wg, L.wu, L.wd, L.w.capacity_factor, logit_bias=L.bias,
                               tokens=tokens)
    tie, mismatch = check_routing(L, g, ref["logits"])
    check_dispatch(L, g)
    same = (np.sort(g["idx"][tokens], 1) == np.sort(ref["idx"][tokens], 1)).all(1)
    keep_same = ((g["slot_of"][tokens] >= 0) == (ref["slot_of"][tokens] >= 0)).all(1)
    ok = same & keep_same
    r_pre, r_out = check_layer_out(L, g["out"], g["y"], g["slot_of"], ref["out"][ok], tokens[ok])
    kept = g["counts_kept"].astype(np.int64)
    REPORT[name] = {"T": L.w.T, "near_tie_tokens": int(tie.sum()), "routing_mismatch_tokens": int(mismatch.sum()),
                    "counts_raw": g["counts_raw"].tolist(), "counts_kept": kept.tolist(),
                    "dropped": int(2 * L.w.T - kept.sum()),
                    "expert0_share_raw": float(g["counts_raw"][0] / (2 * L.w.T)),
                    "imbalance_max_over_mean_kept": float(kept.max() / kept.mean()),
                    "sampled_tokens": int(len(tokens)), "compared_tokens": int(ok.sum()),
                    "max_err_over_rms_fp32_combine": r_pre, "max_err_over_rms_bf16_out": r_out}
    return ref


def test_grok_prefill_full_size(grok):
    host, dev = grok
    w = W["grok_prefill"]
    L = LayerInputs(w, host=host, dev_weights=dev)
    g = run_steps(L, keep_h=False)
    np.testing.assert_array_equal(g["counts_kept"], g["counts_raw"])  # cf = E/k: nothing dropped
    assert int(g["offsets"][-1]) == 2 * w.T
    _check(L, g, _sample(w.T, 62, 11), "grok_prefill")


def test_grok_skew_full_size(grok):
    host, dev = grok
    w = W["grok_skew"]
    L = LayerInputs(w, host=host, dev_weights=dev)
    g = run_steps(L, keep_h=False)
    cap = oracle.capacity(w.T, 2, 8, w.capacity_factor)
    assert g["counts_kept"].max() <= cap and g["counts_raw"][0] > cap  # expert 0 overflows
    partly = np.nonzero((g["slot_of"] < 0).any(1))[0]
    extra = np.random.default_rng(5).choice(partly, size=min(16, partly.size), replace=False)
    _check(L, g, _sample(w.T, 46, 12, extra), "grok_skew")


def test_grok_decode_full_size(grok):
    host, dev = grok
    w = W["grok_decode"]
    calls = (0, 57, 99)
    outs = []
    for c in calls:
        L = LayerInputs(w, call=c, host=host, dev_weights=dev)
        g = run_steps(L, keep_h=False)
        assert int(g["offsets"][-1]) == 2 * w.T  # cap = T: nothing dropped
        check_routing(L, g, oracle.router_logits(L.x, L.wr))
        check_dispatch(L, g)
        outs.append((L, g))
    # with no capacity drop every token is independent, so one oracle call covers all sampled calls
    x_all = np.concatenate([L.x for L, _ in outs])
    ref = oracle.layer_forward(x_all, host["wr"], host["wg"], host["wu"], host["wd"], float("inf"))
    res = []
    for i, (L, g) in enumerate(outs):
        rows = np.arange(w.T)
        res.append(check_layer_out(L, g["out"], g["y"], g["slot_of"], ref["out"][i * w.T:(i + 1) * w.T], rows))
    REPORT["grok_decode"] = {"calls_checked": list(calls), "max_err_over_rms": [list(r) for r in res],
                             "experts_used": [int((g["counts_kept"] > 0).sum()) for _, g in outs]}


def test_grok_decode_int8_full_size(grok):
    """int8 expert weights at full Grok size: every code and scale against the
    oracle's own quantisation, then the decode layer against the oracle's 8-bit
    layer (its own codes for weights and rows)."""
    import sparse_moe_layer_07_b200 as moe

    host, dev = grok
    w = W["grok_decode"]
    cfg = moe.Config(w.T, w.d, w.f, capacity_factor=w.capacity_factor, dtype="bf16")
    qw = moe.QuantizedExperts(cfg, dev["wg"], dev["wu"], dev["wd"])
    torch.cuda.synchronize()
    ref_q = {}
    for name, gq, gs in (("wg", qw.q_gate, qw.s_gate), ("wu", qw.q_up, qw.s_up), ("wd", qw.q_down, qw.s_down)):
        qs, ss = [], []
        for e in range(8):
            q, s = oracle.quantize_int8(host[name][e])
            assert np.array_equal(gq[e].cpu().numpy(), q), (name, e)
            assert np.array_equal(gs[e].cpu().numpy(), s), (name, e)
            qs.append(q)
            ss.append(s)
        ref_q[name] = (np.stack(qs), np.stack(ss))
    calls = (0, 99)
    outs = []
    for c in calls:
        L = LayerInputs(w, call=c, host=host, dev_weights=dev)
        g = run_steps_w8(L, qw)
        assert int(g["offsets"][-1]) == 2 * w.T
        check_routing(L, g, oracle.router_logits(L.x, L.wr))
        check_dispatch(L, g)
        outs.append((L, g))
    # no capacity drop: tokens are independent, so one oracle call covers both batches
    x_all = np.concatenate([L.x for L, _ in outs])
    ref = oracle.layer_forward_w8(x_all, host["wr"], *ref_q["wg"], *ref_q["wu"], *ref_q["wd"], float("inf"))
    res = [check_layer_out(L, g["out"], g["y"], g["slot_of"], ref["out"][i * w.T:(i + 1) * w.T], np.arange(w.T))
           for i, (L, g) in enumerate(outs)]
    REPORT["grok_decode_int8"] = {"calls_checked": list(calls), "weight_codes_bit_exact": True,
                                  "max_err_over_rms": [list(r) for r in res]}
