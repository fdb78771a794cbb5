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


def _bench_launches_equal(L, g):
    """The launch configuration the benchmark times (router, dispatch, gate/up, and
    the down pass summing into token order with one rounding pass), and the
    one-call layer, give the bits of the step-by-step path checked above."""
    import sparse_moe_layer_07_b200 as moe

    c, D = L.cfg, L.dev
    idx, wts, _ = moe.router_topk(c, D["x"], D["wr"], D["bias"])
    disp = moe.dispatch(c, D["x"], idx, wts)
    h = moe.expert_gate_up(c, disp["x_perm"], disp["offsets"], D["wg"], D["wu"])
    out = moe.expert_down_combine(c, h, disp["offsets"], D["wd"], disp["row_scale"], disp["perm"])
    del h
    torch.cuda.synchronize()
    assert torch.equal(out, g["out"])
    del out
    one = moe.layer_forward(c, D["x"], D["wr"], D["wg"], D["wu"], D["wd"], logit_bias=D["bias"])
    torch.cuda.synchronize()
    assert torch.equal(one, g["out"])
    assert moe.get_device_error() == 0


def test_grok_prefill_full_size(grok):
    host, dev = grok
    w = W["grok_prefill"]
    L = LayerInputs(w, host=host, dev_weights=dev)
    g = run_steps(L, keep_h=False)
    np.testing.assert_array_equal(g["counts_kept"], g["counts_raw"])  # cf = E/k: nothing dropped
    assert int(g["offsets"][-1]) == 2 * w.T
    _check(L, g, _sample(w.T, 62, 11), "grok_prefill")
    _bench_launches_equal(L, g)


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
    _bench_launches_equal(L, g)


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
    oracle's own quantisation, then the decode layer against the weight-only
    definition (the oracle's plain layer on exact activations and the
    dequantised weights), and, as a check of the kernel's internals, against
    the oracle's 8-bit layer that replays the activation row codes."""
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
    deq = [oracle.DequantizedExperts(*ref_q[k]) for k in ("wg", "wu", "wd")]
    ref = oracle.layer_forward(x_all, host["wr"], *deq, float("inf"))
    res = [check_layer_out(L, g["out"], g["y"], g["slot_of"], ref["out"][i * w.T:(i + 1) * w.T], np.arange(w.T))
           for i, (L, g) in enumerate(outs)]
    ref8 = oracle.layer_forward_w8(x_all, host["wr"], *ref_q["wg"], *ref_q["wu"], *ref_q["wd"], float("inf"))
    res8 = [check_layer_out(L, g["out"], g["y"], g["slot_of"], ref8["out"][i * w.T:(i + 1) * w.T], np.arange(w.T))
            for i, (L, g) in enumerate(outs)]
    REPORT["grok_decode_int8"] = {"calls_checked": list(calls), "weight_codes_bit_exact": True,
                                  "max_err_over_rms_weight_only": [list(r) for r in res],
                                  "max_err_over_rms_row_codes_replayed": [list(r) for r in res8]}


def test_grok_train_full_size(grok):
    """Training pair at the full Grok prefill size, in the configuration the
    benchmark times: dx on sampled tokens (each differentiated in fp64 by the
    oracle), and for two experts whole columns of dW_gate / dW_up and rows of
    dW_down (the oracle's hidden-unit slices), within the backward bar."""
    import sparse_moe_layer_07_b200 as moe
    from synth import normal

    host, dev = grok
    w = W["grok_prefill"]
    L = LayerInputs(w, host=host, dev_weights=dev)
    c = L.cfg
    ws = torch.empty(moe.workspace_size_train(c), dtype=torch.uint8, device="cuda")
    moe.layer_forward_train(c, L.dev["x"], dev["wr"], dev["wg"], dev["wu"], dev["wd"], ws)
    go = normal(configs.SEED, 907, (w.T, w.d), dtype="bf16")
    g = moe.layer_backward(c, L.dev["x"], dev["wr"], dev["wg"], dev["wu"], dev["wd"], to_dev(go), ws)
    torch.cuda.synchronize()
    assert moe.get_device_error() == 0
    tol = 8e-2  # max |err| over RMS, the backward bar of test_gpu_train
    tokens = _sample(w.T, 14, 13)
    ref = oracle.layer_backward(L.x, L.wr, L.wg, L.wu, L.wd, w.capacity_factor, go, tokens=tokens)
    gap = oracle.near_tie_gap(ref["logits"])[tokens]
    rows = tokens[gap > 1e-3]
    dx = g["dx"].float().cpu().numpy().astype(np.float64)[rows]
    want = ref["dx"][rows]
    rms = float(np.sqrt(np.mean(want ** 2)))
    err_dx = float(np.max(np.abs(dx - want))) / rms
    assert err_dx <= tol, err_dx
    res = {"dx_tokens": int(rows.size), "dx_max_err_over_rms": err_dx}
    cols = [0, 1, 12345, w.f - 1]
    for e in (0, 5):
        sl = oracle.expert_weight_grad_slices(L.x, L.wr, L.wg, L.wu, L.wd, w.capacity_factor, go, e, cols)
        pairs = (("dw_gate", g["dw_gate"][e][:, cols], sl["dw_gate_cols"]),
                 ("dw_up", g["dw_up"][e][:, cols], sl["dw_up_cols"]),
                 ("dw_down", g["dw_down"][e][cols, :], sl["dw_down_rows"]))
        for name, got_t, want in pairs:
            got = got_t.cpu().numpy().astype(np.float64)
            rms = float(np.sqrt(np.mean(want ** 2)))
            err = float(np.max(np.abs(got - want))) / rms
            assert err <= tol, (name, e, err)
            res[f"{name}_e{e}_max_err_over_rms"] = err
    REPORT["grok_train"] = res
