"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI,
run the oracle on the same input bits, and compare them with the tolerances
stated in the test plan.

Tolerances (derived in the design notes):
  logits  |dl| <= (d + 2) * 2^-24 * sum_i |x_i w_i| + 2^-23 |l|   (fp32 FMA chain)
  weights |dw| <= (|dl_0| + |dl_1|) / 4 + 4e-7                    (sigmoid slope <= 1/4)
  indices, counts, offsets, perm, slot_of, drop mask: bit-exact; tokens whose
          oracle gap between the 2nd and 3rd logit is < 1e-3 are excluded and
          counted, and dispatch is then checked against the oracle's capacity
          step fed with the GPU's indices
  out     max|err| <= 2e-2 RMS(out) (bf16), <= 1e-5 RMS(out) (fp32)
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import sparse_moe_layer_07_b200 as moe
from synth import configs

NEAR_TIE = 1e-3
OUT_TOL = {"bf16": 2e-2, "f32": 1e-5}


def to_dev(a, device="cuda"):
    t = torch.from_numpy(np.ascontiguousarray(a)).to(device)
    return t.view(torch.bfloat16) if a.dtype == np.uint16 else t


def to_np64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


class LayerInputs:
    """Host (numpy, storage bits) and device copies of one workload's tensors."""

    def __init__(self, w: configs.Workload, call: int = 0, host=None, dev_weights=None, x=None):
        self.w = w
        if host is None:
            host = dict(wr=configs.make_router(w), wg=configs.make_w_gate(w), wu=configs.make_w_up(w),
                        wd=configs.make_w_down(w))
        self.x = configs.make_x(w, call) if x is None else x
        self.wr, self.wg, self.wu, self.wd = host["wr"], host["wg"], host["wu"], host["wd"]
        self.bias = configs.make_bias(w)
        if dev_weights is None:
            self.dev = {k: to_dev(getattr(self, k)) for k in ("x", "wr", "wg", "wu", "wd")}
        else:
            self.dev = dict(dev_weights)
            self.dev["x"] = to_dev(self.x)
        self.dev["bias"] = None if self.bias is None else to_dev(self.bias)
        self.cfg = moe.Config(w.T, w.d, w.f, capacity_factor=w.capacity_factor, dtype=w.storage)


def run_steps(L: LayerInputs, keep_h=True):
    """Run router -> dispatch -> gate/up -> down -> combine through the separate entry points."""
    c, D = L.cfg, L.dev
    idx, wts, logits = moe.router_topk(c, D["x"], D["wr"], D["bias"], want_logits=True)
    disp = moe.dispatch(c, D["x"], idx, wts)
    h = moe.expert_gate_up(c, disp["x_perm"], disp["offsets"], D["wg"], D["wu"])
    y = moe.expert_down(c, h, disp["offsets"], D["wd"], disp["row_scale"])
    out = moe.combine(c, y, disp["slot_of"], wts, weights_applied=True)
    torch.cuda.synchronize()
    r = {"idx": idx.cpu().numpy(), "w": wts.cpu().numpy(), "logits": logits.cpu().numpy().astype(np.float64),
         "out": out}
    for k in ("counts_raw", "counts_kept", "offsets", "perm", "slot_of", "row_scale"):
        r[k] = disp[k].cpu().numpy()
    r["x_perm"] = disp["x_perm"]
    r["h"] = h if keep_h else None
    r["y"] = y
    return r


def run_steps_w8(L, qw):
    """Router -> dispatch -> int8 expert FFN -> combine through the separate entry points."""
    c, D = L.cfg, L.dev
    idx, wts, logits = moe.router_topk(c, D["x"], D["wr"], D["bias"], want_logits=True)
    disp = moe.dispatch(c, D["x"], idx, wts)
    y, ws = moe.expert_ffn_w8(c, disp["x_perm"], disp["offsets"], qw, disp["row_scale"])
    out = moe.combine(c, y, disp["slot_of"], wts, weights_applied=True)
    torch.cuda.synchronize()
    g = {"idx": idx.cpu().numpy(), "w": wts.cpu().numpy(), "logits": logits.cpu().numpy().astype(np.float64),
         "out": out, "y": y, "ws": moe.w8_workspace_views(c, ws), "x_perm": disp["x_perm"]}
    for k in ("counts_raw", "counts_kept", "offsets", "perm", "slot_of", "row_scale"):
        g[k] = disp[k].cpu().numpy()
    return g


def logit_bound(x, wr, logits64, d):
    ax = np.abs(oracle.to_f64(x))
    aw = np.abs(oracle.to_f64(wr))
    s = ax @ aw.T
    return (d + 2) * 2.0 ** -24 * s + 2.0 ** -23 * np.abs(logits64)


def check_routing(L: LayerInputs, g, ref_logits):
    """Logits within the fp32 bound; indices bit-exact except near ties; weights within bound.
    Returns (near-tie token mask, mismatching-token mask)."""
    T = L.w.T
    bound = logit_bound(L.x, L.wr, ref_logits, L.w.d)
    dl = np.abs(g["logits"] - ref_logits)
    assert np.all(dl <= bound), f"logit error {np.max(dl - bound):.3e} above bound"
    ref_idx, ref_w = oracle.top2_softmax(ref_logits)
    gap = oracle.near_tie_gap(ref_logits)
    tie = gap < NEAR_TIE
    same = np.sort(g["idx"], axis=1) == np.sort(ref_idx, axis=1)
    same = same.all(axis=1)
    bad = ~same & ~tie
    assert not bad.any(), f"{bad.sum()} tokens route differently without a near tie: {np.nonzero(bad)[0][:10]}"
    # weights per (token, expert) for tokens whose pair matches
    rows = np.nonzero(same)[0]
    for j in range(2):
        e = g["idx"][rows, j]
        jr = np.where(ref_idx[rows, 0] == e, 0, 1)
        wref = ref_w[rows, jr]
        tol = (bound[rows, g["idx"][rows, 0]] + bound[rows, g["idx"][rows, 1]]) / 4 + 4e-7
        assert np.all(np.abs(g["w"][rows, j] - wref) <= tol), "routing weight outside bound"
    assert np.allclose(g["w"].sum(axis=1), 1.0, atol=2e-7)
    return tie, ~same


def check_dispatch(L: LayerInputs, g):
    """Bit-exact against the oracle's capacity step fed with the GPU's indices."""
    cap = oracle.capacity(L.w.T, 2, 8, L.w.capacity_factor)
    assert moe.capacity(L.cfg) == min(cap, L.w.T)
    ref = oracle.dispatch(g["idx"], g["w"].astype(np.float64), 8, cap)
    np.testing.assert_array_equal(g["counts_raw"], ref["counts_raw"])
    np.testing.assert_array_equal(g["counts_kept"], ref["counts_kept"])
    np.testing.assert_array_equal(g["offsets"], ref["offsets"])
    n = ref["n_kept"]
    np.testing.assert_array_equal(g["perm"][:n], ref["perm"])
    np.testing.assert_array_equal(g["slot_of"], ref["slot_of"])
    np.testing.assert_array_equal(g["row_scale"][:n], ref["row_scale"].astype(np.float32))
    assert np.all(g["counts_kept"] <= cap)
    return ref


def check_out_rows(L: LayerInputs, got_rows, ref_rows, dtype):
    """max|got - ref| <= OUT_TOL * RMS(ref) over the given rows; returns max|err| / RMS."""
    rms = float(np.sqrt(np.mean(ref_rows ** 2)))
    err = float(np.max(np.abs(got_rows - ref_rows))) if ref_rows.size else 0.0
    tol = OUT_TOL[dtype] * rms
    assert err <= tol, f"max|err| {err:.3e} > {tol:.3e} (rms {rms:.3e})"
    return err / rms if rms else 0.0


def combine_fp32(y_t, slot_of_rows):
    """The combine's fp32 sum before the output rounding, from the GPU's expert outputs
    y_t (device, [T*k, d], routing weight already applied): 0 + y[slot0] + y[slot1]
    in fp32 with slot 0 first; skipped slots add nothing."""
    s = np.asarray(slot_of_rows)
    used = np.unique(s[s >= 0])
    ys = y_t[torch.as_tensor(used, device=y_t.device, dtype=torch.long)].float().cpu().numpy() if used.size else None
    pos = {int(v): i for i, v in enumerate(used)}
    out = np.zeros((s.shape[0], y_t.shape[1]), dtype=np.float32)
    for j in range(s.shape[1]):
        m = s[:, j] >= 0
        if m.any():
            out[m] = out[m] + ys[[pos[int(v)] for v in s[m, j]]]
    return out


def check_layer_out(L: LayerInputs, got_t, y_t, slot_of, ref_rows, rows):
    """Layer output on `rows` against the oracle.

    Rows whose assignments were all dropped must be exactly zero on both sides;
    RMS and the bar are taken over the rows the layer computes.  fp32 layers: max|err| <= 1e-5 RMS directly.  bf16 layers: the output is the
    fp32 combine rounded once to bf16, and that rounding alone can exceed
    2e-2 RMS when max|out| > ~5 RMS (half an ulp is 2^-8 relative).  So the check
    is split: (1) the fp32 combine of the GPU's expert outputs is within
    max|err| <= 2e-2 RMS of the oracle; (2) the bf16 output equals that fp32
    value rounded to nearest-even, bit for bit.  Returns (pre-rounding max|err|/RMS,
    output max|err|/RMS)."""
    rows = np.asarray(rows)
    computed = (np.asarray(slot_of)[rows] >= 0).any(axis=1)
    got_all = to_np64(got_t[torch.as_tensor(rows, device=got_t.device)]) if len(rows) else np.zeros((0, L.w.d))
    # rows with no kept assignment must be exactly zero; the bar applies to the computed rows
    assert np.all(got_all[~computed] == 0.0) and np.all(ref_rows[~computed] == 0.0)
    rows, ref_rows, got = rows[computed], ref_rows[computed], got_all[computed]
    if L.w.storage != "bf16":
        r = check_out_rows(L, got, ref_rows, "f32")
        return r, r
    pre = combine_fp32(y_t, slot_of[rows])
    r_pre = check_out_rows(L, pre.astype(np.float64), ref_rows, "bf16")
    import synth

    rounded = oracle.to_f64(synth.round_bf16(pre.astype(np.float64)).reshape(pre.shape))
    assert np.array_equal(got, rounded), "bf16 output is not the rounded fp32 combine"
    rms = float(np.sqrt(np.mean(ref_rows ** 2))) if ref_rows.size else 1.0
    return r_pre, float(np.max(np.abs(got - ref_rows))) / rms if ref_rows.size else 0.0
