"""Pins of the CPU oracle against brute force, closed forms and the pages' values.

Each check is written as a function of an oracle object so that the last test
can plant plausible mistakes in a copy of the oracle and show that some pin
fails for every one of them.
"""
import copy
import itertools
import json
import math
import os
import types

import numpy as np
import pytest

import oracle.moe_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------------------
# brute-force helpers (pure Python loops, no numpy linear algebra)
# ----------------------------------------------------------------------------
def bf_logits(x, wr, bias=None):
    T, d = len(x), len(x[0])
    E = len(wr)
    out = [[0.0] * E for _ in range(T)]
    for t in range(T):
        for e in range(E):
            s = 0.0
            for i in range(d):
                s += float(x[t][i]) * float(wr[e][i])
            out[t][e] = s + (0.0 if bias is None else float(bias[e]))
    return out


def bf_top2(row):
    """The unique pair whose members both beat every other expert under (logit desc, index asc)."""
    E = len(row)

    def beats(a, b):
        return row[a] > row[b] or (row[a] == row[b] and a < b)

    found = []
    for a, b in itertools.combinations(range(E), 2):
        if all(beats(a, c) and beats(b, c) for c in range(E) if c not in (a, b)):
            found.append((a, b) if beats(a, b) else (b, a))
    assert len(found) == 1
    return found[0]


def bf_matvec(v, m):
    """v [n] times m [n][p] -> [p]."""
    p = len(m[0])
    out = [0.0] * p
    for i in range(len(v)):
        vi = float(v[i])
        row = m[i]
        for j in range(p):
            out[j] += vi * float(row[j])
    return out


def bf_expert(xt, wg, wu, wd):
    g = bf_matvec(xt, wg)
    u = bf_matvec(xt, wu)
    h = [gi / (1.0 + math.exp(-gi)) * ui for gi, ui in zip(g, u)]
    return bf_matvec(h, wd)


def bf_layer(x, wr, wg, wu, wd, cap, bias=None):
    """Every expert evaluated densely on every token, masked by brute-force top-2 and rank."""
    lg = bf_logits(x, wr, bias)
    T, d, E = len(x), len(x[0]), len(wr)
    out = [[0.0] * d for _ in range(T)]
    pairs = [bf_top2(r) for r in lg]
    for t in range(T):
        l0, l1 = lg[t][pairs[t][0]], lg[t][pairs[t][1]]
        w = {pairs[t][0]: 1.0 / (1.0 + math.exp(l1 - l0)), pairs[t][1]: 1.0 / (1.0 + math.exp(l0 - l1))}
        for e in range(E):
            if e not in w:
                continue
            earlier = sum(1 for s in range(t) if e in pairs[s])  # rank among all earlier routings to e
            if earlier >= cap:
                continue
            y = bf_expert(x[t], wg[e], wu[e], wd[e])
            for i in range(d):
                out[t][i] += w[e] * y[i]
    return lg, pairs, out


def rand_layer(rng, T, d, f, E, scale_r=1.0):
    x = rng.standard_normal((T, d))
    wr = rng.standard_normal((E, d)) * scale_r
    wg = rng.standard_normal((E, d, f)) / math.sqrt(d)
    wu = rng.standard_normal((E, d, f)) / math.sqrt(d)
    wd = rng.standard_normal((E, f, d)) / math.sqrt(f)
    return x, wr, wg, wu, wd


# ----------------------------------------------------------------------------
# the pins, as functions of an oracle object
# ----------------------------------------------------------------------------
def pin_router_logits(o):
    rng = np.random.default_rng(1)
    x = rng.standard_normal((5, 7))
    wr = rng.standard_normal((8, 7))
    bias = rng.standard_normal(8)
    np.testing.assert_allclose(o.router_logits(x, wr), bf_logits(x, wr), rtol=0, atol=1e-12)
    np.testing.assert_allclose(o.router_logits(x, wr, bias), bf_logits(x, wr, bias), rtol=0, atol=1e-12)


def pin_top2_brute_force(o):
    rng = np.random.default_rng(2)
    # small integer logits make exact ties frequent
    lg = rng.integers(-3, 4, size=(400, 8)).astype(np.float64)
    idx, _ = o.top2_softmax(lg)
    for t in range(lg.shape[0]):
        assert tuple(idx[t]) == bf_top2(list(lg[t])), t


def pin_softmax_closed_form(o):
    rng = np.random.default_rng(3)
    lg = rng.standard_normal((300, 8)) * 2
    idx, w = o.top2_softmax(lg)
    l0 = lg[np.arange(300), idx[:, 0]]
    l1 = lg[np.arange(300), idx[:, 1]]
    np.testing.assert_allclose(w[:, 0], 1.0 / (1.0 + np.exp(l1 - l0)), rtol=1e-13, atol=0)
    np.testing.assert_allclose(w.sum(axis=1), 1.0, rtol=0, atol=1e-15)
    assert np.all(w[:, 0] >= w[:, 1])


def pin_zero_router(o):
    x = np.random.default_rng(4).standard_normal((6, 16))
    idx, w = o.top2_softmax(o.router_logits(x, np.zeros((8, 16))))
    assert np.all(idx == np.array([0, 1])) and np.all(w == 0.5)


def pin_scale_invariance(o):
    rng = np.random.default_rng(5)
    x = rng.standard_normal((50, 12))
    wr = rng.standard_normal((8, 12))
    a, _ = o.top2_softmax(o.router_logits(x, wr))
    b, _ = o.top2_softmax(o.router_logits(x, 3.5 * wr))
    np.testing.assert_array_equal(a, b)


def pin_capacity_values(o):
    assert o.capacity(64, 2, 8, 1.25) == 20
    assert o.capacity(2048, 2, 8, 1.25) == 640
    assert o.capacity(8192, 2, 8, 4.0) == 8192
    assert o.capacity(16384, 2, 8, 1.25) == 5120
    assert o.capacity(10, 2, 8, 1.0) == 3          # 2.5 rounds up
    assert o.capacity(32, 2, 8, float("inf")) == 32


def pin_dispatch_brute_force(o):
    rng = np.random.default_rng(6)
    for T, E, cap in [(40, 8, 7), (64, 8, 20), (33, 4, 5), (17, 8, 100)]:
        idx = np.stack([rng.choice(E, 2, replace=False) for _ in range(T)]).astype(np.int32)
        w = rng.random((T, 2))
        r = o.dispatch(idx, w, E, cap)
        slot_of, perm, off = r["slot_of"], r["perm"], r["offsets"]
        kept_count = np.zeros(E, dtype=int)
        for t in range(T):
            for j in range(2):
                e = idx[t, j]
                earlier = sum(1 for s in range(t) if e in idx[s])
                keep = earlier < cap
                assert (slot_of[t, j] >= 0) == keep
                if keep:
                    assert slot_of[t, j] == off[e] + earlier
                    assert perm[slot_of[t, j]] == t
                    assert r["row_scale"][slot_of[t, j]] == w[t, j]
                    kept_count[e] += 1
        np.testing.assert_array_equal(r["counts_kept"], kept_count)
        np.testing.assert_array_equal(r["counts_raw"], np.bincount(idx.ravel(), minlength=E))
        assert np.all(r["counts_kept"] <= cap)
        assert r["n_kept"] == int((slot_of >= 0).sum())
        assert sorted(perm.tolist()) == sorted(int(t) for t, j in zip(*np.nonzero(slot_of >= 0)))
        assert sorted(slot_of[slot_of >= 0].tolist()) == list(range(r["n_kept"]))


def pin_no_drop(o):
    rng = np.random.default_rng(7)
    T = 64
    idx = np.stack([rng.choice(8, 2, replace=False) for _ in range(T)]).astype(np.int32)
    r = o.dispatch(idx, rng.random((T, 2)), 8, o.capacity(T, 2, 8, 8 / 2))
    assert r["dropped"] == 0 and r["n_kept"] == 2 * T


def pin_hand_built_drop(o):
    # 8 tokens, every one routed to experts (0, 1); capacity 3 keeps tokens 0-2 only
    T, d, f = 8, 4, 3
    rng = np.random.default_rng(8)
    x = np.abs(rng.standard_normal((T, d))) + 0.1
    wr = np.zeros((8, d))
    wr[0] = 2.0
    wr[1] = 1.0
    _, _, wg, wu, wd = rand_layer(rng, T, d, f, 8)
    cf = 3 * 8 / (T * 2)  # ceil(cf*T*k/E) = 3
    assert o.capacity(T, 2, 8, cf) == 3
    r = o.layer_forward(x, wr, wg, wu, wd, cf)
    assert np.all(r["idx"] == np.array([0, 1]))
    assert list(r["slot_of"][:, 0]) == [0, 1, 2, -1, -1, -1, -1, -1]
    assert list(r["slot_of"][:, 1]) == [3, 4, 5, -1, -1, -1, -1, -1]
    assert np.all(r["out"][3:] == 0.0)
    assert np.all(np.abs(r["out"][:3]).sum(axis=1) > 0)


def pin_layer_dense_brute_force(o):
    rng = np.random.default_rng(9)
    T, d, f, E = 9, 5, 6, 8
    x, wr, wg, wu, wd = rand_layer(rng, T, d, f, E)
    bias = rng.standard_normal(E) * 0.3
    for cf in (1.0, 2.0, float("inf")):
        cap = o.capacity(T, 2, E, cf)
        lg, pairs, out = bf_layer(x.tolist(), wr.tolist(), wg.tolist(), wu.tolist(), wd.tolist(), cap, bias)
        r = o.layer_forward(x, wr, wg, wu, wd, cf, logit_bias=bias)
        assert [tuple(p) for p in r["idx"]] == pairs
        np.testing.assert_allclose(r["out"], out, rtol=1e-12, atol=1e-12)


def pin_identity_experts(o):
    # d = f and W_gate = W_up = W_down = I: each expert computes silu(x) * x
    rng = np.random.default_rng(10)
    T, d, E = 12, 6, 8
    x = rng.standard_normal((T, d))
    wr = rng.standard_normal((E, d))
    eye = np.broadcast_to(np.eye(d), (E, d, d)).copy()
    r = o.layer_forward(x, wr, eye, eye, eye, float("inf"))
    np.testing.assert_allclose(r["out"], x / (1 + np.exp(-x)) * x, rtol=1e-13, atol=1e-14)


def pin_two_expert_dense(o):
    # E = k = 2, cf = 1: every token goes to both experts, nothing is dropped
    rng = np.random.default_rng(11)
    T, d, f = 10, 4, 7
    x, wr, wg, wu, wd = rand_layer(rng, T, d, f, 2)
    r = o.layer_forward(x, wr, wg, wu, wd, 1.0)
    lg = x @ wr.T
    w0 = 1 / (1 + np.exp(lg[:, 1] - lg[:, 0]))
    y = []
    for e in range(2):
        ye = np.array([bf_expert(x[t], wg[e].tolist(), wu[e].tolist(), wd[e].tolist()) for t in range(T)])
        y.append(ye)
    np.testing.assert_allclose(r["out"], w0[:, None] * y[0] + (1 - w0)[:, None] * y[1], rtol=1e-12, atol=1e-12)


def pin_swiglu_expert_brute_force(o):
    # one expert on its own (d != f, so a transposed operand cannot even run):
    # swiglu_hidden and swiglu_expert against pure-Python loops, row by row
    rng = np.random.default_rng(14)
    n, d, f = 4, 5, 7
    x = rng.standard_normal((n, d))
    wg = rng.standard_normal((d, f)) / math.sqrt(d)
    wu = rng.standard_normal((d, f)) / math.sqrt(d)
    wd = rng.standard_normal((f, d)) / math.sqrt(f)
    h = o.swiglu_hidden(x, wg, wu)
    y = o.swiglu_expert(x, wg, wu, wd)
    assert h.shape == (n, f) and y.shape == (n, d)
    for r in range(n):
        g = bf_matvec(x[r], wg.tolist())
        u = bf_matvec(x[r], wu.tolist())
        np.testing.assert_allclose(h[r], [gi / (1.0 + math.exp(-gi)) * ui for gi, ui in zip(g, u)],
                                   rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(y[r], bf_expert(x[r], wg.tolist(), wu.tolist(), wd.tolist()),
                                   rtol=1e-12, atol=1e-13)


def pin_bf16_decoding(o):
    bits = np.array([0x3F80, 0xC000, 0x3E80, 0x0000, 0x8000, 0x4049], dtype=np.uint16)
    np.testing.assert_array_equal(o.to_f64(bits), [1.0, -2.0, 0.25, 0.0, -0.0, 3.140625])


def pin_quantize_int8(o):
    rng = np.random.default_rng(12)
    w = (rng.standard_normal((3, 40, 24)) * rng.random((1, 1, 24)) * 4).astype(np.float32)
    w[1, :, 5] = 0.0  # an all-zero output channel
    q, sc = o.quantize_int8(w)
    assert q.dtype == np.int8 and sc.dtype == np.float32 and sc.shape == (3, 24)
    # scale is the channel's max magnitude over 127 (channel = last axis)
    np.testing.assert_array_equal(sc, (np.abs(w).max(axis=1) / np.float32(127)).astype(np.float32))
    assert sc[1, 5] == 0 and np.all(q[1, :, 5] == 0)
    # the largest magnitude of every non-zero channel maps to +-127
    am = np.abs(w).argmax(axis=1)
    for e in range(3):
        for n in range(24):
            if sc[e, n] > 0:
                assert abs(int(q[e, am[e, n], n])) == 127
    assert np.abs(q.astype(int)).max() <= 127
    # nearest code: round-trip error at most half a step (+ fp32 division slack)
    err = np.abs(o.dequantize_int8(q, sc) - w)
    assert np.all(err <= sc[:, None, :] * (0.5 + 1e-6))
    # symmetric
    qn, _ = o.quantize_int8(-w)
    np.testing.assert_array_equal(qn, -q)
    # weights that are exactly k * 2^-4 with max |k| = 127 quantize to k
    k = rng.integers(-127, 128, size=(2, 16, 8)).astype(np.float32)
    k[:, 0, :] = 127
    qk, sk = o.quantize_int8(k * np.float32(0.0625))
    np.testing.assert_array_equal(qk, k.astype(np.int8))
    # bf16 bit patterns are accepted and mean the same values
    bits = (w.view(np.uint32) >> 16).astype(np.uint16)
    wb = (bits.astype(np.uint32) << 16).view(np.float32)
    qb, sb = o.quantize_int8(bits)
    qf, sf = o.quantize_int8(wb)
    np.testing.assert_array_equal(qb, qf)
    np.testing.assert_array_equal(sb, sf)


def pin_quantized_layer_uses_dequantized_weights(o):
    rng = np.random.default_rng(13)
    T, d, f = 7, 5, 6
    x, wr, wg, wu, wd = rand_layer(rng, T, d, f, 8)
    qs = [o.quantize_int8(m) for m in (wg, wu, wd)]
    deq = [o.dequantize_int8(q, s) for q, s in qs]
    lazy = [o.DequantizedExperts(q, s) for q, s in qs]
    a = o.layer_forward(x, wr, *deq, 2.0)["out"]
    b = o.layer_forward(x, wr, *lazy, 2.0)["out"]
    np.testing.assert_array_equal(a, b)
    lg, pairs, ref = bf_layer(x.tolist(), wr.tolist(), deq[0].tolist(), deq[1].tolist(), deq[2].tolist(),
                              o.capacity(T, 2, 8, 2.0))
    np.testing.assert_allclose(a, ref, rtol=1e-12, atol=1e-12)


def pin_quantize_rows(o):
    rng = np.random.default_rng(14)
    v = (rng.standard_normal((6, 300)) * np.array([[1e-3], [1.0], [50.0], [0.0], [3.0], [7.0]])).astype(np.float32)
    hi, lo, sc = o.quantize_rows(v)
    assert hi.dtype == np.int8 and lo.dtype == np.int8 and sc.dtype == np.float32
    code = 256 * hi.astype(int) + lo.astype(int)
    assert np.abs(code).max() <= 32512 and lo.min() >= -128 and lo.max() <= 127
    np.testing.assert_array_equal(sc, (np.abs(v).max(axis=1) / np.float32(32512)).astype(np.float32))
    assert sc[3] == 0 and np.all(code[3] == 0)
    # the largest magnitude of each non-zero row codes to +-32512
    am = np.abs(v).argmax(axis=1)
    for r in range(6):
        if sc[r] > 0:
            assert abs(code[r, am[r]]) == 32512
    # nearest code: half a step (+ fp32 division slack)
    err = np.abs(o.dequantize_rows(hi, lo, sc) - v)
    assert np.all(err <= sc[:, None] * (0.5 + 1e-6))
    # hi/lo split: hi = floor((code + 128) / 256) for a few hand values
    for c, h, l in [(0, 0, 0), (127, 0, 127), (128, 1, -128), (-128, 0, -128), (-129, -1, 127),
                    (32512, 127, 0), (-32512, -127, 0), (383, 1, 127), (384, 2, -128)]:
        hh, ll = np.floor_divide(c + 128, 256), c - 256 * np.floor_divide(c + 128, 256)
        assert (hh, ll) == (h, l)
    vv = np.array([[1.0, -1.0, 0.5, 127.0 / 256]], dtype=np.float32) * np.float32(32512 / 256)
    h2, l2, s2 = o.quantize_rows(vv)
    assert s2[0] == np.float32(2.0 ** -8)  # 127 / 32512, exact
    np.testing.assert_array_equal(256 * h2.astype(int) + l2.astype(int), [[32512, -32512, 16256, 127 * 127]])


def pin_int8_layer_exact(o):
    # the 8-bit layer equals the float layer run on the dequantised weights and rows
    rng = np.random.default_rng(15)
    T, d, f = 9, 6, 5
    x, wr, wg, wu, wd = rand_layer(rng, T, d, f, 8)
    q = [o.quantize_int8(m) for m in (wg, wu, wd)]
    r = o.layer_forward_w8(x, wr, q[0][0], q[0][1], q[1][0], q[1][1], q[2][0], q[2][1], 2.0)
    deq = [o.dequantize_int8(*qq) for qq in q]
    lg = o.router_logits(x, wr)
    idx, w = o.top2_softmax(lg)
    disp = o.dispatch(idx, w, 8, o.capacity(T, 2, 8, 2.0))
    ref = np.zeros((T, d))
    for t in range(T):
        for j in range(2):
            if disp["slot_of"][t, j] < 0:
                continue
            e = idx[t, j]
            xr = o.dequantize_rows(*o.quantize_rows(x[t:t + 1]))[0]
            g = [sum(xr[k] * deq[0][e][k, n] for k in range(d)) for n in range(f)]
            u = [sum(xr[k] * deq[1][e][k, n] for k in range(d)) for n in range(f)]
            h = np.array([gi / (1 + math.exp(-gi)) * ui for gi, ui in zip(g, u)])
            hr = o.dequantize_rows(*o.quantize_rows(h.astype(np.float32)[None, :]))[0]
            ref[t] += w[t, j] * np.array([sum(hr[k] * deq[2][e][k, n] for k in range(f)) for n in range(d)])
    np.testing.assert_allclose(r["out"], ref, rtol=1e-12, atol=1e-12)


# ----------------------------------------------------------------------------
# backward pass
# ----------------------------------------------------------------------------
def _bwd_case(seed, T=6, d=5, f=4, E=8, bias=True):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, d))
    wr = rng.standard_normal((E, d))
    b = rng.standard_normal(E) * 0.5 if bias else None
    wg = rng.standard_normal((E, d, f)) * 0.7
    wu = rng.standard_normal((E, d, f)) * 0.7
    wd = rng.standard_normal((E, f, d)) * 0.7
    go = rng.standard_normal((T, d))
    return x, wr, b, wg, wu, wd, go


def pin_backward_finite_differences(o):
    # every gradient entry against central differences of L = sum(out * dout), on a case
    # with dropped assignments (cap = 2 for 6 tokens x 2 slots over 8 experts) and a bias
    x, wr, b, wg, wu, wd, go = _bwd_case(21)
    cf = 1.0
    r = o.layer_backward(x, wr, wg, wu, wd, cf, go, logit_bias=b)
    assert r["dropped"] > 0
    assert o.near_tie_gap(r["logits"]).min() > 1e-3

    def loss(x_, wr_, b_, wg_, wu_, wd_):
        return float(np.sum(o.layer_forward(x_, wr_, wg_, wu_, wd_, cf, logit_bias=b_)["out"] * go))

    args = [x, wr, b, wg, wu, wd]
    names = ["dx", "dw_router", "dbias", "dw_gate", "dw_up", "dw_down"]
    eps = 1e-6
    for a_i, name in enumerate(names):
        base = args[a_i]
        num = np.zeros(base.shape)
        for pos in np.ndindex(base.shape):
            hi = [a.copy() if i == a_i else a for i, a in enumerate(args)]
            lo = [a.copy() if i == a_i else a for i, a in enumerate(args)]
            hi[a_i][pos] += eps
            lo[a_i][pos] -= eps
            num[pos] = (loss(*hi) - loss(*lo)) / (2 * eps)
        np.testing.assert_allclose(r[name], num, rtol=1e-6, atol=1e-6, err_msg=name)


def pin_backward_autograd(o):
    # a larger case against torch autograd (float64) of the forward restated with the
    # oracle's routing decisions held fixed
    import torch

    T, d, f, E = 40, 12, 10, 8
    x, wr, b, wg, wu, wd, go = _bwd_case(22, T, d, f, E)
    cf = 1.25
    r = o.layer_backward(x, wr, wg, wu, wd, cf, go, logit_bias=b)
    assert r["dropped"] > 0
    tx, twr, tb, twg, twu, twd = (torch.tensor(a, requires_grad=True) for a in (x, wr, b, wg, wu, wd))
    lg = tx @ twr.T + tb
    idx = torch.tensor(r["idx"], dtype=torch.int64)
    sel = torch.gather(lg, 1, idx)
    wsm = torch.softmax(sel, dim=1)
    out = torch.zeros(T, d, dtype=torch.float64)
    for t in range(T):
        for j in range(2):
            if r["slot_of"][t, j] < 0:
                continue
            e = int(idx[t, j])
            hdn = torch.nn.functional.silu(tx[t] @ twg[e]) * (tx[t] @ twu[e])
            out = out.index_add(0, torch.tensor([t]), (wsm[t, j] * (hdn @ twd[e]))[None])
    (out * torch.tensor(go)).sum().backward()
    for name, ten in zip(["dx", "dw_router", "dbias", "dw_gate", "dw_up", "dw_down"], (tx, twr, tb, twg, twu, twd)):
        np.testing.assert_allclose(r[name], ten.grad.numpy(), rtol=1e-10, atol=1e-10, err_msg=name)


def pin_backward_dropped_token(o):
    # a token whose two assignments are both dropped has out = 0 whatever its x is, so
    # its dx, dlogits and dweight are 0; gradients are linear in dout
    x, wr, b, wg, wu, wd, go = _bwd_case(23, T=8)
    bias = np.array([40.0, 30.0, 0, 0, 0, 0, 0, 0])
    r = o.layer_backward(x, wr, wg, wu, wd, 0.5, go, logit_bias=bias)
    cap = o.capacity(8, 2, 8, 0.5)
    assert cap == 1 and (r["idx"] == [0, 1]).all()
    assert np.all(r["dx"][1:] == 0) and np.all(r["dlogits"][1:] == 0) and np.all(r["dweight"][1:] == 0)
    assert np.any(r["dx"][0] != 0)
    r2 = o.layer_backward(x, wr, wg, wu, wd, 0.5, 3.0 * go, logit_bias=bias)
    for k in ("dx", "dw_router", "dw_gate", "dw_up", "dw_down"):
        np.testing.assert_allclose(r2[k], 3.0 * r[k], rtol=1e-12, atol=1e-12)


def pin_backward_subsets_and_slices(o):
    # the token-subset and hidden-unit-slice forms give exactly the corresponding
    # parts of the whole backward
    x, wr, b, wg, wu, wd, go = _bwd_case(24, T=10, d=6, f=7)
    full = o.layer_backward(x, wr, wg, wu, wd, 1.0, go, logit_bias=b)
    sub = [1, 4, 9]
    part = o.layer_backward(x, wr, wg, wu, wd, 1.0, go, logit_bias=b, tokens=sub)
    for k in ("dx", "dlogits", "dweight"):
        np.testing.assert_allclose(part[k][sub], full[k][sub], rtol=1e-12, atol=1e-12)
        rest = np.setdiff1d(np.arange(10), sub)
        assert np.all(part[k][rest] == 0)
    for e in range(8):
        cols = [0, 3, 6]
        sl = o.expert_weight_grad_slices(x, wr, wg, wu, wd, 1.0, go, e, cols, logit_bias=b)
        np.testing.assert_allclose(sl["dw_gate_cols"], full["dw_gate"][e][:, cols], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(sl["dw_up_cols"], full["dw_up"][e][:, cols], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(sl["dw_down_rows"], full["dw_down"][e][cols, :], rtol=1e-12, atol=1e-12)


ALL_PINS = [pin_router_logits, pin_top2_brute_force, pin_softmax_closed_form, pin_zero_router,
            pin_scale_invariance, pin_capacity_values, pin_dispatch_brute_force, pin_no_drop,
            pin_hand_built_drop, pin_layer_dense_brute_force, pin_identity_experts,
            pin_two_expert_dense, pin_bf16_decoding, pin_quantize_int8,
            pin_quantized_layer_uses_dequantized_weights, pin_quantize_rows, pin_int8_layer_exact,
            pin_backward_finite_differences, pin_backward_autograd, pin_backward_dropped_token,
            pin_backward_subsets_and_slices, pin_swiglu_expert_brute_force]


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda p: p.__name__)
def test_pin(pin):
    pin(O)


def test_expert_batch_size_golden():
    with open(os.path.join(GOLDEN, "expert_batch_size.json")) as fh:
        g = json.load(fh)
    for c in g["cases"]:
        assert O.expert_batch_size(c["global_batch"], c["seq_len"]) == c["tokens_per_expert"]


def test_utilization_balanced_is_one():
    np.testing.assert_allclose(O.expert_utilization([250] * 8), 1.0)
    u = O.expert_utilization([400, 100, 250, 250, 250, 250, 250, 250])
    assert u[0] == pytest.approx(1.6) and u.sum() == pytest.approx(8 / 2 * 2)


def test_near_tie_gap():
    lg = np.array([[3.0, 1.0, 2.0, 0.5, 0, 0, 0, 0]])
    assert O.near_tie_gap(lg)[0] == pytest.approx(1.0)


# ----------------------------------------------------------------------------
# planted mistakes: each mutant of the oracle must fail at least one pin
# ----------------------------------------------------------------------------
def _mutant(**overrides):
    m = types.SimpleNamespace(**{k: getattr(O, k) for k in dir(O) if not k.startswith("_")})
    for k, v in overrides.items():
        setattr(m, k, v)
    # layer_forward must call the mutated pieces
    def layer_forward(x, w_router, w_gate, w_up, w_down, capacity_factor, logit_bias=None,
                      top_k=2, tokens=None, keep_hidden=False):
        saved = {k: getattr(O, k) for k in overrides}
        try:
            for k, v in overrides.items():
                setattr(O, k, v)
            return saved.get("layer_forward", O.layer_forward)(
                x, w_router, w_gate, w_up, w_down, capacity_factor, logit_bias, top_k, tokens, keep_hidden)
        finally:
            for k, v in saved.items():
                setattr(O, k, v)
    m.layer_forward = layer_forward

    def layer_backward(*a, **k):
        saved = {kk: getattr(O, kk) for kk in overrides}
        try:
            for kk, v in overrides.items():
                setattr(O, kk, v)
            return overrides.get("layer_backward", saved.get("layer_backward", O.layer_backward))(*a, **k)
        finally:
            for kk, v in saved.items():
                setattr(O, kk, v)
    m.layer_backward = layer_backward
    return m


def _top2_ascending_ties(lg, top_k=2):
    lg = np.asarray(lg, dtype=np.float64)
    order = np.argsort(-lg, axis=1, kind="stable")[:, :top_k]
    # ties resolved toward the higher index
    rev = lg.shape[1] - 1 - np.argsort(-lg[:, ::-1], axis=1, kind="stable")[:, :top_k]
    sel = np.take_along_axis(lg, rev, axis=1)
    ex = np.exp(sel - sel.max(axis=1, keepdims=True))
    return rev.astype(np.int32), ex / ex.sum(axis=1, keepdims=True)


def _softmax_all8(lg, top_k=2):
    lg = np.asarray(lg, dtype=np.float64)
    order = np.argsort(-lg, axis=1, kind="stable")[:, :top_k]
    p = np.exp(lg - lg.max(axis=1, keepdims=True))
    p = p / p.sum(axis=1, keepdims=True)
    return order.astype(np.int32), np.take_along_axis(p, order, axis=1)


def _dispatch_off_by_one(idx, w, E, cap):
    return _orig_dispatch(idx, w, E, cap + 1)


_orig_dispatch = O.dispatch
_orig_silu = O.silu
_orig_router = O.router_logits
_orig_hidden = O.swiglu_hidden
_orig_capacity = O.capacity
_orig_expert = O.swiglu_expert

MUTANTS = {
    "silu_is_identity": dict(silu=lambda z: z),
    "sigmoid_sign_flipped": dict(silu=lambda z: z / (1.0 + np.exp(z))),
    "router_bias_dropped": dict(router_logits=lambda x, wr, b=None: _orig_router(x, wr, None)),
    "router_transposed_scale": dict(router_logits=lambda x, wr, b=None: 2 * _orig_router(x, wr, b)),
    "ties_to_higher_index": dict(top2_softmax=_top2_ascending_ties),
    "softmax_over_all_experts": dict(top2_softmax=_softmax_all8),
    "capacity_off_by_one": dict(dispatch=_dispatch_off_by_one),
    "capacity_floor": dict(capacity=lambda T, k, E, cf: T if math.isinf(cf) else int(math.floor(cf * T * k / E))),
    "gate_up_swapped": dict(swiglu_hidden=lambda x, g, u: _orig_hidden(x, u, g)),
    "expert_gate_up_swapped": dict(swiglu_expert=lambda x, g, u, dn: _orig_expert(x, u, g, dn)),
    "expert_silu_dropped": dict(swiglu_expert=lambda x, g, u, dn: ((O.to_f64(x) @ O.to_f64(g))
                                                                   * (O.to_f64(x) @ O.to_f64(u))) @ O.to_f64(dn)),
    "quant_per_row": dict(quantize_int8=lambda w: _quant_rows(w)),
    "quant_scale_128": dict(quantize_int8=lambda w: _quant_div(w, 128.0)),
    "quant_floor": dict(quantize_int8=lambda w: _quant_floor(w)),
    "rows_hi_rounds": dict(quantize_rows=lambda v: _rows_round_hi(v)),
    "rows_no_h_requant": dict(layer_forward_w8=lambda *a, **k: _w8_skip_h(*a, **k)),
    "bwd_silu_grad_sigmoid_only": dict(silu_grad=lambda z: 1.0 / (1.0 + np.exp(-z))),
    "bwd_no_router_term_in_dx": dict(layer_backward=lambda *a, **k: _bwd_no_router_dx(*a, **k)),
    "bwd_softmax_grad_without_mean": dict(layer_backward=lambda *a, **k: _bwd_no_mean(*a, **k)),
    "bwd_gate_up_grads_swapped": dict(layer_backward=lambda *a, **k: _bwd_swap_gu(*a, **k)),
}


def _bwd_no_router_dx(x, wr, *a, **k):
    r = _orig_bwd(x, wr, *a, **k)
    r["dx"] = r["dx"] - r["dlogits"] @ O.to_f64(wr)
    return r


def _bwd_no_mean(x, wr, *a, **k):
    r = _orig_bwd(x, wr, *a, **k)
    extra = np.zeros_like(r["dlogits"])
    mean = np.sum(r["w"] * r["dweight"], axis=1)
    for t in range(extra.shape[0]):
        for j in range(r["idx"].shape[1]):
            extra[t, r["idx"][t, j]] += r["w"][t, j] * mean[t]
    r["dlogits"] = r["dlogits"] + extra
    r["dx"] = r["dx"] + extra @ O.to_f64(wr)
    r["dw_router"] = r["dlogits"].T @ O.to_f64(x)
    r["dbias"] = r["dlogits"].sum(axis=0)
    return r


def _bwd_swap_gu(*a, **k):
    r = _orig_bwd(*a, **k)
    r["dw_gate"], r["dw_up"] = r["dw_up"], r["dw_gate"]
    return r


_orig_bwd = O.layer_backward


def _rows_round_hi(v):
    hi, lo, s = _orig_rows(v)
    code = 256 * hi.astype(np.int64) + lo
    h2 = np.rint(code / 256.0).astype(np.int64)
    return np.clip(h2, -128, 127).astype(np.int8), (code - 256 * h2).clip(-128, 127).astype(np.int8), s


def _w8_skip_h(x, wr, qg, sg, qu, su, qd, sd, cf, logit_bias=None, top_k=2, tokens=None):
    saved = O.quantize_rows
    calls = {"n": 0}

    def only_first(v):
        calls["n"] += 1
        if calls["n"] % 2 == 0:  # pass H through unquantised
            v = np.asarray(v, dtype=np.float64)
            return np.zeros(v.shape, np.int8), np.zeros(v.shape, np.int8), np.zeros(v.shape[:-1], np.float32)
        return saved(v)
    O.quantize_rows = only_first
    try:
        return _orig_w8(x, wr, qg, sg, qu, su, qd, sd, cf, logit_bias, top_k, tokens)
    finally:
        O.quantize_rows = saved


_orig_rows = O.quantize_rows
_orig_w8 = O.layer_forward_w8


def _quant_rows(w):
    q, s = _orig_quant(np.swapaxes(np.asarray(w, dtype=np.float32), -1, -2))
    return np.swapaxes(q, -1, -2), s


def _quant_div(w, m):
    wf = np.asarray(w, dtype=np.float32)
    s = (np.abs(wf).max(axis=-2) / np.float32(m)).astype(np.float32)
    q = np.clip(np.rint(wf / np.where(s > 0, s, 1)[..., None, :]), -127, 127).astype(np.int8)
    return q, s


def _quant_floor(w):
    wf = np.asarray(w, dtype=np.float32)
    s = (np.abs(wf).max(axis=-2) / np.float32(127)).astype(np.float32)
    q = np.clip(np.floor(wf / np.where(s > 0, s, 1)[..., None, :]), -127, 127).astype(np.int8)
    return q, s


_orig_quant = O.quantize_int8


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name):
    m = _mutant(**MUTANTS[name])
    failures = 0
    for pin in ALL_PINS:
        try:
            pin(m)
        except Exception:  # a failed assertion, or a pin that cannot even run on the mutant
            failures += 1
    assert failures >= 1, f"no pin catches mutant {name}"
