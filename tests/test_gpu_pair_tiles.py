"""CTA-pair (2-SM) tiles of the bf16 grouped GEMMs, through the C ABI.

Both tile shapes accumulate every output element over K in the same order
(16-wide K steps, fp32), so the pair path must give the single-CTA path's
bits exactly: H, Y, the fused layer output and the training forward's saved
pre-activations.  It is also checked against the oracle with the bf16 layer
bar (max|err| <= 2e-2 RMS before the output rounding).

The ragged case sets the expert row counts directly so that every kind of
last pair block appears: no rows, 1 row, 64, 65 and 128 rows (the second CTA
computes rows past the expert's end only), 129 (both CTAs hold kept rows), 255,
and more than one block.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import sparse_moe_layer_07_b200 as moe
from synth import configs, normal

from parity_util import LayerInputs, check_layer_out, run_steps, to_dev, to_np64

pytestmark = pytest.mark.gpu

W = configs.WORKLOADS

CASES = {
    "ragged_300": (W["mid_bf16"], dict(T=300, d=256, f=384)),
    "wide_700": (W["mid_bf16"], dict(T=700, d=512, f=256)),
    "skew_1000": (W["grok_skew"], dict(T=1000, d=256, f=256)),
    "no_drop_2500": (W["mid_bf16"], dict(T=2500, d=256, f=640, capacity_factor=float("inf"))),
}


def _both(fn):
    with moe.gemm_tiles("single"):
        a = fn()
        torch.cuda.synchronize()
    with moe.gemm_tiles("pair"):
        b = fn()
        torch.cuda.synchronize()
    return a, b


@pytest.mark.parametrize("name", sorted(CASES))
def test_pair_tiles_match_single_tiles_and_the_oracle(name):
    base, over = CASES[name]
    w = configs.scaled(base, name=f"pair_{name}", **over)
    L = LayerInputs(w)
    D = L.dev
    g1, g2 = _both(lambda: run_steps(L))
    n = int(g2["offsets"][-1])  # grouped rows past the kept ones are never written
    assert np.array_equal(g1["offsets"], g2["offsets"]) and n > 0
    assert torch.equal(g1["h"][:n], g2["h"][:n])
    assert torch.equal(g1["y"][:n], g2["y"][:n])
    assert torch.equal(g1["out"], g2["out"])
    o1, o2 = _both(lambda: moe.layer_forward(L.cfg, D["x"], D["wr"], D["wg"], D["wu"], D["wd"], logit_bias=D["bias"]))
    assert torch.equal(o1, o2)
    ref = oracle.layer_forward(L.x, L.wr, L.wg, L.wu, L.wd, w.capacity_factor, logit_bias=L.bias)
    same = (np.sort(g2["idx"], 1) == np.sort(ref["idx"], 1)).all(1)
    rows = np.nonzero(same)[0]
    check_layer_out(L, g2["out"], g2["y"], g2["slot_of"], ref["out"][rows], rows)
    assert moe.get_device_error() == 0


def test_pair_tiles_training_forward_saves_the_same_state():
    w = configs.scaled(W["mid_bf16"], name="pair_train", T=700, d=256, f=512)
    L = LayerInputs(w)
    c, D = L.cfg, L.dev

    def fwd():
        ws = torch.zeros(moe.workspace_size_train(c), dtype=torch.uint8, device="cuda")
        out = moe.layer_forward_train(c, D["x"], D["wr"], D["wg"], D["wu"], D["wd"], ws, logit_bias=D["bias"])
        return out, ws

    (o1, ws1), (o2, ws2) = _both(fwd)
    assert torch.equal(o1, o2)
    assert torch.equal(ws1, ws2)  # G, U, H, the routing state: byte for byte
    assert moe.get_device_error() == 0


# rows per expert: empty, a single row, tails held by the first CTA alone (64,
# 65, 128), the first tail that reaches the second CTA (129), 255, two blocks + 2
COUNTS = (0, 1, 64, 65, 128, 129, 255, 514)


def test_pair_tiles_every_kind_of_last_block():
    T, d, f = 700, 256, 384
    w = configs.scaled(W["mid_bf16"], name="pair_blocks", T=T, d=d, f=f, capacity_factor=4.0)
    L = LayerInputs(w)
    c, D = L.cfg, L.dev
    n = int(sum(COUNTS))
    assert n <= T * 2
    offsets = np.concatenate([[0], np.cumsum(COUNTS)]).astype(np.int32)
    xs = normal(configs.SEED, 931, (T * 2, d), dtype="bf16")
    x_perm = to_dev(xs)
    off = to_dev(offsets)
    scale = np.linspace(0.25, 1.0, T * 2, dtype=np.float32)
    (h1, y1), (h2, y2) = _both(lambda: moe.expert_ffn(c, x_perm, off, D["wg"], D["wu"], D["wd"], to_dev(scale)))
    assert torch.equal(h1[:n], h2[:n])
    assert torch.equal(y1[:n], y2[:n])
    h = to_np64(h2[:n])
    y = to_np64(y2[:n])
    x64 = oracle.to_f64(xs)
    wg, wu, wd = oracle.to_f64(L.wg), oracle.to_f64(L.wu), oracle.to_f64(L.wd)
    h_ref = np.zeros((n, f))
    y_ref = np.zeros((n, d))
    y_mag = np.zeros((n, d))
    for e in range(8):
        a, b = offsets[e], offsets[e + 1]
        if b > a:
            h_ref[a:b] = oracle.swiglu_hidden(x64[a:b], wg[e], wu[e])
            y_ref[a:b] = scale[a:b, None] * oracle.swiglu_expert(x64[a:b], wg[e], wu[e], wd[e])
            y_mag[a:b] = scale[a:b, None] * (np.abs(h_ref[a:b]) @ np.abs(wd[e]))
    # H is rounded once to bf16 (unit roundoff 2^-8: 8 significant bits) after
    # an fp32 sum over d = 256 products; Y sums those rounded H values against
    # W_down in fp32, so its error is at most 2^-8 sum_k |h_k w_k| plus the fp32
    # sum's.  Bars: twice the rounding bound, plus a floor for the fp32 sums.
    h_rms = float(np.sqrt(np.mean(h_ref ** 2)))
    assert np.all(np.abs(h - h_ref) <= 2.0 ** -7 * np.abs(h_ref) + 1e-4 * h_rms)
    y_rms = float(np.sqrt(np.mean(y_ref ** 2)))
    assert np.all(np.abs(y - y_ref) <= 2.0 ** -7 * y_mag + 1e-5 * y_rms)
    assert moe.get_device_error() == 0
