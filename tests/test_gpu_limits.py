"""Size limits and degenerate batches through the C ABI.

- a large batch (T = 2^22 tokens: 8.4M grouped rows, past what 16-bit or
  naive 32-bit products of row x width would hold in several buffers) with the
  routing and dispatch checked over every token and the output on a sample;
- one and two tokens (the weight-streaming path with a single MMA column);
- the smallest widths the tensor-core path accepts (d = f = 128, bf16).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import sparse_moe_layer_07_b200 as moe
from synth import configs

from parity_util import LayerInputs, check_dispatch, check_layer_out, check_routing, run_steps

pytestmark = pytest.mark.gpu

W = configs.WORKLOADS


def test_large_batch_four_million_tokens():
    w = configs.scaled(W["mid_bf16"], name="large_T", T=1 << 22, d=128, f=256, capacity_factor=1.25)
    L = LayerInputs(w)
    g = run_steps(L, keep_h=False)
    logits = oracle.router_logits(L.x, L.wr)
    tie, mismatch = check_routing(L, g, logits)
    assert mismatch.sum() <= tie.sum()
    check_dispatch(L, g)
    rng = np.random.default_rng(3)
    tokens = np.sort(rng.choice(w.T, size=48, replace=False))
    tokens = np.unique(np.concatenate([tokens, [0, w.T - 1]]))
    ref = oracle.layer_forward(L.x, L.wr, L.wg, L.wu, L.wd, w.capacity_factor, tokens=tokens)
    same = (np.sort(g["idx"][tokens], 1) == np.sort(ref["idx"][tokens], 1)).all(1)
    check_layer_out(L, g["out"], g["y"], g["slot_of"], ref["out"][same], tokens[same])
    out = moe.layer_forward(L.cfg, L.dev["x"], L.dev["wr"], L.dev["wg"], L.dev["wu"], L.dev["wd"])
    torch.cuda.synchronize()
    assert torch.equal(out, g["out"])
    assert moe.get_device_error() == 0


@pytest.mark.parametrize("T", [1, 2, 3])
def test_one_to_three_tokens(T):
    w = configs.scaled(W["mid_bf16"], name=f"tokens_{T}", T=T, d=256, f=384, capacity_factor=4.0)
    L = LayerInputs(w)
    g = run_steps(L)
    check_routing(L, g, oracle.router_logits(L.x, L.wr))
    check_dispatch(L, g)
    ref = oracle.layer_forward(L.x, L.wr, L.wg, L.wu, L.wd, w.capacity_factor)
    check_layer_out(L, g["out"], g["y"], g["slot_of"], ref["out"], np.arange(T))
    out = moe.layer_forward(L.cfg, L.dev["x"], L.dev["wr"], L.dev["wg"], L.dev["wu"], L.dev["wd"])
    torch.cuda.synchronize()
    assert torch.equal(out, g["out"])


@pytest.mark.parametrize("T", [40, 700])
def test_smallest_widths(T):
    # d = f = 128: one N block for gate/up, the 128-column down kernel (d % 256 != 0)
    w = configs.scaled(W["mid_bf16"], name=f"narrow_{T}", T=T, d=128, f=128, capacity_factor=1.25)
    L = LayerInputs(w)
    g = run_steps(L)
    check_routing(L, g, oracle.router_logits(L.x, L.wr))
    check_dispatch(L, g)
    ref = oracle.layer_forward(L.x, L.wr, L.wg, L.wu, L.wd, w.capacity_factor)
    check_layer_out(L, g["out"], g["y"], g["slot_of"], ref["out"], np.arange(T))
    assert moe.get_device_error() == 0
