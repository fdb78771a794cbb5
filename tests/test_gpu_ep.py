"""Expert parallelism on one GPU: `world` virtual ranks run the phases of
layer_forward_ep in lockstep, and the two all-to-alls are done in-process by
slicing (no collective; the GPU kernels involved never wait on each other).
Every rank's output is checked against the oracle on that rank's batch, with
the bf16 bar of the single-GPU layer."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import sparse_moe_layer_07_b200 as moe
from sparse_moe_layer_07_b200.expert_parallel import ep_experts, ep_finish, ep_plan, ep_prepare
from synth import configs, normal

from parity_util import LayerInputs, to_dev

pytestmark = pytest.mark.gpu

W = configs.WORKLOADS


def _splits_start(splits):
    return np.concatenate([[0], np.cumsum(splits)[:-1]]).astype(np.int64)


@pytest.mark.parametrize("world,skew", [(2, False), (4, False), (4, True), (8, True)])
def test_expert_parallel_ranks_match_the_oracle(world, skew):
    base = W["grok_skew"] if skew else W["mid_bf16"]
    w = configs.scaled(base, name=f"ep{world}", T=300, d=256, f=384, capacity_factor=1.25)
    L0 = LayerInputs(w)  # weights (shared by all ranks) and rank 0's batch
    xs = [L0.x] + [normal(configs.SEED, configs.TID_X + 1000 * r, (w.T, w.d), dtype="bf16") for r in range(1, world)]
    D = L0.dev
    cfg = L0.cfg
    states = [ep_prepare(cfg, to_dev(x), D["wr"], D["bias"]) for x in xs]
    table = np.stack([st["counts"].cpu().numpy() for st in states])
    plans = [ep_plan(table, r, world) for r in range(world)]
    # all-to-all 1: rank q gets, from every rank p, p's x_perm slice for q's experts
    x_recv = []
    for q in range(world):
        parts = []
        for p in range(world):
            s0 = _splits_start(plans[p]["send_splits"])[q]
            parts.append(states[p]["disp"]["x_perm"][s0:s0 + plans[p]["send_splits"][q]])
        x_recv.append(torch.cat(parts))
    y_recv = [ep_experts(cfg, x_recv[q], plans[q], D["wg"], D["wu"], D["wd"]) for q in range(world)]
    # all-to-all 2: rank p gets back, from every rank q, the outputs of the rows it sent
    outs = []
    for p in range(world):
        parts = []
        for q in range(world):
            s0 = _splits_start(plans[q]["recv_splits"])[p]
            parts.append(y_recv[q][s0:s0 + plans[q]["recv_splits"][p]])
        outs.append(ep_finish(cfg, torch.cat(parts), states[p]))
    torch.cuda.synchronize()
    if skew:
        # expert 0's owner receives more rows than its own batch would hold
        assert max(int(pl["offsets"][-1]) for pl in plans) > w.T * 2
    for r in range(world):
        ref = oracle.layer_forward(xs[r], L0.wr, L0.wg, L0.wu, L0.wd, w.capacity_factor, logit_bias=L0.bias)
        slot_of = states[r]["disp"]["slot_of"]
        kept = slot_of.cpu().numpy() >= 0
        assert np.array_equal(kept, ref["slot_of"] >= 0)
        # the combine's fp32 value before rounding: the same kernel with an fp32 output
        cfg32 = moe.Config(w.T, w.d, w.f, capacity_factor=w.capacity_factor, dtype="f32")
        parts = []
        for q in range(world):
            s0 = _splits_start(plans[q]["recv_splits"])[r]
            parts.append(y_recv[q][s0:s0 + plans[q]["recv_splits"][r]])
        pre = moe.combine(cfg32, torch.cat(parts), slot_of, states[r]["w"], weights_applied=False)
        torch.cuda.synchronize()
        pre = pre.cpu().numpy().astype(np.float64)
        rows = kept.any(1)
        rms = float(np.sqrt(np.mean(ref["out"][rows] ** 2)))
        assert np.max(np.abs(pre[rows] - ref["out"][rows])) <= 2e-2 * rms
        assert np.all(pre[~rows] == 0) and np.all(ref["out"][~rows] == 0)
        import synth

        rounded = oracle.to_f64(synth.round_bf16(pre).reshape(pre.shape))
        assert np.array_equal(outs[r].float().cpu().numpy().astype(np.float64), rounded)
    assert moe.get_device_error() == 0
