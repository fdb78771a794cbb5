"""Token shards under the global capacity rule on one GPU: the shards of one
batch run one after another (no collective; the table of every shard's route
counts is stacked directly), and the concatenated result must equal the
unsharded layer bit for bit, with the same keep mask as the oracle's global
dispatch."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import sparse_moe_layer_07_b200 as moe
from sparse_moe_layer_07_b200.sharded import layer_forward_shard
from synth import configs

from parity_util import LayerInputs

pytestmark = pytest.mark.gpu

W = configs.WORKLOADS

CASES = {
    # skewed router, cf 1.0: expert 0 overflows, so later shards lose assignments
    "shard_skew_drop": (W["grok_skew"], dict(T=1000, d=256, f=384, capacity_factor=1.0), (300, 400, 300)),
    # every shard above the weight-streaming size, so shards and batch run the same kernels
    "shard_uneven": (W["mid_bf16"], dict(T=1100, d=256, f=256, capacity_factor=0.9), (257, 586, 257)),
    "shard_fp32": (W["tiny_f32"], dict(T=640, d=128, f=192, capacity_factor=1.0), (200, 440)),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_shards_equal_the_whole_batch(name):
    base, over, sizes = CASES[name]
    w = configs.scaled(base, name=name, **over)
    L = LayerInputs(w)
    D = L.dev
    cfg = L.cfg
    whole = moe.layer_forward(cfg, D["x"], D["wr"], D["wg"], D["wu"], D["wd"], logit_bias=D["bias"])
    bounds = np.cumsum((0,) + sizes)
    assert bounds[-1] == w.T
    cfgs = [moe.Config(int(n), w.d, w.f, capacity_factor=w.capacity_factor, dtype=w.storage) for n in sizes]
    xs = [D["x"][bounds[i]:bounds[i + 1]].contiguous() for i in range(len(sizes))]
    # the table a rank would all-gather: every shard's route counts, in shard order
    counts = []
    for c, x in zip(cfgs, xs):
        idx, _, _ = moe.router_topk(c, x, D["wr"], D["bias"])
        counts.append(moe.route_counts(c, idx))
    table = torch.stack(counts)
    outs, kept = [], []
    for i, (c, x) in enumerate(zip(cfgs, xs)):
        out, disp = layer_forward_shard(c, w.T, lambda _counts: table, i, x, D["wr"], D["wg"], D["wu"], D["wd"],
                                        logit_bias=D["bias"])
        outs.append(out)
        kept.append(disp["slot_of"].cpu().numpy() >= 0)
    torch.cuda.synchronize()
    ref = oracle.layer_forward(L.x, L.wr, L.wg, L.wu, L.wd, w.capacity_factor, logit_bias=L.bias, tokens=[0])
    assert ref["dropped"] > 0
    assert np.array_equal(np.concatenate(kept), ref["slot_of"] >= 0)
    assert torch.equal(torch.cat(outs), whole)
    assert moe.get_device_error() == 0
