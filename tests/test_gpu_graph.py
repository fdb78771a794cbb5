"""The layer's launches captured in a CUDA graph and replayed: the replay gives
the eager call's output bit for bit, also after new input is copied into the
captured buffer (the way a serving loop reuses a graph)."""
from __future__ import annotations

import pytest
import torch

import sparse_moe_layer_07_b200 as moe
from synth import configs

from parity_util import LayerInputs, to_dev

pytestmark = pytest.mark.gpu

W = configs.WORKLOADS


@pytest.mark.parametrize("T,cf", [(32, 4.0), (700, 1.25)])
def test_layer_replays_from_a_cuda_graph(T, cf):
    w = configs.scaled(W["mid_bf16"], name=f"graph_{T}", T=T, d=256, f=384, capacity_factor=cf)
    L = LayerInputs(w)
    D, c = L.dev, L.cfg
    x2 = to_dev(configs.make_x(w, call=7))
    eager1 = moe.layer_forward(c, D["x"], D["wr"], D["wg"], D["wu"], D["wd"])
    eager2 = moe.layer_forward(c, x2, D["wr"], D["wg"], D["wu"], D["wd"])
    x_in = D["x"].clone()
    out = torch.empty_like(eager1)
    ws = torch.empty(moe.workspace_size(c), dtype=torch.uint8, device="cuda")
    cap = torch.cuda.Stream()
    cap.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(cap):
        moe.layer_forward(c, x_in, D["wr"], D["wg"], D["wu"], D["wd"], out=out, ws=ws)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=cap, capture_error_mode="relaxed"):
        moe.layer_forward(c, x_in, D["wr"], D["wg"], D["wu"], D["wd"], out=out, ws=ws)
    out.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, eager1)
    x_in.copy_(x2)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, eager2)
    assert moe.get_device_error() == 0
