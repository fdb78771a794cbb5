"""moe_dispatch_noalloc, the dispatch entry point for callers that cannot
allocate device memory (plug-ins hosted by a runtime that owns all device
memory and gives them no workspace, latency-critical loops that cannot afford
cudaMalloc's synchronisation).  Its scratch is a fixed array inside the
library, shared by every call, so this file checks it against the regular
moe_dispatch (caller workspace) on two calls in a row: the second, smaller call
runs over the stale contents the first one left behind.  Dispatch outputs are
integer and index data, so the comparison is bit-exact.  This file is collected
last so that a failure here cannot hide the other tests' results.
"""
import numpy as np
import pytest
import torch

import sparse_moe_layer_07_b200 as moe
from synth import configs

pytestmark = pytest.mark.gpu


def _routed(T, call):
    w = configs.scaled(configs.WORKLOADS["mid_bf16"], name="noalloc", T=T, d=256, f=384)
    x = torch.from_numpy(configs.make_x(w, call) if call == 0 else
                         configs.normal(configs.SEED, 900 + call, (T, 256), dtype="bf16")).view(torch.bfloat16)
    wr = torch.from_numpy(configs.make_router(w)).view(torch.bfloat16)
    x, wr = x.cuda(), wr.cuda()
    cfg = moe.Config(T, 256, 384, capacity_factor=1.25, dtype="bf16")
    idx, wts, _ = moe.router_topk(cfg, x, wr)
    return cfg, x, idx, wts


@pytest.mark.parametrize("T,call", [(3000, 0), (777, 1)])
def test_noalloc_dispatch_matches_dispatch(T, call):
    cfg, x, idx, wts = _routed(T, call)
    ref = moe.dispatch(cfg, x, idx, wts)
    got = moe.dispatch_noalloc(cfg, x, idx, wts)
    torch.cuda.synchronize()
    for k in ("counts_raw", "counts_kept", "offsets", "slot_of"):
        assert torch.equal(got[k], ref[k]), k
    n = int(ref["offsets"][-1])
    assert n > 0 and int(ref["counts_raw"].sum()) == 2 * T
    assert torch.equal(got["perm"][:n], ref["perm"][:n])
    assert torch.equal(got["row_scale"][:n], ref["row_scale"][:n])
    assert torch.equal(got["x_perm"][:n], ref["x_perm"][:n])
    assert moe.get_device_error() == 0


def test_noalloc_dispatch_at_the_size_limit():
    # T = MOE_NOALLOC_MAX_TOKENS: the last histogram block's entries reach the end
    # of the fixed array; one more token is refused before any launch
    T, d = moe.NOALLOC_MAX_TOKENS, 128
    x = torch.from_numpy(configs.normal(configs.SEED, 950, (T, d), dtype="bf16")).view(torch.bfloat16).cuda()
    wr = torch.from_numpy(configs.normal(configs.SEED, 951, (8, d), std=0.02, dtype="bf16")).view(torch.bfloat16)
    cfg = moe.Config(T, d, 128, capacity_factor=1.0, dtype="bf16")
    idx, wts, _ = moe.router_topk(cfg, x, wr.cuda())
    ref = moe.dispatch(cfg, x, idx, wts, gather=False)
    got = moe.dispatch_noalloc(cfg, x, idx, wts, gather=False)
    torch.cuda.synchronize()
    for k in ("counts_raw", "counts_kept", "offsets", "slot_of"):
        assert torch.equal(got[k], ref[k]), k
    n = int(ref["offsets"][-1])
    assert int(ref["counts_raw"].sum()) == 2 * T and n < 2 * T  # cf 1.0: the fuller experts drop some
    assert torch.equal(got["perm"][:n], ref["perm"][:n])
    assert torch.equal(got["row_scale"][:n], ref["row_scale"][:n])
    assert moe.get_device_error() == 0
    big = moe.Config(T + 1, d, 128, capacity_factor=1.0, dtype="bf16")
    with pytest.raises(RuntimeError, match="MOE_ERR_UNSUPPORTED"):
        moe.dispatch_noalloc(big, x, idx, wts, gather=False)
