"""Parity of the CUDA path (through the C ABI) with the fp64 CPU oracle.

Small and mid layers are compared element by element on every intermediate
(logits, indices, weights, counts, permutation, slot map, gathered rows, hidden
activation, expert outputs, layer output).  Sizes span several 128-row tiles,
ragged expert tails, both down-projection tile widths, capacity drops and the
no-drop case.
"""
import numpy as np
import pytest
import torch

import oracle
import sparse_moe_layer_07_b200 as moe
from synth import configs

from parity_util import (LayerInputs, check_dispatch, check_layer_out, check_out_rows, check_routing,
                         run_steps, to_dev, to_np64)

pytestmark = pytest.mark.gpu

W = configs.WORKLOADS

SMALL = {
    # name: (base workload, overrides)
    "tiny_f32": (W["tiny_f32"], {}),
    "f32_ragged": (W["tiny_f32"], dict(T=333, d=192, f=320, capacity_factor=1.1)),
    "bf16_tiles_ragged": (W["mid_bf16"], dict(T=700, d=256, f=384)),
    "bf16_down_n128": (W["mid_bf16"], dict(T=300, d=384, f=256, capacity_factor=2.0)),
    "bf16_no_drop": (W["mid_bf16"], dict(T=513, d=512, f=640, capacity_factor=4.0)),
    "bf16_skew_drop": (W["grok_skew"], dict(T=1024, d=256, f=512)),
    "bf16_pair_ragged": (W["mid_bf16"], dict(T=1500, d=512, f=768)),
    # enough down tiles for the 256-column down pass (smaller batches take 128-column tiles)
    "bf16_down_wide": (W["mid_bf16"], dict(T=4608, d=1024, f=256, capacity_factor=4.0)),
    # at most 64 rows per expert on average: the weight-streaming (swap-AB) kernel
    "bf16_stream_no_drop": (W["mid_bf16"], dict(T=96, d=256, f=384, capacity_factor=4.0)),
    "bf16_stream_ragged": (W["mid_bf16"], dict(T=250, d=384, f=512)),
    "mid_bf16": (W["mid_bf16"], {}),
}


def _workload(name):
    base, over = SMALL[name]
    return configs.scaled(base, name=name, **over) if over else base


@pytest.fixture(scope="module", params=sorted(SMALL))
def case(request):
    w = _workload(request.param)
    L = LayerInputs(w)
    g = run_steps(L)
    ref = oracle.layer_forward(L.x, L.wr, L.wg, L.wu, L.wd, w.capacity_factor, logit_bias=L.bias,
                               keep_hidden=True)
    return L, g, ref


def test_routing(case):
    L, g, ref = case
    tie, mismatch = check_routing(L, g, ref["logits"])
    assert mismatch.sum() <= tie.sum()


def test_dispatch_bit_exact(case):
    L, g, ref = case
    check_dispatch(L, g)
    if (np.sort(g["idx"], 1) == np.sort(ref["idx"], 1)).all():
        np.testing.assert_array_equal(g["counts_kept"], ref["counts_kept"])
        np.testing.assert_array_equal(g["offsets"], ref["offsets"])


def test_gather_bit_exact(case):
    L, g, ref = case
    n = int(g["offsets"][-1])
    xp = g["x_perm"][:n].cpu()
    x = torch.from_numpy(np.ascontiguousarray(L.x))
    if L.w.storage == "bf16":
        x = x.view(torch.bfloat16)
    assert torch.equal(xp, x[torch.from_numpy(g["perm"][:n]).long()])


def test_hidden_and_expert_outputs(case):
    L, g, ref = case
    if not (g["idx"] == ref["idx"]).all():
        pytest.skip("routing differs on a near tie; per-slot comparison not defined")
    n = ref["n_kept"]
    h = to_np64(g["h"][:n])
    href = np.stack([ref["hidden"][s] for s in range(n)])
    rms_h = float(np.sqrt(np.mean(href ** 2)))
    if L.w.storage == "bf16":
        # one bf16 rounding of H (half an ulp = 2^-9 relative) plus fp32 accumulation slack
        assert np.all(np.abs(h - href) <= 2.0 ** -8 * np.abs(href) + 1e-3 * rms_h)
    else:
        assert np.all(np.abs(h - href) <= 1e-5 * np.abs(href) + 1e-5 * rms_h)
    y = to_np64(g["y"][:n])
    yref = np.zeros((n, L.w.d))
    for e in range(8):
        lo, hi = int(ref["offsets"][e]), int(ref["offsets"][e + 1])
        if hi > lo:
            yref[lo:hi] = ref["row_scale"][lo:hi, None] * (href[lo:hi] @ oracle.to_f64(L.wd[e]))
    check_out_rows(L, y, yref, L.w.storage)


def test_layer_output(case):
    L, g, ref = case
    got = to_np64(g["out"])
    same_route = (np.sort(g["idx"], 1) == np.sort(ref["idx"], 1)).all(1)
    same_keep = ((g["slot_of"] >= 0) == (ref["slot_of"] >= 0)).all(1) | ~same_route
    rows = np.nonzero(same_route & same_keep)[0]
    check_layer_out(L, g["out"], g["y"], g["slot_of"], ref["out"][rows], rows)
    # tokens whose assignments were all dropped output exactly zero
    dropped = (g["slot_of"] < 0).all(axis=1)
    assert np.all(got[dropped] == 0.0)


def test_layer_forward_equals_steps(case):
    L, g, ref = case
    D = L.dev
    stats = torch.zeros(3 * 8 + 2, dtype=torch.int32, device="cuda")
    out = moe.layer_forward(L.cfg, D["x"], D["wr"], D["wg"], D["wu"], D["wd"], logit_bias=D["bias"], stats=stats)
    torch.cuda.synchronize()
    assert torch.equal(out, g["out"])
    s = stats.cpu().numpy()
    np.testing.assert_array_equal(s[:8], g["counts_raw"])
    np.testing.assert_array_equal(s[8:16], g["counts_kept"])
    np.testing.assert_array_equal(s[16:25], g["offsets"])
    assert s[25] == L.w.T * 2 - int(g["offsets"][-1])
    assert moe.get_device_error() == 0


def _fused(c):
    return c.dtype == "bf16" and c.T * 2 > 64 * 8 and c.d % 256 == 0


def test_down_combine_equals_down_then_combine(case):
    # down summed into token order == down then combine, bit for bit
    L, g, ref = case
    c, D = L.cfg, L.dev
    if not _fused(c):
        pytest.skip("the fused down-combine covers bf16 tensor-core batches with d % 256 == 0")
    perm = torch.from_numpy(g["perm"]).cuda()
    offsets = torch.from_numpy(g["offsets"]).cuda()
    row_scale = torch.from_numpy(g["row_scale"]).cuda()
    out = moe.expert_down_combine(c, g["h"], offsets, D["wd"], row_scale, perm)
    torch.cuda.synchronize()
    assert torch.equal(out, g["out"])
    assert moe.get_device_error() == 0


def test_deterministic(case):
    L, g, ref = case
    g2 = run_steps(L)
    assert torch.equal(g2["out"], g["out"])
    n = int(g["offsets"][-1])  # perm is defined for the kept rows only
    assert np.array_equal(g2["perm"][:n], g["perm"][:n])


def test_host_buffer_entry_point(case):
    L, g, ref = case
    c, D = L.cfg, L.dev
    x_host = D["x"].cpu().pin_memory()
    out_host = torch.empty((c.T, c.d), dtype=c.torch_dtype).pin_memory()
    ws = torch.empty(moe.workspace_size(c), dtype=torch.uint8, device="cuda")
    moe.layer_forward_host(c, x_host, D["wr"], D["wg"], D["wu"], D["wd"], out_host, ws, logit_bias=D["bias"])
    assert torch.equal(out_host, g["out"].cpu())


def test_host_batches_entry_point(case):
    # several host batches through the copy/compute pipeline: each equals the
    # device-buffer layer on the same x, bit for bit (5 batches cycle both slots)
    L, g, ref = case
    c, D = L.cfg, L.dev
    xs = [configs.make_x(L.w, call) for call in range(3)]
    x_hosts = [to_dev(a, "cpu").pin_memory() for a in xs] + [to_dev(xs[0], "cpu").pin_memory()] * 2
    out_hosts = [torch.full((c.T, c.d), 7.0, dtype=c.torch_dtype).pin_memory() for _ in range(4)]
    out_hosts.append(out_hosts[0])  # a repeated buffer ends with the last batch written to it
    ws = torch.empty(moe.workspace_size_host_batches(c), dtype=torch.uint8, device="cuda")
    moe.layer_forward_host_batches(c, x_hosts, D["wr"], D["wg"], D["wu"], D["wd"], out_hosts, ws,
                                   logit_bias=D["bias"])
    for i, xh in enumerate(x_hosts):
        want = moe.layer_forward(c, xh.cuda(), D["wr"], D["wg"], D["wu"], D["wd"], logit_bias=D["bias"]).cpu()
        if i == 0:
            continue  # out_hosts[0] was overwritten by batch 4 (same x), checked below
        assert torch.equal(out_hosts[i], want), i
    assert torch.equal(out_hosts[0], g["out"].cpu())
    assert moe.get_device_error() == 0


# ---------------------------------------------------------------------------- edge cases
def test_empty_batch():
    c = moe.Config(0, 256, 384, dtype="bf16")
    z = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    out = moe.layer_forward(c, z, torch.zeros(8 * 256, dtype=torch.bfloat16, device="cuda"), z, z, z,
                            ws=torch.zeros(16, dtype=torch.uint8, device="cuda"))
    assert out.numel() == 0


def test_all_tokens_to_two_experts_drop_and_zero():
    # router rigged so that every token picks experts (0, 1); capacity keeps the first `cap` tokens
    w = configs.scaled(W["mid_bf16"], name="rigged", T=256, d=256, f=384, capacity_factor=0.5,
                       logit_bias=(60.0, 50.0, 0, 0, 0, 0, 0, 0))
    L = LayerInputs(w)
    g = run_steps(L)
    cap = oracle.capacity(256, 2, 8, 0.5)
    assert (g["idx"] == np.array([0, 1])).all()
    assert list(g["counts_kept"]) == [cap, cap, 0, 0, 0, 0, 0, 0]
    assert (g["slot_of"][cap:] == -1).all()
    assert np.all(to_np64(g["out"])[cap:] == 0.0)
    ref = oracle.layer_forward(L.x, L.wr, L.wg, L.wu, L.wd, w.capacity_factor, logit_bias=L.bias)
    check_layer_out(L, g["out"], g["y"], g["slot_of"], ref["out"], np.arange(256))


def test_bounded_wait_gives_up_and_the_context_stays_usable():
    # an mbarrier nothing completes: the wait gives up after 50 ms and reports it
    moe.get_device_error(clear=True)
    st = moe.lib.moe_check_bounded_wait(50_000_000, None)
    assert st == 0
    torch.cuda.synchronize()
    assert moe.get_device_error(clear=True) & moe.DEVERR["TIMEOUT"]
    w = configs.scaled(W["mid_bf16"], name="after_timeout", T=300, d=256, f=384)
    L = LayerInputs(w)
    g = run_steps(L)
    ref = oracle.layer_forward(L.x, L.wr, L.wg, L.wu, L.wd, w.capacity_factor)
    check_layer_out(L, g["out"], g["y"], g["slot_of"], ref["out"], np.arange(w.T))
    assert moe.get_device_error() == 0


def test_bad_expert_index_sets_device_error_without_trap():
    c = moe.Config(64, 256, 384, dtype="bf16")
    idx = torch.zeros((64, 2), dtype=torch.int32, device="cuda")
    idx[:, 1] = 1
    idx[5, 0] = 9  # out of range
    wts = torch.full((64, 2), 0.5, device="cuda")
    moe.get_device_error(clear=True)
    d = moe.dispatch(c, None, idx, wts, gather=False)
    torch.cuda.synchronize()
    code = moe.get_device_error(clear=True)
    assert code & moe.DEVERR["EXPERT_INDEX"]
    assert d["counts_raw"].cpu().tolist() == [63, 64, 0, 0, 0, 0, 0, 0]
    assert moe.get_device_error() == 0


def test_bad_slot_in_combine_sets_device_error():
    c = moe.Config(8, 256, 384, dtype="bf16")
    y = torch.ones((16, 256), device="cuda")
    slot = torch.full((8, 2), -1, dtype=torch.int32, device="cuda")
    slot[0, 0] = 3
    slot[1, 0] = 1000  # beyond the buffer
    out = moe.combine(c, y, slot)
    torch.cuda.synchronize()
    assert moe.get_device_error(clear=True) & moe.DEVERR["SLOT_INDEX"]
    o = out.float().cpu()
    assert torch.all(o[0] == 1) and torch.all(o[1] == 0)


def test_expert_utilization_over_calls():
    # counts over several calls, normalised as the oracle's statistic (1.0 when balanced)
    w = configs.scaled(W["grok_skew"], name="util", T=512, d=256, f=384)
    L = LayerInputs(w)
    D = L.dev
    tracker = moe.ExpertUtilization()
    idx_all = []
    for call in range(4):
        x = configs.make_x(w, call)
        stats = torch.zeros(26, dtype=torch.int32, device="cuda")
        moe.layer_forward(L.cfg, to_dev(x), D["wr"], D["wg"], D["wu"], D["wd"], logit_bias=D["bias"], stats=stats)
        tracker.add(stats)
        idx_all.append(oracle.top2_softmax(oracle.router_logits(x, L.wr, L.bias))[0])
    torch.cuda.synchronize()
    counts = np.bincount(np.concatenate(idx_all).ravel(), minlength=8)
    want = oracle.expert_utilization(counts)
    np.testing.assert_allclose(tracker.utilization(), want, rtol=0, atol=2 * 8 / counts.sum())
    assert tracker.utilization()[0] > 1.5  # the biased expert


def test_router_does_not_depend_on_the_batch():
    """A token's logits, experts and weights are the same bits whatever batch it
    arrives in: the router sums four fixed hidden-dimension quarters in a fixed
    order, and only the number of CTAs sharing a tile changes with the batch
    size (one, two or four here); also against the oracle's fp32 bound."""
    w = configs.scaled(W["grok_skew"], name="router_batches", T=20000, d=512, f=256)
    L = LayerInputs(w)
    c = L.cfg
    idx, wts, lg = moe.router_topk(c, L.dev["x"], L.dev["wr"], L.dev["bias"], want_logits=True)
    g = {"idx": idx.cpu().numpy(), "w": wts.cpu().numpy(), "logits": lg.cpu().numpy().astype(np.float64)}
    check_routing(L, g, oracle.router_logits(L.x, L.wr, L.bias))
    for t0, n in ((0, 8192), (8192, 1000), (9192, 40), (19999, 1), (5000, 8000)):
        cs = moe.Config(n, w.d, w.f, capacity_factor=w.capacity_factor, dtype="bf16")
        xs = L.dev["x"][t0:t0 + n].contiguous()
        i2, w2, l2 = moe.router_topk(cs, xs, L.dev["wr"], L.dev["bias"], want_logits=True)
        torch.cuda.synchronize()
        assert torch.equal(l2, lg[t0:t0 + n]), (t0, n)
        assert torch.equal(i2, idx[t0:t0 + n]) and torch.equal(w2, wts[t0:t0 + n]), (t0, n)
    assert moe.get_device_error() == 0


@pytest.mark.parametrize("d", [128, 384, 640, 896])
def test_router_uneven_quarters(d):
    """Hidden sizes of 2, 6, 10 and 14 K blocks of 64: quarters that are empty
    or of unequal length, CTAs with an odd number of blocks (their last
    two-block box runs into the next CTA's range), one, two or four CTAs per
    tile (1 to 20000 tokens); against the oracle's fp32 bound and top-2."""
    for T in (1, 63, 65, 3000, 8192, 20000):
        w = configs.scaled(W["grok_skew"], name=f"router_d{d}_T{T}", T=T, d=d, f=128)
        L = LayerInputs(w)
        idx, wts, lg = moe.router_topk(L.cfg, L.dev["x"], L.dev["wr"], L.dev["bias"], want_logits=True)
        torch.cuda.synchronize()
        g = {"idx": idx.cpu().numpy(), "w": wts.cpu().numpy(), "logits": lg.cpu().numpy().astype(np.float64)}
        tie, mismatch = check_routing(L, g, oracle.router_logits(L.x, L.wr, L.bias))
        assert mismatch.sum() <= tie.sum()
    assert moe.get_device_error() == 0
