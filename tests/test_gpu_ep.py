"""Expert parallelism on one GPU: `world` virtual ranks run the phases of
layer_forward_ep in lockstep, and the two all-to-alls are done in-process by
slicing (no collective; the GPU kernels involved never wait on each other).
Every rank's output is checked against the oracle on that rank's batch, with
the bf16 bar of the single-GPU layer.  Then layer_forward_ep itself runs end
to end in two processes that share the GPU, exchanging over gloo through host
memory (only the host-side collectives wait on the other rank): each rank's
output must equal the virtual ranks' bit for bit."""
from __future__ import annotations

import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

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


def _free_port():
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def _ep_case(world):
    return configs.scaled(W["grok_skew"], name=f"ep_e2e{world}", T=300, d=256, f=384, capacity_factor=1.25)


def _ep_batch(w, rank):
    return configs.make_x(w) if rank == 0 else normal(configs.SEED, configs.TID_X + 1000 * rank, (w.T, w.d),
                                                        dtype="bf16")


def _ep_worker(rank, world, port, q):
    import sys
    from datetime import timedelta

    import torch.distributed as dist

    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    from sparse_moe_layer_07_b200.expert_parallel import layer_forward_ep

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=timedelta(seconds=120))
    try:
        torch.cuda.set_device(0)
        w = _ep_case(world)
        L = LayerInputs(w, x=_ep_batch(w, rank))
        D = L.dev
        out = layer_forward_ep(L.cfg, D["x"], D["wr"], D["wg"], D["wu"], D["wd"], logit_bias=D["bias"])
        torch.cuda.synchronize()
        q.put((rank, out.view(torch.int16).cpu().numpy(), moe.get_device_error()))
    finally:
        dist.destroy_process_group()


def test_layer_forward_ep_end_to_end_two_processes():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_ep_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = {}
    try:
        for _ in range(world):
            r, out, err = q.get(timeout=300)
            got[r] = (out, err)
    finally:
        for p in procs:
            p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    # the same ranks in lockstep in this process, exchanges by slicing
    w = _ep_case(world)
    L0 = LayerInputs(w)
    D, cfg = L0.dev, L0.cfg
    states = [ep_prepare(cfg, to_dev(_ep_batch(w, r)), D["wr"], D["bias"]) for r in range(world)]
    table = np.stack([st["counts"].cpu().numpy() for st in states])
    plans = [ep_plan(table, r, world) for r in range(world)]
    x_recv = [torch.cat([states[p]["disp"]["x_perm"][_splits_start(plans[p]["send_splits"])[q_]:][
        :plans[p]["send_splits"][q_]] for p in range(world)]) for q_ in range(world)]
    y_recv = [ep_experts(cfg, x_recv[q_], plans[q_], D["wg"], D["wu"], D["wd"]) for q_ in range(world)]
    for r in range(world):
        back = torch.cat([y_recv[q_][_splits_start(plans[q_]["recv_splits"])[r]:][:plans[q_]["recv_splits"][r]]
                          for q_ in range(world)])
        want = ep_finish(cfg, back, states[r]).view(torch.int16).cpu().numpy()
        out, err = got[r]
        assert err == 0
        assert np.array_equal(out, want), r
