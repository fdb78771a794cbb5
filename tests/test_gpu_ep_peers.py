"""Expert parallelism over peer memory ("Expert parallelism vs. tensor
parallelism", moe_layer_ep_forward), on one GPU.

`world` ranks held by one process run the peer-memory kernels (dispatch
stores into the owners' grouped buffers, the owners' down kernels add into the
sources' sums); the stream order stands in for the barriers, and no kernel
waits on another.  Every rank's output must equal the single-device layer on
that rank's tokens bit for bit (each row's products and its two-term fp32 sum
do not depend on the rows it shares a tile with), and rank 0's must meet the
oracle's bf16 bar.  The grouped buffers are checked entry by entry against
the placement rule computed on the host.  Then two processes that share the
GPU map each other's buffers through CUDA IPC and run layer_forward_ep_peers
with host barriers (gloo)."""
from __future__ import annotations

import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
import sparse_moe_layer_07_b200 as moe
import synth
from sparse_moe_layer_07_b200.expert_parallel import EpPeerBuffers, ep_forward_peers_local, ep_route, owned_experts
from synth import configs, normal

from parity_util import LayerInputs, to_dev

pytestmark = pytest.mark.gpu

W = configs.WORKLOADS


def _case(world, skew, T=512):
    base = W["grok_skew"] if skew else W["mid_bf16"]
    return configs.scaled(base, name=f"ep_peers{world}", T=T, d=256, f=384, capacity_factor=1.25)


def _batch(w, rank):
    return configs.make_x(w) if rank == 0 else normal(configs.SEED, configs.TID_X + 1000 * rank, (w.T, w.d),
                                                        dtype="bf16")


def _bits(t):
    return t.view(torch.int16).cpu().numpy()


@pytest.mark.parametrize("world,skew", [(1, False), (2, False), (4, False), (4, True), (8, True)])
def test_peer_ranks_equal_the_single_device_layer(world, skew):
    w = _case(world, skew)
    L0 = LayerInputs(w)
    D, cfg = L0.dev, L0.cfg
    xs_host = [_batch(w, r) for r in range(world)]
    xs = [to_dev(x) for x in xs_host]
    bufs = [EpPeerBuffers(cfg, world, xs[0].device) for _ in range(world)]
    outs = ep_forward_peers_local(cfg, xs, D["wr"], D["wg"], D["wu"], D["wd"], D["bias"], bufs=bufs)
    torch.cuda.synchronize()
    if skew and world > 1:
        # expert 0's owner received more rows than one rank's batch can hold
        assert max(int(b.grp_offsets[-1]) for b in bufs) > w.T * 2
    for r in range(world):
        want = moe.layer_forward(cfg, xs[r], D["wr"], D["wg"], D["wu"], D["wd"], logit_bias=D["bias"])
        torch.cuda.synchronize()
        assert np.array_equal(_bits(outs[r]), _bits(want)), r
    # rank 0 against the oracle: its fp32 sums (what the owners added, before
    # the rounding) meet the bf16 bar, and the output is those sums rounded once
    ref = oracle.layer_forward(xs_host[0], L0.wr, L0.wg, L0.wu, L0.wd, w.capacity_factor, logit_bias=L0.bias)
    pre = bufs[0].sums.cpu().numpy().astype(np.float64)
    rows = (ref["slot_of"] >= 0).any(1)
    rms = float(np.sqrt(np.mean(ref["out"][rows] ** 2)))
    assert np.max(np.abs(pre[rows] - ref["out"][rows])) <= 2e-2 * rms
    assert np.all(pre[~rows] == 0) and np.all(ref["out"][~rows] == 0)
    rounded = oracle.to_f64(synth.round_bf16(pre).reshape(pre.shape))
    assert np.array_equal(outs[0].float().cpu().numpy().astype(np.float64), rounded)
    assert moe.get_device_error() == 0


def test_peer_dispatch_places_rows_by_owner_then_source():
    world = 4
    w = _case(world, True, T=320)
    L0 = LayerInputs(w)
    D, cfg = L0.dev, L0.cfg
    xs = [to_dev(_batch(w, r)) for r in range(world)]
    bufs = [EpPeerBuffers(cfg, world, xs[0].device) for _ in range(world)]
    addrs = [b.addrs() for b in bufs]
    peers = [moe.EpPeers(world, r, addrs) for r in range(world)]
    disps = [ep_route(cfg, x, D["wr"], D["bias"]) for x in xs]
    table = torch.stack([d["counts_kept"] for d in disps])
    for r in range(world):
        moe.ep_dispatch_peers(cfg, peers[r], table, xs[r], disps[r], bufs[r].grp_offsets)
    torch.cuda.synchronize()
    assert moe.get_device_error() == 0
    tab = table.cpu().numpy()
    host = [{k: disps[p][k].cpu().numpy() for k in ("offsets", "perm", "row_scale")} for p in range(world)]
    for q in range(world):
        mine = owned_experts(q, world)
        x_grp, src, scale = _bits(bufs[q].x_grp), bufs[q].src.cpu().numpy(), bufs[q].scale.cpu().numpy()
        g, offs = 0, []
        for e in range(cfg.E):
            offs.append(g)
            if e not in mine:
                continue
            for p in range(world):
                o = host[p]["offsets"]
                toks = host[p]["perm"][o[e]:o[e + 1]]
                n = len(toks)
                assert n == tab[p, e]
                assert np.array_equal(src[g:g + n], p * w.T + toks)
                assert np.array_equal(scale[g:g + n], host[p]["row_scale"][o[e]:o[e + 1]])
                assert np.array_equal(x_grp[g:g + n], _bits(xs[p])[toks])
                g += n
        offs.append(g)
        assert np.array_equal(bufs[q].grp_offsets.cpu().numpy(), np.array(offs, dtype=np.int32))
    # every rank's sums were cleared for the owners' adds
    for b in bufs:
        assert not b.sums.any()


def test_peer_dispatch_flags_a_table_that_disagrees_with_the_offsets():
    world = 2
    w = _case(world, False, T=320)
    L0 = LayerInputs(w)
    D, cfg = L0.dev, L0.cfg
    xs = [to_dev(_batch(w, r)) for r in range(world)]
    bufs = [EpPeerBuffers(cfg, world, xs[0].device) for _ in range(world)]
    for b in bufs:
        b.x_grp.fill_(7.0)
    peers = [moe.EpPeers(world, r, [b.addrs() for b in bufs]) for r in range(world)]
    disps = [ep_route(cfg, x, D["wr"], D["bias"]) for x in xs]
    table = torch.stack([d["counts_kept"] for d in disps])
    table[0, 3] += 1  # rank 0's own row no longer matches its offsets
    moe.get_device_error(clear=True)
    moe.ep_dispatch_peers(cfg, peers[0], table, xs[0], disps[0], bufs[0].grp_offsets)
    torch.cuda.synchronize()
    assert moe.get_device_error(clear=True) & moe.DEVERR["OFFSETS"]
    assert not bufs[0].grp_offsets.any()
    for b in bufs:
        assert bool((b.x_grp == 7.0).all())


def test_peer_entry_points_reject_what_they_cannot_run():
    w = _case(2, False, T=320)
    L0 = LayerInputs(w)
    cfg = L0.cfg
    b = EpPeerBuffers(cfg, 2, L0.dev["x"].device)
    peers3 = moe.EpPeers(3, 0, [b.addrs()] * 3)  # 3 does not divide E = 8
    out = torch.empty((cfg.T, cfg.d), dtype=torch.bfloat16, device=b.raw.device)
    with pytest.raises(moe.MoEError) as ex:
        moe.ep_combine_peers(cfg, peers3, out)
    assert ex.value.status == 2
    cfg32 = moe.Config(cfg.T, cfg.d, cfg.f, dtype="f32")
    peers = moe.EpPeers(2, 0, [b.addrs()] * 2)
    with pytest.raises(moe.MoEError) as ex:
        moe.ep_combine_peers(cfg32, peers, torch.empty((cfg.T, cfg.d), dtype=torch.float32, device=b.raw.device))
    assert ex.value.status == 2


def _free_port():
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def _peer_worker(rank, world, port, q):
    import sys
    from datetime import timedelta

    import torch.distributed as dist

    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    from sparse_moe_layer_07_b200.expert_parallel import EpPeerGroup, layer_forward_ep_peers

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=timedelta(seconds=120))
    try:
        torch.cuda.set_device(0)
        w = _case(world, True)
        L = LayerInputs(w, x=_batch(w, rank))
        D = L.dev
        pg = EpPeerGroup(L.cfg)
        try:
            outs = []
            for _ in range(2):  # the group's buffers serve step after step
                out = layer_forward_ep_peers(L.cfg, D["x"], D["wr"], D["wg"], D["wu"], D["wd"], logit_bias=D["bias"],
                                             peer_group=pg)
                torch.cuda.synchronize()
                outs.append(_bits(out))
        finally:
            pg.close()
        q.put((rank, outs, moe.get_device_error()))
    finally:
        dist.destroy_process_group()


def test_layer_forward_ep_peers_two_processes_share_buffers_through_ipc():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_peer_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = {}
    try:
        for _ in range(world):
            r, outs, err = q.get(timeout=300)
            got[r] = (outs, err)
    finally:
        for p in procs:
            p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    w = _case(world, True)
    L0 = LayerInputs(w)
    D, cfg = L0.dev, L0.cfg
    for r in range(world):
        want = _bits(moe.layer_forward(cfg, to_dev(_batch(w, r)), D["wr"], D["wg"], D["wu"], D["wd"],
                                       logit_bias=D["bias"]))
        outs, err = got[r]
        assert err == 0
        for o in outs:
            assert np.array_equal(o, want), r
