"""Expert parallelism: each rank owns E/world experts and exchanges token rows.

"Expert parallelism vs. tensor parallelism" (moe_layer_ep_forward): every rank
routes its own tokens, sends each token row to the rank owning the chosen
expert (all-to-all), runs its own experts on what it receives, and sends the
expert outputs back (all-to-all) for the weighted combine in token order.

Here the send side needs no extra permutation: the dispatch already groups a
rank's kept rows by expert, and the experts of one destination rank are
contiguous, so destination q's rows are one slice of x_perm.  The receive
side regroups rows from rank-major (as the all-to-all delivers them) to
expert-major for the grouped GEMM, and back again for the return trip, with
moe_gather_rows.  Routing weights stay on the source rank: experts return
unweighted outputs and the source's combine applies the weights.

The phases (ep_prepare, ep_plan, ep_experts, ep_finish) are separate so that a
caller can run the exchanges with any transport; layer_forward_ep runs them
with torch.distributed: NCCL moves device memory directly, a host backend
(gloo) moves the rows through host memory.

layer_forward_ep_peers replaces both all-to-alls with stores into the other
ranks' memory (moe_ep_dispatch_peers / moe_ep_expert_ffn_peers): the
dispatch kernel writes each kept row into its owner's grouped buffer, the
owner's down kernel adds the weighted outputs into the source's fp32 sums, and
two barriers across the ranks separate the phases.  EpPeerGroup maps the other
ranks' buffers (CUDA IPC); ep_forward_peers_local runs the same kernels for
`world` ranks held by one process on one device.
"""
from __future__ import annotations

import contextlib

import numpy as np
import torch
import torch.distributed as dist

from . import (Config, EpPeers, combine, dispatch, ep_combine_peers, ep_dispatch_peers, ep_expert_ffn_peers,
               expert_ffn, gather_rows, peer_export, peer_import, peer_release, router_topk)


def owned_experts(rank: int, world: int, E: int = 8):
    """Experts of rank `rank`: a contiguous block of E / world."""
    if world < 1 or E % world:
        raise ValueError(f"world size {world} must divide E = {E}")
    n = E // world
    return list(range(rank * n, (rank + 1) * n))


def ep_plan(table, rank: int, world: int):
    """Exchange plan of rank `rank` from table[p, e] = rows rank p sends to expert e.

    send_splits[q]: rows this rank sends to rank q (slices of its x_perm, in order);
    recv_splits[p]: rows it receives from rank p.  Received rows are rank-major
    and, within a source, expert-major; `fwd` lists for every grouped
    (expert-major, then source-major) row the received row it comes from, `inv`
    is its inverse, and `offsets` [E + 1] bound the grouped rows of each expert
    (empty for experts of other ranks)."""
    table = np.asarray(table, dtype=np.int64)
    E = table.shape[1]
    mine = owned_experts(rank, world, E)
    n = len(mine)
    send = [int(table[rank, q * n:(q + 1) * n].sum()) for q in range(world)]
    recv = [int(table[p, mine].sum()) for p in range(world)]
    start = np.zeros((world, n), dtype=np.int64)
    pos = 0
    for p in range(world):
        for j, e in enumerate(mine):
            start[p, j] = pos
            pos += table[p, e]
    fwd = np.empty(pos, dtype=np.int32)
    offsets = np.zeros(E + 1, dtype=np.int32)
    g = 0
    for e in range(E):
        offsets[e] = g
        if e in mine:
            j = mine.index(e)
            for p in range(world):
                c = int(table[p, e])
                fwd[g:g + c] = np.arange(start[p, j], start[p, j] + c, dtype=np.int32)
                g += c
    offsets[E] = g
    inv = np.empty_like(fwd)
    inv[fwd] = np.arange(fwd.size, dtype=np.int32)
    return {"send_splits": send, "recv_splits": recv, "fwd": fwd, "inv": inv, "offsets": offsets, "mine": mine}


def ep_prepare(cfg: Config, x, w_router, logit_bias=None, stream=None):
    """Route and group this rank's tokens; counts_kept [E] is what the table gathers."""
    idx, w, _ = router_topk(cfg, x, w_router, logit_bias, stream=stream)
    disp = dispatch(cfg, x, idx, w, stream=stream)
    return {"idx": idx, "w": w, "disp": disp, "counts": disp["counts_kept"]}


def ep_experts(cfg: Config, x_recv, plan, w_gate, w_up, w_down, stream=None):
    """Run this rank's experts on the received rows; returns their (unweighted)
    outputs in received order, fp32 [n_recv, d]."""
    n = int(plan["offsets"][-1])
    dev = x_recv.device
    if n == 0:
        return torch.empty((0, cfg.d), dtype=torch.float32, device=dev)
    # the grouped GEMM reads up to T * top_k rows: size its buffers for the received rows
    t_e = (n + cfg.top_k - 1) // cfg.top_k
    cfg_e = Config(t_e, cfg.d, cfg.f, E=cfg.E, top_k=cfg.top_k, capacity_factor=float("inf"), dtype=cfg.dtype)
    x_grp = torch.empty((t_e * cfg.top_k, cfg.d), dtype=x_recv.dtype, device=dev)
    gather_rows(x_recv, torch.from_numpy(plan["fwd"]).to(dev), out=x_grp[:n], stream=stream)
    offsets = torch.from_numpy(plan["offsets"]).to(dev)
    _, y_grp = expert_ffn(cfg_e, x_grp, offsets, w_gate, w_up, w_down, None, stream=stream)
    return gather_rows(y_grp, torch.from_numpy(plan["inv"]).to(dev), stream=stream)


def ep_finish(cfg: Config, y_back, state, stream=None):
    """Weighted combine of the returned expert outputs, one row per kept slot in
    this rank's x_perm order (the combine reads only those slots)."""
    return combine(cfg, y_back, state["disp"]["slot_of"], state["w"], weights_applied=False, stream=stream)


def _host_transport(t, group=None):
    """True when the group's backend moves only host tensors (gloo) and t is on a GPU:
    the exchange then goes through host memory (NCCL moves device memory itself)."""
    return t.is_cuda and dist.get_backend(group) != "nccl"


def _all_to_all_rows(send, send_splits, recv_splits, group=None):
    host = _host_transport(send, group)
    src = send.contiguous().cpu() if host else send.contiguous()
    out = torch.empty((sum(recv_splits),) + tuple(send.shape[1:]), dtype=send.dtype, device=src.device)
    a, b = out, src
    if src.dtype == torch.bfloat16 and dist.get_backend(group) != "nccl":
        # a host backend has no 16-bit float type: the rows travel as int32 pairs
        # of their bits (rows hold an even number of values)
        a, b = out.view(torch.int32), src.view(torch.int32)
    dist.all_to_all_single(a, b, recv_splits, send_splits, group=group)
    return out.to(send.device) if host else out


def gather_table(counts, group=None):
    """table[p, e] = counts of rank p, on the host."""
    world = dist.get_world_size(group)
    c = counts.contiguous().cpu() if _host_transport(counts, group) else counts.contiguous()
    parts = [torch.empty_like(c) for _ in range(world)]
    dist.all_gather(parts, c, group=group)
    return torch.stack(parts).cpu().numpy()


def layer_forward_ep(cfg: Config, x, w_router, w_gate, w_up, w_down, logit_bias=None, group=None, stream=None):
    """The layer with expert parallelism over the ranks of `group`: this rank's
    tokens in, this rank's output rows out.  w_gate/w_up/w_down hold all E
    experts' layout; only this rank's experts are read."""
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    st = ep_prepare(cfg, x, w_router, logit_bias, stream=stream)
    plan = ep_plan(gather_table(st["counts"], group), rank, world)
    n_send = sum(plan["send_splits"])
    x_recv = _all_to_all_rows(st["disp"]["x_perm"][:n_send], plan["send_splits"], plan["recv_splits"], group)
    y_recv = ep_experts(cfg, x_recv, plan, w_gate, w_up, w_down, stream=stream)
    y_back = _all_to_all_rows(y_recv, plan["recv_splits"], plan["send_splits"], group)
    return ep_finish(cfg, y_back, st, stream=stream)


# ---------------------------------------------------------------- peer memory

class EpPeerBuffers:
    """One rank's exchange buffers for the peer-memory path, carved from one
    allocation so that a single IPC handle maps them all (the same layout on
    every rank), plus its local scratch: with R = world * T * top_k rows,
    x_grp [R, d], src [R] int32, scale [R] fp32, sums [T, d] fp32 (shared), and
    h [R, f], grp_offsets [E + 1] (local)."""

    def __init__(self, cfg: Config, world: int, device):
        R = world * cfg.T * cfg.top_k
        esz = torch.empty((), dtype=cfg.torch_dtype).element_size()
        sizes = [R * cfg.d * esz, R * 4, R * 4, cfg.T * cfg.d * 4]
        self.part_offsets, off = [], 0
        for n in sizes:
            self.part_offsets.append(off)
            off += (n + 255) // 256 * 256
        self.raw = torch.empty((max(off, 256),), dtype=torch.uint8, device=device)
        o = self.part_offsets
        self.x_grp = self.raw[o[0]:o[0] + sizes[0]].view(cfg.torch_dtype).view(R, cfg.d)
        self.src = self.raw[o[1]:o[1] + sizes[1]].view(torch.int32)
        self.scale = self.raw[o[2]:o[2] + sizes[2]].view(torch.float32)
        self.sums = self.raw[o[3]:o[3] + sizes[3]].view(torch.float32).view(cfg.T, cfg.d)
        self.h = torch.empty((R, cfg.f), dtype=cfg.torch_dtype, device=device)
        self.grp_offsets = torch.empty((cfg.E + 1,), dtype=torch.int32, device=device)

    def addrs(self, base=None):
        """(x_grp, src, scale, sums) addresses given the allocation's address
        `base` in this process (default: this rank's own)."""
        b = self.raw.data_ptr() if base is None else int(base)
        return tuple(b + o for o in self.part_offsets)


def ep_route(cfg: Config, x, w_router, logit_bias=None, stream=None):
    """Route and dispatch this rank's tokens without gathering x (the peer
    dispatch reads x itself)."""
    idx, w, _ = router_topk(cfg, x, w_router, logit_bias, stream=stream)
    return dispatch(cfg, x, idx, w, gather=False, stream=stream)


def ep_forward_peers_local(cfg: Config, xs, w_router, w_gate, w_up, w_down, logit_bias=None, bufs=None,
                           stream=None):
    """The peer-memory path for len(xs) ranks held by this process on one
    device: rank r's tokens xs[r] [T, d], its output returned at [r].  The
    stream's order stands in for the barriers: every rank's dispatch, then
    every rank's experts, then every rank's rounding."""
    world = len(xs)
    dev = xs[0].device
    if bufs is None:
        bufs = [EpPeerBuffers(cfg, world, dev) for _ in range(world)]
    addrs = [b.addrs() for b in bufs]
    peers = [EpPeers(world, r, addrs) for r in range(world)]
    disps = [ep_route(cfg, x, w_router, logit_bias, stream=stream) for x in xs]
    table = torch.stack([d["counts_kept"] for d in disps])
    for r in range(world):
        ep_dispatch_peers(cfg, peers[r], table, xs[r], disps[r], bufs[r].grp_offsets, stream=stream)
    for r in range(world):
        ep_expert_ffn_peers(cfg, peers[r], bufs[r].grp_offsets, w_gate, w_up, w_down, bufs[r].h, stream=stream)
    return [ep_combine_peers(cfg, peers[r], torch.empty((cfg.T, cfg.d), dtype=cfg.torch_dtype, device=dev),
                             stream=stream) for r in range(world)]


def ep_barrier(group=None, device=None):
    """Every rank's earlier work on the current stream is done before any
    rank's later work starts: a one-element NCCL all-reduce on the stream (no
    host wait), or a host barrier after the stream drains (gloo)."""
    if dist.get_backend(group) == "nccl":
        dist.all_reduce(torch.zeros((1,), dtype=torch.int32, device=device), group=group)
    else:
        if device is not None and torch.device(device).type == "cuda":
            torch.cuda.current_stream(device).synchronize()
        dist.barrier(group=group)


def gather_table_device(counts, group=None):
    """table [world, E] int32 on counts' device: row p = counts of rank p."""
    world = dist.get_world_size(group)
    if dist.get_backend(group) == "nccl":
        out = torch.empty((world * counts.numel(),), dtype=counts.dtype, device=counts.device)
        dist.all_gather_into_tensor(out, counts.contiguous(), group=group)
        return out.view(world, -1)
    return torch.from_numpy(gather_table(counts, group).astype(np.int32)).to(counts.device)


class EpPeerGroup:
    """This rank's exchange buffers and the other ranks', mapped into this
    process: the buffers are exported once (moe_peer_export), the handles are
    all-gathered, and every other rank's are imported (moe_peer_import).
    close() releases the mappings; every rank must call it (it ends with a
    barrier, so that no buffer is freed while another rank still maps it)."""

    def __init__(self, cfg: Config, group=None, device=None):
        self.cfg, self.group = cfg, group
        self.rank, self.world = dist.get_rank(group), dist.get_world_size(group)
        dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
        self.device = dev
        self.bufs = EpPeerBuffers(cfg, self.world, dev)
        handle = peer_export(self.bufs.raw)
        handles = [None] * self.world
        dist.all_gather_object(handles, handle, group=group)
        self._mapped = []
        addrs = []
        try:
            for q, hq in enumerate(handles):
                if q == self.rank:
                    addrs.append(self.bufs.addrs())
                else:
                    a = peer_import(hq)
                    self._mapped.append((a, hq))
                    addrs.append(self.bufs.addrs(a))
        except Exception:
            # leave nothing mapped; the other ranks learn of it at their next collective
            for a, h in self._mapped:
                peer_release(a, h)
            self._mapped = []
            raise
        self.peers = EpPeers(self.world, self.rank, addrs)

    def close(self):
        if self.device.type == "cuda":
            torch.cuda.synchronize(self.device)
        for a, h in self._mapped:
            peer_release(a, h)
        self._mapped = []
        dist.barrier(group=self.group)


def layer_forward_ep_peers(cfg: Config, x, w_router, w_gate, w_up, w_down, logit_bias=None, group=None,
                           peer_group: EpPeerGroup | None = None, stream=None):
    """The layer with expert parallelism over peer memory: this rank's tokens
    in, this rank's output rows out (bit for bit the single-device layer on
    them).  peer_group: an EpPeerGroup for cfg (made here, and closed, when
    None)."""
    own = peer_group is None
    pg = EpPeerGroup(cfg, group, x.device) if own else peer_group
    try:
        # the barriers order the current stream: run every phase on it
        with torch.cuda.stream(stream) if stream is not None else contextlib.nullcontext():
            disp = ep_route(cfg, x, w_router, logit_bias)
            table = gather_table_device(disp["counts_kept"], group)
            ep_dispatch_peers(cfg, pg.peers, table, x, disp, pg.bufs.grp_offsets)
            ep_barrier(group, x.device)
            ep_expert_ffn_peers(cfg, pg.peers, pg.bufs.grp_offsets, w_gate, w_up, w_down, pg.bufs.h)
            ep_barrier(group, x.device)
            return ep_combine_peers(cfg, pg.peers,
                                    torch.empty((cfg.T, cfg.d), dtype=cfg.torch_dtype, device=x.device))
    finally:
        if own:
            pg.close()
