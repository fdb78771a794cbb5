"""The multi-rank path of bench.py on CPU: two gloo ranks check that weights
generated on rank 0 reach rank 1 unchanged, that each rank runs a distinct
batch, and that timing is the max over ranks with whole-job throughput."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import sys

    sys.path.insert(0, ROOT)
    import bench
    from synth import configs

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        w = configs.scaled(configs.WORKLOADS["mid_bf16"], name="gloo", T=16, d=256, f=384)
        if rank == 0:
            W = {"wr": torch.from_numpy(configs.make_router(w).astype(np.int32))}
        else:
            W = {"wr": torch.zeros((8, 256), dtype=torch.int32)}
        bench.share_weights(W, world)
        x = bench.rank_x(w, rank)
        t = bench.max_over_ranks(3.0 + 2.0 * rank, torch.device("cpu"), world)
        q.put((rank, W["wr"].numpy().copy(), x.copy(), t,
               bench.throughput(world, w.T, 10, t)))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict()
    for _ in range(2):
        r = q.get(timeout=120)
        res[r[0]] = r
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    from synth import configs

    w = configs.scaled(configs.WORKLOADS["mid_bf16"], name="gloo", T=16, d=256, f=384)
    expect_wr = configs.make_router(w).astype(np.int32)
    assert np.array_equal(res[0][1], expect_wr) and np.array_equal(res[1][1], expect_wr)
    assert np.array_equal(res[0][2], configs.make_x(w))
    assert not np.array_equal(res[0][2], res[1][2])
    assert res[0][3] == res[1][3] == 5.0
    assert res[0][4] == pytest.approx(2 * 16 * 10 / 0.005)


def _shard_worker(rank, world, port, q):
    import sys

    sys.path.insert(0, ROOT)
    import oracle
    from sparse_moe_layer_07_b200.sharded import gather_shard_counts

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        idx, _, cap, per = _global_routing(oracle)
        mine = idx[rank * per:(rank + 1) * per]
        counts = torch.from_numpy(np.bincount(mine.ravel(), minlength=8).astype(np.int32))
        table = gather_shard_counts(counts).numpy()
        prior = table[:rank].sum(0)
        seen = np.zeros(8, dtype=np.int64)
        kept = np.zeros(mine.shape, dtype=bool)
        for t in range(per):
            for j in range(2):
                e = mine[t, j]
                kept[t, j] = prior[e] + seen[e] < cap
                seen[e] += 1
        q.put((rank, table, kept))
    finally:
        dist.destroy_process_group()


def _global_routing(oracle):
    rng = np.random.default_rng(31)
    T, d = 90, 16
    x = rng.standard_normal((T, d))
    wr = rng.standard_normal((8, d)) * 0.3
    lg = oracle.router_logits(x, wr, np.array([1.5, 0.5, 0, 0, 0, 0, 0, 0]))
    idx, w = oracle.top2_softmax(lg)
    return idx, w, oracle.capacity(T, 2, 8, 1.0), T // 3


def test_three_gloo_ranks_shard_the_global_capacity():
    # each rank holds a contiguous third of the batch; one all-gather of the E route
    # counts per rank lets every rank apply the global lowest-index-first rule alone
    import oracle

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_worker, args=(r, 3, port, q)) for r in range(3)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(3):
        r = q.get(timeout=120)
        res[r[0]] = r
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    idx, w, cap, per = _global_routing(oracle)
    ref = oracle.dispatch(idx, w, 8, cap)
    assert ref["dropped"] > 0
    want_table = np.stack([np.bincount(idx[r * per:(r + 1) * per].ravel(), minlength=8) for r in range(3)])
    for r in range(3):
        assert np.array_equal(res[r][1], want_table)
    kept = np.concatenate([res[r][2] for r in range(3)])
    assert np.array_equal(kept, ref["slot_of"] >= 0)


def _ep_worker(rank, world, port, q):
    # the exchange plan and the two all-to-alls of expert parallelism, carrying token ids
    import sys

    sys.path.insert(0, ROOT)
    import oracle
    from sparse_moe_layer_07_b200.expert_parallel import (_all_to_all_rows, ep_barrier, ep_plan, gather_table,
                                                          gather_table_device)

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        idx, w, cap, per = _ep_routing(oracle, world, rank)
        disp = oracle.dispatch(idx, w, 8, cap)
        table = gather_table(torch.from_numpy(disp["counts_kept"].astype(np.int32)))
        # the peer-memory path's table (int32 tensor on the counts' device) and barrier
        t_dev = gather_table_device(torch.from_numpy(disp["counts_kept"].astype(np.int32)))
        assert t_dev.dtype == torch.int32 and np.array_equal(t_dev.numpy(), table)
        ep_barrier(device="cpu")
        plan = ep_plan(table, rank, world)
        # each row carries (source rank, token, expert)
        n = disp["n_kept"]
        experts = np.repeat(np.arange(8), disp["counts_kept"])
        rows = torch.from_numpy(np.stack([np.full(n, rank), disp["perm"], experts], 1).astype(np.int64))
        recv = _all_to_all_rows(rows[:sum(plan["send_splits"])], plan["send_splits"], plan["recv_splits"])
        # the same rows in bf16 (small integers are exact; 4 columns, as bf16 rows travel in int32 pairs)
        rows16 = torch.cat([rows, torch.zeros((n, 1), dtype=torch.int64)], 1).to(torch.bfloat16)
        recv16 = _all_to_all_rows(rows16[:sum(plan["send_splits"])], plan["send_splits"], plan["recv_splits"])
        assert recv16.dtype == torch.bfloat16
        assert torch.equal(recv16[:, :3].to(torch.int64), recv) and not recv16[:, 3].any()
        grouped = recv.numpy()[plan["fwd"]]
        back = _all_to_all_rows(torch.from_numpy(grouped[plan["inv"]]), plan["recv_splits"], plan["send_splits"])
        q.put((rank, table, grouped, plan["offsets"], back.numpy(), rows.numpy()))
    finally:
        dist.destroy_process_group()


def _ep_routing(oracle, world, rank):
    rng = np.random.default_rng(40 + rank)
    T, d = 50, 16
    x = rng.standard_normal((T, d))
    wr = np.random.default_rng(39).standard_normal((8, d))
    lg = oracle.router_logits(x, wr, np.array([1.0, 0.5, 0, 0, 0, 0, 0, -1.0]))
    idx, w = oracle.top2_softmax(lg)
    return idx, w, oracle.capacity(T, 2, 8, 1.25), T


@pytest.mark.parametrize("world", [2, 4])
def test_expert_parallel_exchange_on_gloo_ranks(world):
    import oracle

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_ep_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(world):
        r = q.get(timeout=120)
        res[r[0]] = r
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    n_own = 8 // world
    for rank in range(world):
        _, table, grouped, offsets, back, sent = res[rank]
        # grouped rows of each own expert: every source's kept tokens of that expert, source-major, token order
        for e in range(rank * n_own, (rank + 1) * n_own):
            want = []
            for src in range(world):
                idx, w, cap, _ = _ep_routing(oracle, world, src)
                d = oracle.dispatch(idx, w, 8, cap)
                toks = d["perm"][d["offsets"][e]:d["offsets"][e + 1]]
                want += [(src, int(t), e) for t in toks]
            got = [tuple(int(v) for v in r) for r in grouped[offsets[e]:offsets[e + 1]]]
            assert got == want, (rank, e)
        assert all(offsets[e + 1] == offsets[e] for e in range(8) if e // n_own != rank)
        # the return trip puts every row back where this rank sent it from
        assert np.array_equal(back, sent[:back.shape[0]]) and back.shape[0] == sent.shape[0]


def _peer_group_worker(rank, world, port, q, fail_rank):
    # EpPeerGroup's mapping lifecycle on gloo ranks, with the CUDA IPC calls
    # replaced by host fakes (no GPU): handles are exchanged, every other
    # rank's buffers are "imported", close() releases each mapping once, and
    # an import that fails releases what was already mapped before raising
    import sys

    sys.path.insert(0, ROOT)
    from sparse_moe_layer_07_b200 import Config
    import sparse_moe_layer_07_b200.expert_parallel as ep

    released = []
    ep.peer_export = lambda t: f"handle-{rank}".encode()

    def fake_import(h):
        src = int(h.decode().split("-")[1])
        if rank == fail_rank and src == world - 1:
            raise RuntimeError("import refused")
        return (1 << 40) * (src + 1)

    ep.peer_import = fake_import
    ep.peer_release = lambda addr, h: released.append((addr, h))
    from datetime import timedelta

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=timedelta(seconds=10))
    try:
        cfg = Config(64, 256, 384)
        try:
            pg = ep.EpPeerGroup(cfg, device="cpu")
        except RuntimeError as exc:
            q.put((rank, "raised", str(exc), released))
            return
        addrs = [tuple(pg.peers._c.x_grp[i] for i in range(world)), tuple(pg.peers._c.sums[i] for i in range(world))]
        own = pg.bufs.addrs()
        try:
            pg.close()
            status = "ok"
        except RuntimeError:
            # a rank that failed never reaches close()'s barrier: the others see it fail
            status = "peer failed"
        q.put((rank, status, (addrs, own, pg.bufs.part_offsets), released))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("fail_rank", [-1, 0])
def test_peer_group_maps_every_other_rank_and_releases_once(fail_rank):
    world = 3
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_peer_group_worker, args=(r, world, port, q, fail_rank)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    try:
        for _ in range(world):
            r = q.get(timeout=120)
            res[r[0]] = r[1:]
    finally:
        for p in procs:
            p.join(timeout=60)
    for rank in range(world):
        status, payload, released = res[rank]
        if rank == fail_rank:
            # the import of the last rank failed: the one made before it is released, then the error surfaces
            assert status == "raised" and "refused" in payload
            others = [s for s in range(world) if s not in (rank, world - 1)]
            assert released == [((1 << 40) * (s + 1), f"handle-{s}".encode()) for s in others]
            continue
        assert status == ("ok" if fail_rank < 0 else "peer failed")
        (x_grp, sums), own, offs = payload
        for s in range(world):
            base = own[0] - offs[0] if s == rank else (1 << 40) * (s + 1)
            assert x_grp[s] == base + offs[0] and sums[s] == base + offs[3]
        assert sorted(released) == sorted(((1 << 40) * (s + 1), f"handle-{s}".encode())
                                          for s in range(world) if s != rank)
