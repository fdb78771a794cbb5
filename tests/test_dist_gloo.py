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
