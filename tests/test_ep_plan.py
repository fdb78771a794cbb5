"""Host logic of expert parallelism and token sharding (no GPU, no ranks):
the exchange plan's splits, regroup permutation and offsets, and the global
capacity of a sharded batch."""
import numpy as np
import pytest

from sparse_moe_layer_07_b200 import Config
from sparse_moe_layer_07_b200.expert_parallel import ep_plan, owned_experts
from sparse_moe_layer_07_b200.sharded import global_capacity


def test_owned_experts_partition_the_experts():
    for world in (1, 2, 4, 8):
        seen = sum((owned_experts(r, world) for r in range(world)), [])
        assert seen == list(range(8))
    with pytest.raises(ValueError):
        owned_experts(0, 3)


def test_single_rank_plan_is_the_identity():
    table = np.array([[3, 0, 5, 1, 0, 2, 4, 1]])
    p = ep_plan(table, 0, 1)
    assert p["send_splits"] == [16] and p["recv_splits"] == [16]
    assert np.array_equal(p["fwd"], np.arange(16)) and np.array_equal(p["inv"], np.arange(16))
    assert np.array_equal(p["offsets"], np.concatenate([[0], np.cumsum(table[0])]))


@pytest.mark.parametrize("world", [2, 4, 8])
def test_plan_regroups_source_major_rows_expert_major(world):
    rng = np.random.default_rng(world)
    table = rng.integers(0, 7, size=(world, 8))
    n = 8 // world
    for rank in range(world):
        p = ep_plan(table, rank, world)
        mine = list(range(rank * n, (rank + 1) * n))
        # every source sends this rank its experts' rows; every rank receives its share
        assert p["recv_splits"] == [int(table[s, mine].sum()) for s in range(world)]
        assert p["send_splits"] == [int(table[rank, q * n:(q + 1) * n].sum()) for q in range(world)]
        # label received rows by (source, expert) in arrival order, then regroup
        labels = [(s, e) for s in range(world) for e in mine for _ in range(table[s, e])]
        grouped = [labels[i] for i in p["fwd"]]
        want = [(s, e) for e in mine for s in range(world) for _ in range(table[s, e])]
        assert grouped == want
        assert np.array_equal(np.asarray(p["fwd"])[p["inv"]], np.arange(len(labels)))
        counts = np.diff(p["offsets"])
        assert all(counts[e] == (table[:, e].sum() if e in mine else 0) for e in range(8))


def test_all_rows_to_one_expert():
    table = np.zeros((4, 8), dtype=np.int64)
    table[:, 0] = [5, 0, 7, 1]
    p0 = ep_plan(table, 0, 4)
    assert p0["recv_splits"] == [5, 0, 7, 1] and p0["offsets"][-1] == 13
    for r in (1, 2, 3):
        pr = ep_plan(table, r, 4)
        assert pr["recv_splits"] == [0, 0, 0, 0] and pr["fwd"].size == 0


def test_global_capacity_uses_the_whole_batch():
    shard = Config(300, 256, 384, capacity_factor=1.25, dtype="bf16")
    assert global_capacity(shard, 1200) == int(np.ceil(1.25 * 1200 * 2 / 8))
    inf = Config(300, 256, 384, capacity_factor=float("inf"), dtype="bf16")
    assert global_capacity(inf, 1200) == 1200


def test_peer_buffers_layout_is_aligned_and_disjoint():
    import torch

    from sparse_moe_layer_07_b200 import Config
    from sparse_moe_layer_07_b200.expert_parallel import EpPeerBuffers

    cfg = Config(300, 256, 384)
    world = 4
    b = EpPeerBuffers(cfg, world, "cpu")
    R = world * cfg.T * cfg.top_k
    assert b.x_grp.shape == (R, cfg.d) and b.x_grp.dtype == torch.bfloat16
    assert b.src.numel() == R and b.scale.numel() == R and b.sums.shape == (cfg.T, cfg.d)
    assert b.h.shape == (R, cfg.f) and b.grp_offsets.numel() == cfg.E + 1
    parts = [b.x_grp, b.src, b.scale, b.sums]
    spans = sorted((t.data_ptr(), t.data_ptr() + t.numel() * t.element_size()) for t in parts)
    for (a0, a1), (b0, _) in zip(spans, spans[1:]):
        assert a1 <= b0
    assert spans[-1][1] <= b.raw.data_ptr() + b.raw.numel()
    # another process sees the same layout from its own mapping of the allocation
    assert b.addrs() == tuple(t.data_ptr() for t in parts)
    assert b.addrs(1 << 40) == tuple((1 << 40) + o for o in b.part_offsets)
    assert all(o % 256 == 0 for o in b.part_offsets)


def test_peer_table_checks_its_shape():
    from sparse_moe_layer_07_b200 import EP_MAX_WORLD, EpPeers

    with pytest.raises(ValueError):
        EpPeers(EP_MAX_WORLD + 1, 0, [(0, 0, 0, 0)] * (EP_MAX_WORLD + 1))
    with pytest.raises(ValueError):
        EpPeers(2, 2, [(0, 0, 0, 0)] * 2)
    with pytest.raises(ValueError):
        EpPeers(2, 0, [(0, 0, 0, 0)])
    p = EpPeers(2, 1, [(16, 32, 48, 64), (80, 96, 112, 128)])
    assert (p._c.world, p._c.rank) == (2, 1)
    assert (p._c.x_grp[1], p._c.src[1], p._c.scale[1], p._c.sums[1]) == (80, 96, 112, 128)
