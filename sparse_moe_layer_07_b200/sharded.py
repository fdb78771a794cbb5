"""A batch split into token shards across ranks, under the global capacity rule.

"Routing: top-2 without auxiliary loss" sets the capacity from the whole batch
and drops overflow lowest token index first.  With the batch split into
contiguous token shards, one per rank, in rank order, every rank needs one
thing from the others: how many assignments each expert received from the
tokens of earlier shards.  That is one all-gather of E integers per rank
(gather_shard_counts); everything else runs on the rank's own tokens through
the C ABI (moe_route_counts, moe_dispatch_shard, the expert FFN, the combine).
With capacity_factor = +inf or E/top_k no assignment is dropped and the shards
need no exchange at all.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import Config, capacity, combine, dispatch_shard, expert_ffn, route_counts, router_topk


def gather_shard_counts(counts: torch.Tensor, group=None) -> torch.Tensor:
    """Every rank's route counts in rank order, [world, E] int32 on counts' device."""
    world = dist.get_world_size(group)
    parts = [torch.empty_like(counts) for _ in range(world)]
    dist.all_gather(parts, counts.contiguous(), group=group)
    return torch.stack(parts)


def global_capacity(cfg_shard: Config, tokens_global: int) -> int:
    """Capacity of the whole batch (moe_capacity of the global config)."""
    g = Config(tokens_global, cfg_shard.d, cfg_shard.f, E=cfg_shard.E, top_k=cfg_shard.top_k,
               capacity_factor=cfg_shard.capacity_factor, dtype=cfg_shard.dtype)
    return capacity(g)


def layer_forward_shard(cfg: Config, tokens_global: int, shard_counts_fn, shard: int, x, w_router, w_gate, w_up,
                        w_down, logit_bias=None, stream=None):
    """This rank's tokens through the layer with the global capacity.  shard_counts_fn
    maps this shard's route counts to the [n_shards, E] table of all shards'
    counts (gather_shard_counts under torch.distributed)."""
    idx, w, _ = router_topk(cfg, x, w_router, logit_bias, stream=stream)
    table = shard_counts_fn(route_counts(cfg, idx, stream=stream))
    disp = dispatch_shard(cfg, global_capacity(cfg, tokens_global), table, shard, x, idx, w, stream=stream)
    _, y = expert_ffn(cfg, disp["x_perm"], disp["offsets"], w_gate, w_up, w_down, disp["row_scale"], stream=stream)
    return combine(cfg, y, disp["slot_of"], stream=stream), disp
