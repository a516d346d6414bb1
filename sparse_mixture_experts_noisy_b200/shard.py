"""One layer batch with its tokens split over several GPUs (one rank per GPU).

A token's queue place at an expert depends on every earlier token of the batch:
all first choices come before all second choices, tokens in order within a
choice rank ("nanoMoEの深層解剖", slides 17-20), and places past the capacity
C = ceil(cf * N * k / E) of the *whole* batch are dropped.  So the ranks
exchange one small table, their per-(choice, expert) counts ([k, E] int32),
with an all-gather; each rank then turns the gathered table into the first
queue place of each (choice, expert) on its own tokens and runs the rest of
the layer locally.  Routing, expert FFN and combine are per token and need no
communication.  The result equals one unsharded call on the concatenated batch:
the same drop set and, per token, the same output.

Tokens are split in contiguous ranges in rank order (rank 0 holds the first
tokens).  All compute runs in libmoe.so; torch.distributed only moves the
counts.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import moe


def exchange_counts(counts_je: torch.Tensor, group=None) -> torch.Tensor:
    """All-gather each rank's [k, E] counts -> [G, k, E] in rank order."""
    world = dist.get_world_size(group)
    k, E = counts_je.shape
    if dist.get_backend(group) == "nccl":
        out = torch.empty((world * k, E), dtype=counts_je.dtype, device=counts_je.device)
        dist.all_gather_into_tensor(out, counts_je.contiguous(), group=group)
        return out.view(world, k, E)
    parts = [torch.empty_like(counts_je) for _ in range(world)]
    dist.all_gather(parts, counts_je.contiguous(), group=group)
    return torch.stack(parts)


def sharded_forward(x, W_g, W_up, W_down, k, cf, N_total, group=None, b_g=None, noise=None, sigma=0.0,
                    stream=None):
    """This rank's part of one batch of N_total tokens.  x: [N_local, d] (device).
    -> (y [N_local, d], dict of routing tables for this rank)."""
    rank = dist.get_rank(group)
    E = W_g.shape[0]
    N_local = x.shape[0]
    topk, gates, _ = moe.moe_route(x, W_g, k, b_g=b_g, noise=noise, sigma=sigma, want_logits=False,
                                   stream=stream)
    ws = moe.shard_workspace(N_local, E, k, x.device)
    counts_je = moe.moe_shard_count(topk, E, ws, stream=stream)
    all_counts = exchange_counts(counts_je, group)
    base = moe.moe_shard_base(all_counts, rank, stream=stream)
    C = moe.capacity(N_total, E, k, cf)
    d = moe.moe_shard_dispatch(topk, x, E, C, counts_je, base, ws, stream=stream)
    out = moe.moe_expert_ffn(d["x_gathered"], d["offsets"], d["counts"], W_up, W_down, stream=stream)
    y = moe.moe_combine(out, d["slot"], topk, d["offsets"], gates, stream=stream)
    return y, dict(topk_idx=topk, gates=gates, slot=d["slot"], counts=d["counts"], base=base,
                   counts_je=counts_je, all_counts=all_counts, C=C)
