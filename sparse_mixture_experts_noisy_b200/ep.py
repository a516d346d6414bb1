"""Expert-parallel layer: the experts are split over G ranks (one rank per GPU).

Rank r owns the contiguous expert range [E*r/G, E*(r+1)/G) and holds only those
experts' W_up and W_down; every rank holds W_g and routes its own tokens.  The
all-to-all dispatch and combine of "Mixture of Experts (MoE) 12段階極小ビジュアル
解剖シミュレーター" STEP 7 and STEP 11-12 (tokens go to the experts that hold
the weights and come back weighted) run as:

  1. route this rank's tokens (moe_route);
  2. slots with the capacity of the *whole* batch: the per-(choice, expert)
     counts are all-gathered as in shard.py ("nanoMoEの深層解剖" slides 17-20:
     all first choices queue before all second choices, tokens in order);
  3. gather the kept rows expert-major (moe_shard_dispatch);
  4. all-gather the kept counts [E], so that every rank knows how many rows
     each rank sends to each expert;
  5. all-to-all: rank r's rows for rank q's experts (one contiguous block of
     its expert-major rows) go to q;
  6. each rank runs its experts' FFN on what it received, one call per source
     rank (each source's block is expert-major over the receiver's experts);
  7. all-to-all back into the original layout;
  8. combine on this rank (moe_combine).

All arithmetic runs in libmoe.so; the collectives move rows and counts.  The
steps are split into functions so that a test can run the ranks one after
another on one GPU with the collectives emulated (`Comm`).  Steps 4-7 need
the kept counts on the host to size the exchange (one device-to-host copy).
"""
from __future__ import annotations

from dataclasses import dataclass

import torch
import torch.distributed as dist

from . import moe
from .shard import exchange_counts


def expert_range(E: int, G: int, r: int) -> tuple[int, int]:
    """The experts rank r owns: [lo, hi)."""
    return E * r // G, E * (r + 1) // G


@dataclass
class Plan:
    """Row counts of the exchange for one rank, from the kept counts [G, E]."""
    send_splits: list   # rows this rank sends to each rank (its expert-major blocks)
    recv_splits: list   # rows this rank receives from each rank
    send_offsets: list  # start row of each destination's block in this rank's gathered rows
    recv_counts: list   # per source: kept rows of each of this rank's experts


def ep_plan(kept_all, G: int, rank: int) -> Plan:
    """kept_all: [G][E] kept rows per (rank, expert) (host ints)."""
    E = len(kept_all[0])
    lo, hi = expert_range(E, G, rank)
    send, starts = [], []
    run = 0
    for q in range(G):
        qlo, qhi = expert_range(E, G, q)
        n = int(sum(kept_all[rank][qlo:qhi]))
        starts.append(run)
        send.append(n)
        run += n
    recv_counts = [[int(c) for c in kept_all[s][lo:hi]] for s in range(G)]
    recv = [sum(c) for c in recv_counts]
    return Plan(send, recv, starts, recv_counts)


class Comm:
    """The two collectives the layer uses, over a torch.distributed group."""

    def __init__(self, group=None):
        self.group = group

    def rank(self) -> int:
        return dist.get_rank(self.group)

    def world(self) -> int:
        return dist.get_world_size(self.group)

    def all_gather(self, t: torch.Tensor) -> torch.Tensor:
        """[*shape] -> [G, *shape] in rank order."""
        if t.dim() == 2:
            return exchange_counts(t, self.group)
        return exchange_counts(t.view(1, -1), self.group).view(self.world(), *t.shape)

    def all_to_all(self, outputs: list, inputs: list) -> None:
        """outputs[q] <- what rank q sends here; inputs[q] goes to rank q."""
        if dist.get_backend(self.group) == "nccl":
            dist.all_to_all(outputs, inputs, group=self.group)
            return
        # backends without an all-to-all (gloo): point-to-point pairs
        me = self.rank()
        reqs = []
        for q in range(self.world()):
            peer = q if self.group is None else dist.get_global_rank(self.group, q)
            if q == me:
                outputs[q].copy_(inputs[q])
                continue
            if inputs[q].numel():
                reqs.append(dist.isend(inputs[q].contiguous(), peer, group=self.group))
            if outputs[q].numel():
                reqs.append(dist.irecv(outputs[q], peer, group=self.group))
        for r in reqs:
            r.wait()


def _pad128(n: int) -> int:
    return max(128, (n + 127) // 128 * 128)


def step_route(x, W_g, k, E, b_g=None, noise=None, sigma=0.0, stream=None):
    """Steps 1-2 (local part): routing and this rank's [k, E] counts."""
    topk, gates, _ = moe.moe_route(x, W_g, k, b_g=b_g, noise=noise, sigma=sigma, want_logits=False,
                                   stream=stream)
    ws = moe.shard_workspace(x.shape[0], E, k, x.device)
    counts_je = moe.moe_shard_count(topk, E, ws, stream=stream)
    return dict(topk=topk, gates=gates, ws=ws, counts_je=counts_je)


def step_dispatch(st, x, E, k, cf, N_total, all_counts, rank, stream=None):
    """Steps 2-3: slots against the whole batch's capacity, expert-major rows."""
    base = moe.moe_shard_base(all_counts, rank, stream=stream)
    C = moe.capacity(N_total, E, k, cf)
    d = moe.moe_shard_dispatch(st["topk"], x, E, C, st["counts_je"], base, st["ws"], stream=stream)
    st.update(dispatch=d, C=C)
    return st


def step_send_views(st, plan: Plan):
    """Step 5 (send side): this rank's gathered rows, one contiguous view per destination."""
    xg = st["dispatch"]["x_gathered"]
    return [xg[s0:s0 + n] for s0, n in zip(plan.send_offsets, plan.send_splits)]


def step_recv_buffers(plan: Plan, d: int, dtype, device):
    """Step 5 (receive side): one buffer per source, padded to whole 128-row
    tiles for the expert FFN; the exchange fills the first rows of each."""
    bufs = [torch.empty((_pad128(n), d), dtype=dtype, device=device) for n in plan.recv_splits]
    return bufs, [b[:n] for b, n in zip(bufs, plan.recv_splits)]


def step_experts(plan: Plan, recv_bufs, W_up_local, W_down_local, stream=None, act=moe.ACT_RELU, b_up=None,
                 b_down=None):
    """Step 6: this rank's experts on each source's rows (one call per source)."""
    outs = []
    dev = W_up_local.device
    for buf, counts in zip(recv_bufs, plan.recv_counts):
        c = torch.tensor(counts, dtype=torch.int32)
        offs = torch.zeros(len(counts) + 1, dtype=torch.int32)
        offs[1:] = torch.cumsum(c, 0)
        out = moe.moe_expert_ffn(buf, offs.to(dev), c.to(dev), W_up_local, W_down_local, stream=stream, act=act,
                                 b_up=b_up, b_down=b_down)
        outs.append(out)
    return outs


def step_return_views(st, plan: Plan):
    """Step 7 (receive side): the rows coming back land in the layout they left."""
    xg = st["dispatch"]["x_gathered"]
    og = torch.empty_like(xg)
    st["out_gathered"] = og
    return [og[s0:s0 + n] for s0, n in zip(plan.send_offsets, plan.send_splits)]


def step_combine(st, stream=None):
    """Step 8."""
    d = st["dispatch"]
    return moe.moe_combine(st["out_gathered"], d["slot"], st["topk"], d["offsets"], st["gates"], stream=stream)


def expert_parallel_forward(x, W_g, W_up_local, W_down_local, k, cf, N_total, comm: Comm | None = None,
                            b_g=None, noise=None, sigma=0.0, stream=None):
    """This rank's part of one batch of N_total tokens with the experts split
    over the group.  x: [N_local, d] (device); W_up_local / W_down_local: this
    rank's experts (expert_range).  -> (y [N_local, d], dict of tables)."""
    comm = comm or Comm()
    G, rank = comm.world(), comm.rank()
    E = W_g.shape[0]
    st = step_route(x, W_g, k, E, b_g=b_g, noise=noise, sigma=sigma, stream=stream)
    all_counts = comm.all_gather(st["counts_je"])
    step_dispatch(st, x, E, k, cf, N_total, all_counts, rank, stream=stream)
    kept_all = comm.all_gather(st["dispatch"]["counts"]).cpu().tolist()
    plan = ep_plan(kept_all, G, rank)
    bufs, recv_views = step_recv_buffers(plan, x.shape[1], x.dtype, x.device)
    comm.all_to_all(recv_views, step_send_views(st, plan))
    outs = step_experts(plan, bufs, W_up_local, W_down_local, stream=stream)
    back = step_return_views(st, plan)
    comm.all_to_all(back, [o[:n] for o, n in zip(outs, plan.recv_splits)])
    y = step_combine(st, stream=stream)
    return y, dict(topk_idx=st["topk"], gates=st["gates"], slot=st["dispatch"]["slot"],
                   counts=st["dispatch"]["counts"], plan=plan)
