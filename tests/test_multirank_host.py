"""Multi-process host logic on CPU with the gloo backend (no GPU).

1. Token-sharded dispatch: ranks hold contiguous token ranges of one batch,
   exchange their per-(choice, expert) counts with shard.exchange_counts, and
   apply the shard rule (place = base[j][e] + place among the shard's j-th
   choices of e, dropped at the whole batch's capacity).  Rank 0 checks the
   union against the unsharded oracle.
2. bench.py's rank plumbing: max over ranks and whole-job throughput.
3. Expert parallelism: every rank's exchange plan (rows it sends to and
   receives from each rank) agrees with every other rank's, and ep.Comm's
   all-to-all delivers each block to its owner and back.
"""
import datetime
import math
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _init(rank, world, port):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))


def _shard_worker(rank, world, port, N, E, k, cf, seed):
    import sys
    sys.path.insert(0, ROOT)
    import oracle
    from sparse_mixture_experts_noisy_b200.shard import exchange_counts
    _init(rank, world, port)
    try:
        rng = np.random.default_rng(seed)
        logits = rng.integers(-3, 4, size=(N, E)).astype(np.float32)   # many ties
        idx, _ = oracle.route_from_logits(logits, k)
        lo, hi = N * rank // world, N * (rank + 1) // world
        mine = idx[lo:hi]
        T = np.zeros((k, E), dtype=np.int32)
        for j in range(k):
            T[j] = np.bincount(mine[:, j], minlength=E)
        all_T = exchange_counts(torch.from_numpy(T)).numpy()
        assert all_T.shape == (world, k, E) and np.array_equal(all_T[rank], T)
        base = np.zeros((k, E), dtype=np.int64)
        for j in range(k):
            base[j] = all_T[:, :j, :].sum(axis=(0, 1)) + all_T[:rank, j, :].sum(axis=0)
        C = oracle.capacity(N, E, k, cf)
        place = np.zeros(mine.shape, dtype=np.int64)
        for j in range(k):
            seen = np.zeros(E, dtype=np.int64)
            for t in range(hi - lo):
                e = mine[t, j]
                place[t, j] = base[j, e] + seen[e]
                seen[e] += 1
        got = dist.get_world_size()
        parts = [None] * got
        dist.all_gather_object(parts, (lo, hi, place.tolist()))
        if rank == 0:
            full_place = np.concatenate([np.array(p[2], dtype=np.int64).reshape(p[1] - p[0], k) for p in parts])
            ref_place, _ = oracle.assign_slots(idx, E, N)        # places before any cut
            assert np.array_equal(full_place, ref_place)
            ref_slot, ref_counts = oracle.assign_slots(idx, E, C)
            assert np.array_equal(np.where(full_place < C, full_place, -1), ref_slot)
            kept = full_place < C
            assert [int(np.sum(kept & (idx == e))) for e in range(E)] == ref_counts.tolist()
    finally:
        dist.barrier()
        dist.destroy_process_group()


@pytest.mark.parametrize("world,N,E,k,cf", [(2, 300, 6, 2, 1.0), (3, 257, 5, 3, 0.7), (2, 64, 8, 2, math.inf)])
def test_sharded_dispatch_matches_unsharded_oracle(world, N, E, k, cf):
    mp.start_processes(_shard_worker, args=(world, _port(), N, E, k, cf, 11), nprocs=world,
                       start_method="spawn", join=True)


def _bench_worker(rank, world, port):
    import sys
    sys.path.insert(0, ROOT)
    _init(rank, world, port)
    try:
        import bench
        d = bench.Dist.__new__(bench.Dist)
        d.world, d.rank, d.local_rank, d.pg = world, rank, rank, dist
        mx = d.max(1.0 + rank, device="cpu")
        assert mx == float(world)
        agg = bench.aggregate(1000, 10, world, mx)
        assert agg["value"] == pytest.approx(1000 * 10 * world / world)
        assert agg["ms_per_step"] == pytest.approx(1e3 * world / 10)
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_bench_takes_the_slowest_rank():
    mp.start_processes(_bench_worker, args=(2, _port()), nprocs=2, start_method="spawn", join=True)


def _ep_worker(rank, world, port, E, seed):
    import sys
    sys.path.insert(0, ROOT)
    from sparse_mixture_experts_noisy_b200 import ep
    _init(rank, world, port)
    try:
        comm = ep.Comm()
        rng = np.random.default_rng(seed + rank)
        kept = torch.from_numpy(rng.integers(0, 9, size=E).astype(np.int32))
        kept_all = comm.all_gather(kept)
        assert kept_all.shape == (world, E) and torch.equal(kept_all[rank], kept)
        plan = ep.ep_plan(kept_all.tolist(), world, rank)
        plans = [None] * world
        dist.all_gather_object(plans, (plan.send_splits, plan.recv_splits, plan.recv_counts))
        for q in range(world):
            assert plans[q][0][rank] == plan.recv_splits[q]
            lo, hi = ep.expert_range(E, world, rank)
            assert plan.recv_counts[q] == kept_all[q, lo:hi].tolist()
        # rows tagged (source, expert, row) travel to the expert's owner and back
        d = 3
        rows = []
        for e in range(E):
            for i in range(int(kept[e])):
                rows.append([rank, e, i])
        xg = torch.tensor(rows, dtype=torch.float32).reshape(-1, d)
        sends = [xg[s0:s0 + n] for s0, n in zip(plan.send_offsets, plan.send_splits)]
        recv = [torch.empty((n, d)) for n in plan.recv_splits]
        comm.all_to_all(recv, sends)
        lo, hi = ep.expert_range(E, world, rank)
        for s in range(world):
            got = recv[s]
            assert torch.all(got[:, 0] == s)
            assert torch.all((got[:, 1] >= lo) & (got[:, 1] < hi))
            assert got.shape[0] == sum(plan.recv_counts[s])
        back = [torch.empty_like(t) for t in sends]
        comm.all_to_all(back, [r.clone() for r in recv])
        assert torch.equal(torch.cat(back), xg)
    finally:
        dist.barrier()
        dist.destroy_process_group()


@pytest.mark.parametrize("world,E", [(2, 8), (4, 8), (3, 7)])
def test_expert_parallel_exchange(world, E):
    mp.start_processes(_ep_worker, args=(world, _port(), E, 21), nprocs=world, start_method="spawn", join=True)
