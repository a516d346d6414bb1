"""Token-sharded batches on the GPU (needs a B200).

The G shards of one batch run one after another on one GPU; the all-gather of
their counts is emulated by stacking the tables, which is all the exchange
does.  Every shard's output must equal, bit for bit, the rows of the same
calls made once on the whole batch, and the drop set must be the same.  The
shards are also checked against the oracle on the whole batch (replaying the
GPU's fp32 logits): top-k, the drop set and each expert's row order bit for
bit, and the output of a sample of tokens within the bf16 tolerance and the
per-element rounding model."""
import numpy as np
import pytest
import torch

import oracle
from sparse_mixture_experts_noisy_b200 import moe
from sparse_mixture_experts_noisy_b200.synth import WORKLOADS
from tests.gpu_util import (Case, TOL, bf16_error_sigma, check_elementwise_bf16, rel_err, require_gpu,
                            to_host_bits, values)


def check_shards_against_oracle(case, cuts, topks, slots, y, lg):
    """Sharded results against the oracle on the whole batch, given the GPU's
    logits of every token (batch-size independent, so the shards' logits are
    the whole batch's)."""
    wl, inp = case.wl, case.inp
    idx, g = oracle.route_from_logits(lg, wl.k, inp.noise, wl.sigma)
    C = oracle.capacity(wl.N, wl.E, wl.k, wl.cf)
    slot_ref, counts_ref = oracle.assign_slots(idx, wl.E, C)
    tk = np.concatenate(topks)
    sl = np.concatenate(slots)
    assert np.array_equal(tk, idx), "top-k of the shards differs from the oracle"
    assert np.array_equal(sl < 0, slot_ref < 0), "drop set differs from the oracle"
    # inside every shard, each expert's rows come in the oracle's queue order
    for g_, (a, b) in enumerate(zip(cuts[:-1], cuts[1:])):
        for e in range(wl.E):
            m = (tk[a:b] == e) & (sl[a:b] >= 0)
            local = sl[a:b][m]
            glob = slot_ref[a:b][m]
            assert np.array_equal(np.argsort(local, kind="stable"), np.argsort(glob, kind="stable")), (g_, e)
    rng = np.random.default_rng(17)
    tokens = set(rng.choice(wl.N, size=min(wl.N, 96), replace=False).tolist())
    for a, b in zip(cuts[:-1], cuts[1:]):
        tokens |= {a, b - 1}
    tokens = np.array(sorted(tokens))
    ref = oracle.forward(inp.x, inp.W_g, inp.b_g, inp.noise, wl.sigma, wl.k, wl.cf, inp.W_up, inp.W_down,
                         logits=lg, tokens=tokens, nthreads=8)
    yh = values(to_host_bits(y))[tokens]
    err = rel_err(yh, ref["y"])
    assert err <= TOL[wl.dtype], f"sharded output vs oracle: {err:.3g}"
    sig = bf16_error_sigma(inp, wl, tokens, idx, g, slot_ref, ref["y"])
    check_elementwise_bf16(yh, ref["y"], sig, "sharded")

pytestmark = pytest.mark.gpu

CASES = {
    "mixtral_small_3": (WORKLOADS["mixtral"].with_(N=3000, d=256, d_ff=512), 3),
    "fine_small_2": (WORKLOADS["fine"].with_(N=2500, d=128, d_ff=176), 2),
    "decode_4": (WORKLOADS["decode"].with_(N=64, d=512, d_ff=1024), 4),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_sharded_equals_unsharded(name):
    require_gpu()
    wl, G = CASES[name]
    case = Case(wl, seed=3)
    # reference: the same staged calls on the whole batch (the fused forward's
    # small-batch plan rounds the expert outputs differently)
    topk_r, gates_r, _ = moe.moe_route(case.x, case.W_g, wl.k, b_g=case.b_g, noise=case.noise, sigma=wl.sigma,
                                       want_logits=False)
    d_r = moe.moe_dispatch(topk_r, case.x, wl.E, wl.cf)
    out_r = moe.moe_expert_ffn(d_r["x_gathered"], d_r["offsets"], d_r["counts"], case.W_up, case.W_down)
    y_ref = moe.moe_combine(out_r, d_r["slot"], topk_r, d_r["offsets"], gates_r)
    cuts = [wl.N * g // G for g in range(G + 1)]
    routes, wss, counts = [], [], []
    for g in range(G):
        sl = slice(cuts[g], cuts[g + 1])
        noise = None if case.noise is None else case.noise[sl].contiguous()
        topk, gates, lg = moe.moe_route(case.x[sl].contiguous(), case.W_g, wl.k, b_g=case.b_g, noise=noise,
                                        sigma=wl.sigma)
        ws = moe.shard_workspace(cuts[g + 1] - cuts[g], wl.E, wl.k, case.x.device)
        routes.append((topk, gates, lg))
        wss.append(ws)
        counts.append(moe.moe_shard_count(topk, wl.E, ws))
    all_counts = torch.stack(counts)
    C = moe.capacity(wl.N, wl.E, wl.k, wl.cf)
    ys, slots = [], []
    host_counts = all_counts.cpu().numpy().astype(np.int64)
    for g in range(G):
        base = moe.moe_shard_base(all_counts, g)
        expect = np.zeros((wl.k, wl.E), dtype=np.int64)
        for j in range(wl.k):
            expect[j] = host_counts[:, :j, :].sum(axis=(0, 1)) + host_counts[:g, j, :].sum(axis=0)
        assert np.array_equal(base.cpu().numpy(), expect)
        topk, gates, _ = routes[g]
        xs = case.x[cuts[g]:cuts[g + 1]].contiguous()
        d = moe.moe_shard_dispatch(topk, xs, wl.E, C, counts[g], base, wss[g])
        out = moe.moe_expert_ffn(d["x_gathered"], d["offsets"], d["counts"], case.W_up, case.W_down)
        ys.append(moe.moe_combine(out, d["slot"], topk, d["offsets"], gates))
        slots.append(d["slot"])
        # kept rows are numbered 0..counts[e]-1 per expert inside the shard
        s, c = d["slot"].cpu().numpy(), d["counts"].cpu().numpy()
        tk = topk.cpu().numpy()
        for e in range(wl.E):
            got = np.sort(s[(tk == e) & (s >= 0)])
            assert np.array_equal(got, np.arange(c[e]))
    torch.cuda.synchronize()
    y = torch.cat(ys)
    assert torch.equal(y.view(torch.int16), y_ref.view(torch.int16))
    dropped = torch.cat(slots) < 0
    assert torch.equal(dropped, d_r["slot"] < 0)
    lg = torch.cat([r[2] for r in routes]).cpu().numpy()
    check_shards_against_oracle(case, cuts, [r[0].cpu().numpy() for r in routes],
                                [s_.cpu().numpy() for s_ in slots], y, lg)
