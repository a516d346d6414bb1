"""Expert-parallel layer (ep.py) with its ranks run one after another on one
GPU (needs a B200).  The all-gathers are emulated by stacking each rank's
table and the all-to-alls by copying each rank's send views into the
receivers' buffers, which is all the collectives do.  The result must match
the same batch run as one unsharded call: the same slots and drop set bit for
bit, and the output within the bf16 tolerance (a rank's expert calls see
fewer rows, which can choose a different tile plan).  It is also checked
against the oracle on the whole batch, replaying the GPU's fp32 logits:
top-k, drop set and queue order bit for bit, a sample of token outputs within
the bf16 tolerance and the per-element rounding model."""
import numpy as np
import pytest
import torch

from sparse_mixture_experts_noisy_b200 import ep, moe
from sparse_mixture_experts_noisy_b200.synth import WORKLOADS
from tests.gpu_util import Case, TOL, rel_err, require_gpu, to_host_bits, values
from tests.test_gpu_shard import check_shards_against_oracle

pytestmark = pytest.mark.gpu

CASES = {
    "mixtral_small_G2": (WORKLOADS["mixtral"].with_(N=2048, d=256, d_ff=512), 2),
    "mixtral_small_G4": (WORKLOADS["mixtral"].with_(N=3000, d=256, d_ff=384), 4),
    "fine_small_G4": (WORKLOADS["fine"].with_(N=2500, d=128, d_ff=176), 4),
    "decode_G8": (WORKLOADS["decode"].with_(N=64, d=512, d_ff=1024), 8),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_expert_parallel_matches_unsharded(name):
    require_gpu()
    wl, G = CASES[name]
    case = Case(wl, seed=5)
    E, k, d = wl.E, wl.k, wl.d
    # the unsharded reference through the staged calls
    topk_r, gates_r, _ = moe.moe_route(case.x, case.W_g, k, b_g=case.b_g, noise=case.noise, sigma=wl.sigma,
                                       want_logits=False)
    d_r = moe.moe_dispatch(topk_r, case.x, E, wl.cf)
    out_r = moe.moe_expert_ffn(d_r["x_gathered"], d_r["offsets"], d_r["counts"], case.W_up, case.W_down)
    y_ref = moe.moe_combine(out_r, d_r["slot"], topk_r, d_r["offsets"], gates_r)

    cuts = [wl.N * g // G for g in range(G + 1)]
    xs = [case.x[cuts[g]:cuts[g + 1]].contiguous() for g in range(G)]
    ns = [None if case.noise is None else case.noise[cuts[g]:cuts[g + 1]].contiguous() for g in range(G)]
    st = [ep.step_route(xs[g], case.W_g, k, E, b_g=case.b_g, noise=ns[g], sigma=wl.sigma) for g in range(G)]
    all_counts = torch.stack([s["counts_je"] for s in st])
    for g in range(G):
        ep.step_dispatch(st[g], xs[g], E, k, wl.cf, wl.N, all_counts, g)
    kept_all = torch.stack([s["dispatch"]["counts"] for s in st]).cpu().tolist()
    plans = [ep.ep_plan(kept_all, G, g) for g in range(G)]
    for a in range(G):
        for b in range(G):
            assert plans[a].send_splits[b] == plans[b].recv_splits[a]
    sends = [ep.step_send_views(st[g], plans[g]) for g in range(G)]
    recv = [ep.step_recv_buffers(plans[q], d, case.x.dtype, case.x.device) for q in range(G)]
    for q in range(G):
        for s in range(G):
            recv[q][1][s].copy_(sends[s][q])
    outs = []
    for q in range(G):
        lo, hi = ep.expert_range(E, G, q)
        outs.append(ep.step_experts(plans[q], recv[q][0], case.W_up[lo:hi], case.W_down[lo:hi]))
    backs = [ep.step_return_views(st[g], plans[g]) for g in range(G)]
    for g in range(G):
        for q in range(G):
            backs[g][q].copy_(outs[q][g][:plans[q].recv_splits[g]])
    y = torch.cat([ep.step_combine(st[g]) for g in range(G)])
    torch.cuda.synchronize()
    slots = torch.cat([s["dispatch"]["slot"] for s in st])
    assert torch.equal(slots < 0, d_r["slot"] < 0)
    kept_tot = np.sum(kept_all, axis=0)
    assert np.array_equal(kept_tot, d_r["counts"].cpu().numpy())
    err = rel_err(values(to_host_bits(y)), values(to_host_bits(y_ref)))
    assert err <= TOL[wl.dtype], f"{name}: {err:.3g}"
    lg = torch.cat([moe.moe_route(xs[g], case.W_g, k, b_g=case.b_g, noise=ns[g], sigma=wl.sigma)[2]
                    for g in range(G)]).cpu().numpy()
    check_shards_against_oracle(case, cuts, [s["topk"].cpu().numpy() for s in st],
                                [s["dispatch"]["slot"].cpu().numpy() for s in st], y, lg)
