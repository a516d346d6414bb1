"""moe_load_stats on the GPU against the oracle (needs a B200): per-expert
load before the capacity cut, used = min(load, C) ("nanoMoEの深層解剖" slide
14's used_capacity, equal to moe_dispatch's counts) and the gate mass in exact
units of 2^-32 — all bit for bit."""
import numpy as np
import pytest
import torch

import oracle
from sparse_mixture_experts_noisy_b200 import moe
from sparse_mixture_experts_noisy_b200.synth import BF16, Workload, make_inputs
from tests.gpu_util import require_gpu, to_dev

pytestmark = pytest.mark.gpu

CASES = {
    "mixtral_bias_drops": Workload("ls_m", BF16, N=16384, d=256, E=8, d_ff=16, k=2, sigma=0.0, cf=1.25, bias0=1.0),
    "fine_noisy": Workload("ls_f", BF16, N=5000, d=128, E=64, d_ff=16, k=6, sigma=1.0, cf=1.0),
    "one_choice": Workload("ls_1", BF16, N=777, d=64, E=5, d_ff=16, k=1, sigma=0.5, cf=0.6, wg_std=0.5),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_load_stats_match_oracle(name):
    require_gpu()
    wl = CASES[name]
    inp = make_inputs(wl, seed=31, weights=False)
    x, W_g, b_g, noise = to_dev(inp.x), to_dev(inp.W_g), to_dev(inp.b_g), to_dev(inp.noise)
    topk, gates, _ = moe.moe_route(x, W_g, wl.k, b_g=b_g, noise=noise, sigma=wl.sigma, want_logits=False)
    st = moe.moe_load_stats(topk, wl.E, wl.cf, gates=gates)
    plain = moe.moe_load_stats(topk, wl.E, wl.cf)
    disp = moe.moe_dispatch(topk, x, wl.E, wl.cf)
    torch.cuda.synchronize()
    C = oracle.capacity(wl.N, wl.E, wl.k, wl.cf)
    load, used, imp = oracle.load_stats(topk.cpu().numpy(), wl.E, C, gates.cpu().numpy())
    assert np.array_equal(st["load"].cpu().numpy(), load)
    assert np.array_equal(st["used"].cpu().numpy(), used)
    assert np.array_equal(st["importance"].cpu().numpy(), imp)
    assert np.array_equal(st["used"].cpu().numpy(), disp["counts"].cpu().numpy())
    assert plain["importance"] is None
    assert torch.equal(plain["load"], st["load"]) and torch.equal(plain["used"], st["used"])
    assert int(st["load"].sum()) == wl.N * wl.k


def test_load_stats_empty_batch():
    require_gpu()
    topk = torch.empty((0, 2), dtype=torch.int32, device="cuda")
    st = moe.moe_load_stats(topk, 4, 1.0)
    torch.cuda.synchronize()
    assert st["load"].tolist() == [0, 0, 0, 0] and st["used"].tolist() == [0, 0, 0, 0]
