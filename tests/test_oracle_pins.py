"""The CPU oracle against facts fixed outside it (CPU only)."""
import math

import numpy as np
import pytest

import oracle
from tests import oracle_pins as P


@pytest.mark.parametrize("check", P.ALL_CHECKS, ids=lambda c: c.__name__)
def test_pin(check):
    check()


def test_toy_workload_runs_and_fixes_token0():
    """The walkthrough's input vector x = [1.20, -0.40, -0.80] is token 0 of
    the toy workload; its output is the gate-weighted sum of its two experts."""
    from sparse_mixture_experts_noisy_b200.synth import make_inputs
    inp = make_inputs("toy", seed=0)
    assert inp.x[0].tolist() == [np.float32(1.2), np.float32(-0.4), np.float32(-0.8)]
    out = oracle.forward(inp.x, inp.W_g, inp.b_g, inp.noise, 0.0, 2, math.inf, inp.W_up, inp.W_down)
    assert np.all(out["slot"] >= 0)            # cf = inf: nothing dropped
    x64 = inp.x.astype(np.float64)
    u64, w64 = inp.W_up.astype(np.float64), inp.W_down.astype(np.float64)
    ref = sum(float(out["gates"][0, j]) * P.np_expert(x64[0], u64, w64, out["topk_idx"][0, j])
              for j in range(2))
    np.testing.assert_allclose(out["y"][0], ref, rtol=1e-12, atol=1e-12)


def test_threads_do_not_change_results():
    from sparse_mixture_experts_noisy_b200.synth import make_inputs, WORKLOADS
    wl = WORKLOADS["nano"].with_(N=64, d=64, d_ff=96)
    inp = make_inputs(wl, seed=1)
    a = oracle.forward(inp.x, inp.W_g, inp.b_g, inp.noise, 0.0, wl.k, wl.cf, inp.W_up, inp.W_down,
                       nthreads=1)
    b = oracle.forward(inp.x, inp.W_g, inp.b_g, inp.noise, 0.0, wl.k, wl.cf, inp.W_up, inp.W_down,
                       nthreads=5)
    assert np.array_equal(a["y"], b["y"])
