"""The per-element check of the bf16 path (tests/gpu_util.py), on the CPU.

A numpy emulation of the bf16 path's roundings (hidden activations, expert
outputs and y rounded to bf16, everything else in float32) stands in for the
GPU output.  It must pass the check against the oracle; the same output with
one small element made wrong must fail it, although the max-normalised bar of
2e-2 still passes.  This is what the per-element check adds."""
import numpy as np
import pytest

import oracle
from sparse_mixture_experts_noisy_b200.synth import WORKLOADS, bf16_bits_to_f32, f32_to_bf16_bits, make_inputs
from tests.gpu_util import TOL, bf16_error_sigma, check_elementwise_bf16, rel_err, values


def _bf16(a):
    return bf16_bits_to_f32(f32_to_bf16_bits(np.asarray(a, dtype=np.float32)))


def _emulated_bf16_path(inp, wl, idx, g, slot):
    x = values(inp.x).astype(np.float32)
    y = np.zeros((wl.N, wl.d), dtype=np.float32)
    for t in range(wl.N):
        for j in range(wl.k):
            if slot[t, j] < 0:
                continue
            e = idx[t, j]
            wu = bf16_bits_to_f32(inp.W_up[e])
            wd = bf16_bits_to_f32(inp.W_down[e])
            h = _bf16(np.maximum(wu @ x[t], 0.0))
            o = _bf16(wd @ h)
            y[t] += np.float32(g[t, j]) * o
    return _bf16(y).astype(np.float64)


@pytest.fixture(scope="module")
def setup():
    wl = WORKLOADS["mixtral"].with_(N=96, d=128, d_ff=256)
    inp = make_inputs(wl, seed=11)
    ref = oracle.forward(inp.x, inp.W_g, inp.b_g, inp.noise, wl.sigma, wl.k, wl.cf, inp.W_up, inp.W_down,
                         nthreads=2)
    idx, g, slot = ref["topk_idx"], ref["gates"], ref["slot"]
    y = _emulated_bf16_path(inp, wl, idx, g, slot)
    sig = bf16_error_sigma(inp, wl, np.arange(wl.N), idx, g, slot, ref["y"])
    return wl, ref, y, sig


def test_emulated_bf16_path_passes(setup):
    wl, ref, y, sig = setup
    assert rel_err(y, ref["y"]) <= TOL["bf16"]
    worst = check_elementwise_bf16(y, ref["y"], sig, "emulated")
    assert worst < 6.0


def test_a_wrong_small_element_is_caught(setup):
    wl, ref, y, sig = setup
    mx = float(np.max(np.abs(ref["y"])))
    # an element of about 1 % of the largest |y|, set to zero
    cand = np.argwhere((np.abs(ref["y"]) > 0.008 * mx) & (np.abs(ref["y"]) < 0.015 * mx))
    assert len(cand) > 0
    t, i = cand[0]
    bad = y.copy()
    bad[t, i] = 0.0
    assert rel_err(bad, ref["y"]) <= TOL["bf16"]          # the max-normalised bar misses it
    with pytest.raises(AssertionError):
        check_elementwise_bf16(bad, ref["y"], sig, "planted")
    # and a sign flip of a smaller one (the error is twice its size)
    cand = np.argwhere((np.abs(ref["y"]) > 0.005 * mx) & (np.abs(ref["y"]) < 0.009 * mx))
    t2, i2 = cand[len(cand) // 2]
    bad = y.copy()
    bad[t2, i2] = -bad[t2, i2]
    assert rel_err(bad, ref["y"]) <= TOL["bf16"]
    with pytest.raises(AssertionError):
        check_elementwise_bf16(bad, ref["y"], sig, "planted")
