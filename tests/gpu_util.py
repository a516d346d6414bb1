"""Helpers for the GPU parity tests: move seeded inputs to the device, run the
CUDA path through the C ABI, and compare with the CPU oracle."""
from __future__ import annotations

import os

import numpy as np
import torch

import oracle
from sparse_mixture_experts_noisy_b200 import moe
from sparse_mixture_experts_noisy_b200.synth import BF16, make_inputs, bf16_bits_to_f32

# Output tolerance: max |y - y_oracle| / max |y_oracle| (the layer's stated bar).
TOL = {"f32": 1e-5, "bf16": 2e-2}
NTHREADS = max(1, min(32, len(os.sched_getaffinity(0))))


def require_gpu():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    moe.load_library()


def to_dev(a: np.ndarray | None, dtype: str | None = None):
    if a is None:
        return None
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def to_host_bits(t: torch.Tensor) -> np.ndarray:
    """bf16 -> uint16 bit patterns, fp32 -> float32."""
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def values(a: np.ndarray) -> np.ndarray:
    return bf16_bits_to_f32(a).astype(np.float64) if a.dtype == np.uint16 else a.astype(np.float64)


class Case:
    """Device copies of one workload's inputs."""

    def __init__(self, wl, seed=0):
        self.wl = wl
        self.inp = make_inputs(wl, seed)
        i = self.inp
        self.x = to_dev(i.x)
        self.W_g = to_dev(i.W_g)
        self.b_g = to_dev(i.b_g)
        self.noise = to_dev(i.noise)
        self.W_up = to_dev(i.W_up)
        self.W_down = to_dev(i.W_down)

    def forward(self, intermediates=True):
        wl = self.wl
        return moe.moe_forward(self.x, self.W_g, self.W_up, self.W_down, wl.k, wl.cf, b_g=self.b_g,
                               noise=self.noise, sigma=wl.sigma, intermediates=intermediates)

    def oracle_from_logits(self, logits: np.ndarray, tokens=None):
        i, wl = self.inp, self.wl
        return oracle.forward(i.x, i.W_g, i.b_g, i.noise, wl.sigma, wl.k, wl.cf, i.W_up, i.W_down,
                              logits=logits, tokens=tokens, nthreads=NTHREADS)


def rel_err(y: np.ndarray, ref: np.ndarray) -> float:
    scale = float(np.max(np.abs(ref))) if ref.size else 0.0
    if scale == 0.0:
        return float(np.max(np.abs(y))) if y.size else 0.0
    return float(np.max(np.abs(y - ref))) / scale


def check_routing(case: Case, inter, logits_tol=None):
    """Routing bit-exact given the GPU's fp32 logits: top-k, slots, counts;
    logits within fp32 accumulation error of the oracle's; gates within 2e-6."""
    wl, i = case.wl, case.inp
    lg = inter["logits"].cpu().numpy()
    ref_lg = oracle.router_logits(i.x, i.W_g, i.b_g)
    # fp32 summation error bound for a depth-(d/8 + 16) accumulation of the
    # products, plus one rounding of the result and the bias add
    absdot = np.abs(values(i.x)) @ np.abs(i.W_g.astype(np.float64)).T
    eps = 2.0 ** -24
    bound = (wl.d / 8 + 16) * eps * absdot + 2 * eps * np.abs(ref_lg) + 1e-30
    if logits_tol is not None:
        bound = np.maximum(bound, logits_tol)
    err = np.abs(lg.astype(np.float64) - ref_lg.astype(np.float64))
    assert np.all(err <= bound), f"logits off by up to {float(np.max(err / bound)):.3g} x the bound"
    idx, g = oracle.route_from_logits(lg, wl.k, i.noise, wl.sigma)
    gpu_idx = inter["topk_idx"].cpu().numpy()
    assert np.array_equal(gpu_idx, idx), "top-k differs from the oracle on identical logits"
    np.testing.assert_allclose(inter["gates"].cpu().numpy(), g, rtol=0, atol=2e-6)
    C = oracle.capacity(wl.N, wl.E, wl.k, wl.cf)
    slot, counts = oracle.assign_slots(idx, wl.E, C)
    assert np.array_equal(inter["slot"].cpu().numpy(), slot), "slots differ from the oracle"
    assert np.array_equal(inter["counts"].cpu().numpy(), counts), "counts differ from the oracle"
    return lg, idx, g, slot, counts


# ---------------------------------------------------------------------------
# Per-element check of the bf16 path.
#
# The max-normalised error above cannot see a wrong element that is small
# next to the row maximum.  This check bounds every element by the rounding
# the bf16 path performs, as a statistical model: the hidden activations H are
# rounded to bf16 after the activation, each expert output O to bf16 (in the
# prefill plan), and y to bf16; the fp32 accumulations are far finer and are
# covered by a tiny absolute floor.  A round-to-nearest bf16 error of a value v
# is at most 2^-8 |v| and its variance at most (2^-8)^2 v^2 / 3 (a uniform
# error on half an ulp), so for element i of token t
#
#   var_i = (2^-16 / 3) * ( sum_j g_j^2 [ sum_f W_down[e_j][i, f]^2 H_jf^2 + O_ji^2 ] + y_i^2 )
#
# and the test requires |y_i - y_oracle_i| <= Z_MAX * sqrt(var_i) + floor.  The
# model only over-estimates the variance, and with Z_MAX = 8 a correct
# element fails with a probability far below 1e-12.  An element that is wrong
# by more than a few percent of the row's typical magnitude sits hundreds of
# sigmas out, whatever its own size.
U_BF16 = 2.0 ** -8
Z_MAX = 8.0


def bf16_error_sigma(inp, wl, tokens, idx, g, slot, y_ref):
    """sigma_i of the model above for the rows `tokens` (y_ref: the oracle's
    float64 rows for those tokens, same order).  Uses ReLU experts without
    biases, the layer the parity tests run."""
    tokens = np.asarray(tokens)
    x = values(inp.x)[tokens].astype(np.float32)
    var = np.zeros((len(tokens), wl.d))
    u2 = U_BF16 * U_BF16 / 3.0
    idx_t, slot_t, g_t = idx[tokens], slot[tokens], g[tokens].astype(np.float64)
    for e in range(wl.E):
        sel_t, sel_j = np.nonzero((idx_t == e) & (slot_t >= 0))
        if len(sel_t) == 0:
            continue
        wu = bf16_bits_to_f32(inp.W_up[e]) if inp.W_up.dtype == np.uint16 else inp.W_up[e].astype(np.float32)
        wd = bf16_bits_to_f32(inp.W_down[e]) if inp.W_down.dtype == np.uint16 else inp.W_down[e].astype(np.float32)
        H = np.maximum(x[sel_t] @ wu.T, 0.0)
        O = (H @ wd.T).astype(np.float64)
        S2 = ((H * H) @ (wd * wd).T).astype(np.float64)
        gg = g_t[sel_t, sel_j] ** 2
        np.add.at(var, sel_t, gg[:, None] * u2 * (S2 + O * O))
    var += u2 * y_ref * y_ref
    return np.sqrt(var)


def check_elementwise_bf16(y: np.ndarray, y_ref: np.ndarray, sigma: np.ndarray, what: str = "") -> float:
    """Every element within Z_MAX sigma of the oracle (plus a floor of 2^-20 of
    the largest |y_ref| for the fp32 accumulations).  Returns the largest
    |error| / sigma seen."""
    floor = 2.0 ** -20 * (float(np.max(np.abs(y_ref))) if y_ref.size else 0.0)
    err = np.abs(y - y_ref)
    bad = err > Z_MAX * sigma + floor
    ratio = float(np.max(err / np.maximum(sigma, 1e-300))) if y.size else 0.0
    if np.any(bad):
        t, i = np.unravel_index(int(np.argmax(np.where(bad, err / np.maximum(sigma, 1e-300), 0))), err.shape)
        raise AssertionError(f"{what}: {int(bad.sum())} elements outside {Z_MAX} sigma of the rounding model; "
                             f"worst row {t} col {i}: got {y[t, i]:.6g}, oracle {y_ref[t, i]:.6g}, "
                             f"sigma {sigma[t, i]:.3g}")
    return ratio
