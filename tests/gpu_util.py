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
