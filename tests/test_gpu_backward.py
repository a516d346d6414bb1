"""The backward pass on the GPU against the oracle's (needs a B200).

A staged forward (moe_route, moe_dispatch, moe_expert_ffn_train, moe_combine)
followed by moe_backward, against oracle.backward on the same routing: the
oracle replays the GPU's fp32 logits (so top-k and slots are the GPU's, which
are checked bit for bit first) and the GPU's ReLU decisions ([H > 0] of each
kept pair), the two discrete decisions floating point makes on the way.
Bars: fp32 storage 1e-5, bf16 2e-2, as max |got - ref| / max |ref| per token
row of dx, per expert of dW_up and dW_down, and over dW_g and db_g.  An
expert without rows must get exactly zero weight gradients.  The full-size
case (the nanoMoE-shaped layer) is checked on sampled rows and columns that
the oracle computes one by one, and on all of dW_g and db_g."""
import math
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import oracle
from sparse_mixture_experts_noisy_b200 import moe
from sparse_mixture_experts_noisy_b200.synth import BF16, F32, WORKLOADS, Workload, f32_to_bf16_bits, normal_f32
from tests.gpu_util import NTHREADS, TOL, Case, rel_err, require_gpu, to_dev, to_host_bits, values

pytestmark = pytest.mark.gpu

W = WORKLOADS
CASES = {
    # router bias +1 on expert 0: capacity drops (a dropped choice still gets a score gradient)
    "mixtral_small": W["mixtral"].with_(N=1536, d=512, d_ff=1024),
    # ragged weight tiles in every GEMM, and expert row counts that end inside K blocks
    "ragged": W["mixtral"].with_(N=1000, d=640, d_ff=720),
    # 64 experts, k = 6, supplied noise
    "fine_small": W["fine"].with_(N=2048, d=256, d_ff=176),
    # few tokens per expert: the forward's decode plan
    "decode_small": W["decode"].with_(N=64, d=512, d_ff=1024),
    # k = 1: the router gets no gradient
    "switch_k1": W["nano"].with_(N=700, d=128, d_ff=256, k=1, cf=1.0, wg_std=0.1),
    # 16 experts for 6 tokens with 2 choices: at least 4 experts get no rows
    "empty_experts": W["decode"].with_(N=6, d=256, d_ff=256, E=16, k=2),
    # fp32 storage: CUDA-core kernels throughout, drops and noise
    "f32_drops": Workload("f32_drops", F32, N=300, d=40, E=6, d_ff=50, k=3, sigma=0.5, cf=0.8,
                          w_std=0.3, wg_std=0.3),
    # bf16 rows that are not 16-byte multiples: CUDA-core kernels in bf16
    "bf16_unaligned": Workload("bf16_unaligned", BF16, N=200, d=36, E=5, d_ff=20, k=2, sigma=0.0, cf=1.0,
                               w_std=0.2, wg_std=0.3),
    "toy": W["toy"],
}


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def make_dy(wl, seed):
    dy = normal_f32(seed + 5, (wl.N, wl.d), 1.0)
    return f32_to_bf16_bits(dy) if wl.dtype == BF16 else dy


def staged_train_step(case, dy_host):
    """Forward through the staged calls, then the backward.  Returns the GPU
    tensors of both."""
    wl = case.wl
    topk, gates, logits = moe.moe_route(case.x, case.W_g, wl.k, b_g=case.b_g, noise=case.noise, sigma=wl.sigma)
    dsp = moe.moe_dispatch(topk, case.x, wl.E, wl.cf)
    out, H = moe.moe_expert_ffn_train(dsp["x_gathered"], dsp["offsets"], dsp["counts"], case.W_up, case.W_down)
    y = moe.moe_combine(out, dsp["slot"], topk, dsp["offsets"], gates)
    dy = to_dev(dy_host)
    g = moe.moe_backward(case.x, case.W_g, case.W_up, case.W_down, wl.k, topk, gates, dsp["slot"], dsp["offsets"],
                         dsp["counts"], dsp["x_gathered"], H, out, dy)
    torch.cuda.synchronize()
    code, word = moe.check_status(g["ws"])
    assert code == 0, hex(word)
    return dict(topk=topk, gates=gates, logits=logits, y=y, H=H, **dsp), g


def replayed_decisions(case, fw):
    """The oracle's view of the GPU's routing: noisy scores s from the GPU's
    logits, top-k and slots (checked equal to the GPU's), and the ReLU mask
    [N, k, d_ff] of the kept pairs from the GPU's H."""
    wl, inp = case.wl, case.inp
    lg = fw["logits"].cpu().numpy()
    idx, _, s = oracle.route_from_logits(lg, wl.k, inp.noise, wl.sigma, return_scores=True)
    assert np.array_equal(idx, fw["topk"].cpu().numpy())
    slot, counts = oracle.assign_slots(idx, wl.E, oracle.capacity(wl.N, wl.E, wl.k, wl.cf))
    assert np.array_equal(slot, fw["slot"].cpu().numpy())
    assert np.array_equal(counts, fw["counts"].cpu().numpy())
    H = values(to_host_bits(fw["H"]))
    offs = fw["offsets"].cpu().numpy()
    mask = np.zeros((wl.N, wl.k, wl.d_ff), dtype=np.uint8)
    ts, js = np.nonzero(slot >= 0)
    rows = offs[idx[ts, js]] + slot[ts, js]
    mask[ts, js] = (H[rows] > 0).astype(np.uint8)
    return idx, slot, counts, s, mask


def _rows_err(got, ref):
    """Largest per-row max-normalised error."""
    worst = 0.0
    for a, b in zip(got, ref):
        worst = max(worst, rel_err(a, b))
    return worst


@pytest.mark.parametrize("name", sorted(CASES))
def test_backward_small(name):
    wl = CASES[name]
    case = Case(wl, seed=2)
    dy = make_dy(wl, 2)
    fw, g = staged_train_step(case, dy)
    idx, slot, counts, s, mask = replayed_decisions(case, fw)
    i = case.inp
    ref = oracle.backward(i.x, i.W_g, i.W_up, i.W_down, s, idx, slot, values(dy), relu_mask=mask)
    tol = TOL[wl.dtype]
    dx = values(to_host_bits(g["dx"]))
    err = _rows_err(dx, ref["dx"])
    assert err <= tol, f"dx: {err:.3g}"
    for key in ("dW_up", "dW_down"):
        got = g[key].cpu().numpy().astype(np.float64)
        for e in range(wl.E):
            if counts[e] == 0:
                assert np.all(got[e] == 0.0), f"{key}[{e}] of an expert without rows"
                continue
            err = rel_err(got[e], ref[key][e])
            assert err <= tol, f"{key}[{e}]: {err:.3g} (rows {counts[e]})"
    for key in ("dW_g", "db_g"):
        got = g[key].cpu().numpy().astype(np.float64)
        err = rel_err(got, ref[key])
        assert err <= tol, f"{key}: {err:.3g}"
    if wl.k == 1:
        assert np.all(g["dW_g"].cpu().numpy() == 0.0) and np.all(g["db_g"].cpu().numpy() == 0.0)
    if name == "empty_experts":
        assert np.any(counts == 0)
    if name == "mixtral_small":
        assert np.any(slot < 0)


def test_backward_deterministic():
    wl = CASES["fine_small"]
    case = Case(wl, seed=4)
    dy = make_dy(wl, 4)
    _, a = staged_train_step(case, dy)
    _, b = staged_train_step(case, dy)
    for key in ("dx", "dW_g", "db_g", "dW_up", "dW_down"):
        ta, tb = a[key], b[key]
        if ta.dtype == torch.bfloat16:
            ta, tb = ta.view(torch.int16), tb.view(torch.int16)
        assert torch.equal(ta, tb), key


def test_backward_full_size_nano():
    """The nanoMoE-shaped layer at full size (N=8192, d=768, E=8, d_ff=3072):
    dx on 64 sampled tokens, rows of dW_up and columns of dW_down at tile
    edges and random places of every expert, all of dW_g and db_g."""
    wl = WORKLOADS["nano"]
    case = Case(wl, seed=0)
    dy = make_dy(wl, 0)
    fw, g = staged_train_step(case, dy)
    idx, slot, counts, s, mask = replayed_decisions(case, fw)
    rng = np.random.default_rng(5)
    tokens = np.array(sorted(set(rng.choice(wl.N, 62, replace=False).tolist()) | {0, wl.N - 1}))
    ef = []
    for e in range(wl.E):
        for f in {0, 127, 128, 255, 256, wl.d_ff - 1, int(rng.integers(wl.d_ff))}:
            ef.append((e, f))
    i = case.inp
    ref = oracle.backward_sampled(i.x, i.W_g, i.W_up, i.W_down, s, idx, slot, values(dy), tokens, ef,
                                  relu_mask=mask, nthreads=NTHREADS)
    tol = TOL[wl.dtype]
    dx = values(to_host_bits(g["dx"]))[tokens]
    err = _rows_err(dx, ref["dx_rows"])
    assert err <= tol, f"dx: {err:.3g}"
    dWu = g["dW_up"].cpu().numpy().astype(np.float64)
    dWd = g["dW_down"].cpu().numpy().astype(np.float64)
    for q, (e, f) in enumerate(ef):
        scale_u = float(np.max(np.abs(ref["dW_up_rows"][[p for p, (ee, _) in enumerate(ef) if ee == e]])))
        scale_d = float(np.max(np.abs(ref["dW_down_cols"][[p for p, (ee, _) in enumerate(ef) if ee == e]])))
        eu = float(np.max(np.abs(dWu[e, f, :] - ref["dW_up_rows"][q]))) / scale_u
        ed = float(np.max(np.abs(dWd[e, :, f] - ref["dW_down_cols"][q]))) / scale_d
        assert eu <= tol and ed <= tol, (e, f, eu, ed)
    for key in ("dW_g", "db_g"):
        err = rel_err(g[key].cpu().numpy().astype(np.float64), ref[key])
        assert err <= tol, f"{key}: {err:.3g}"


WGRAD_CHILD = r"""
import sys, numpy as np, torch
sys.path.insert(0, {root!r})
from sparse_mixture_experts_noisy_b200.synth import WORKLOADS
from tests.gpu_util import Case
from tests.test_gpu_backward import CASES, make_dy, staged_train_step
case = Case(CASES[{name!r}], seed=3)
_, g = staged_train_step(case, make_dy(case.wl, 3))
np.save({out_u!r}, g["dW_up"].cpu().numpy())
np.save({out_d!r}, g["dW_down"].cpu().numpy())
"""


@pytest.mark.parametrize("name", ["ragged", "empty_experts", "fine_small"])
def test_wgrad_one_cta_form_matches_pairs(name, tmp_path):
    """The weight gradients on CTA pairs (the default) and on single CTAs
    (MOE_WGRAD_PAIR=0, in a child process) agree to fp32 summation-order
    rounding, expert by expert, and both give exact zeros to experts without
    rows."""
    case = Case(CASES[name], seed=3)
    _, g = staged_train_step(case, make_dy(case.wl, 3))
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out_u, out_d = str(tmp_path / "u.npy"), str(tmp_path / "d.npy")
    code = WGRAD_CHILD.format(root=root, name=name, out_u=out_u, out_d=out_d)
    r = subprocess.run([sys.executable, "-c", code], cwd=root, env=dict(os.environ, MOE_WGRAD_PAIR="0"),
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    for key, path in (("dW_up", out_u), ("dW_down", out_d)):
        pair = g[key].cpu().numpy().astype(np.float64)
        single = np.load(path).astype(np.float64)
        for e in range(case.wl.E):
            if not np.any(single[e]):
                assert not np.any(pair[e]), f"{key}[{e}]"
                continue
            err = rel_err(pair[e], single[e])
            assert err <= 1e-5, f"{key}[{e}]: {err:.3g}"
