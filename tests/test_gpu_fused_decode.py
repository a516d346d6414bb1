"""The single-launch small-batch layer (decode_fused.cu) on the GPU (needs a B200).

With moe_set_fused_small_batch(1), moe_forward runs batches of at most 64
bf16 tokens (E <= 16) as one cooperative kernel.  It must
  - match the oracle (routing bit for bit on the GPU's logits, the output
    within the bf16 bar and the per-element rounding model),
  - give exactly the output of the separate kernels of the decode plan (the
    same arithmetic in the same order; they run in a child process with
    MOE_FUSED_DECODE=0),
  - count as one launch, replay from a CUDA graph bit for bit, and leave a
    clean status word."""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

from sparse_mixture_experts_noisy_b200 import moe
from sparse_mixture_experts_noisy_b200.synth import WORKLOADS
from tests.gpu_util import (Case, TOL, bf16_error_sigma, check_elementwise_bf16, check_routing, rel_err,
                            require_gpu, to_host_bits, values)

pytestmark = pytest.mark.gpu

W = WORKLOADS
CASES = {
    "decode_small": W["decode"].with_(N=64, d=512, d_ff=1024),
    "decode_ragged": W["decode"].with_(N=37, d=256, d_ff=320, k=3),
    "one_token": W["decode"].with_(N=1, d=256, d_ff=512),
    # noise, router bias and a capacity cut
    "noisy_capped": W["mixtral"].with_(N=48, d=384, d_ff=640, sigma=0.7, cf=0.5),
    # 16 experts for 20 tokens: experts without tokens
    "empty_experts": W["decode"].with_(N=20, d=256, d_ff=256, E=16, k=2),
    "decode_full": W["decode"],
}

CHILD = r"""
import sys, numpy as np, torch
sys.path.insert(0, {root!r})
from sparse_mixture_experts_noisy_b200 import moe
from sparse_mixture_experts_noisy_b200.synth import WORKLOADS
from tests.gpu_util import Case
wl = WORKLOADS[{base!r}].with_(**{kw!r})
case = Case(wl, seed={seed})
assert moe.forward_launches(wl.N, wl.d, wl.E, wl.d_ff, wl.k, wl.cf, case.x.dtype) > 1
y = case.forward(intermediates=False)
torch.cuda.synchronize()
np.save({out!r}, y.view(torch.int16).cpu().numpy())
"""


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()
    prev = moe.set_fused_small_batch(True)
    yield
    moe.set_fused_small_batch(prev)


def _kw(wl):
    base = {"decode_full": "decode"}.get(wl.name, wl.name)
    ref = W[base]
    kw = {f: getattr(wl, f) for f in ("N", "d", "E", "d_ff", "k", "sigma", "cf") if getattr(wl, f) != getattr(ref, f)}
    return base, kw


@pytest.mark.parametrize("name", sorted(CASES))
def test_fused_small_batch_layer(name, tmp_path):
    wl = CASES[name]
    assert moe.forward_launches(wl.N, wl.d, wl.E, wl.d_ff, wl.k, wl.cf, torch.bfloat16) == 1
    case = Case(wl, seed=6)
    y, inter = case.forward()
    torch.cuda.synchronize()
    lg, idx, g, slot, counts = check_routing(case, inter)
    ref = case.oracle_from_logits(lg)
    yh = values(to_host_bits(y))
    err = rel_err(yh, ref["y"])
    assert err <= TOL["bf16"], f"{name}: {err:.3g}"
    sig = bf16_error_sigma(case.inp, wl, np.arange(wl.N), idx, g, slot, ref["y"])
    check_elementwise_bf16(yh, ref["y"], sig, name)
    if name == "empty_experts":
        assert np.any(counts == 0)
    if name == "noisy_capped":
        assert np.any(slot < 0)
    # the separate kernels, in a child process that switches the fused kernel off
    base, kw = _kw(wl)
    out = str(tmp_path / "y.npy")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, MOE_FUSED_DECODE="0")
    code = CHILD.format(root=root, base=base, kw=kw, seed=6, out=out)
    r = subprocess.run([sys.executable, "-c", code], cwd=root, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    y_sep = np.load(out)
    assert np.array_equal(y.view(torch.int16).cpu().numpy(), y_sep), "fused and separate kernels differ"


def test_fused_layer_graph_replay_and_status():
    wl = CASES["decode_small"]
    case = Case(wl, seed=8)
    layer = moe.MoELayer(case.W_g, case.W_up, case.W_down, wl.k, wl.cf, b_g=case.b_g, sigma=wl.sigma)
    y_eager = layer(case.x, noise=case.noise).clone()
    g = moe.GraphedForward(layer, case.x.clone(), None if case.noise is None else case.noise.clone())
    for _ in range(3):
        y = g.replay()
    torch.cuda.synchronize()
    assert torch.equal(y.view(torch.int16), y_eager.view(torch.int16))
    # new inputs through the captured graph
    other = Case(wl, seed=9)
    g.x.copy_(other.x)
    y2 = g.replay().clone()
    y2_eager = layer(other.x)
    torch.cuda.synchronize()
    assert torch.equal(y2.view(torch.int16), y2_eager.view(torch.int16))
    assert moe.check_status(layer.workspace) == (0, 0)
