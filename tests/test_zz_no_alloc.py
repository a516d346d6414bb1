"""moe_dispatch_noalloc, the dispatch entry point for callers that cannot
allocate device memory when they dispatch (a runtime that forbids cudaMalloc
after start-up, or a plug-in whose framework owns all device memory): it must
give exactly what moe_dispatch gives with a caller workspace, call after call,
although every call reuses the same fixed scratch array (needs a B200).

This file is collected last on purpose, so that a run stopping at the first
failure has already run every other test."""
import ctypes
import math

import numpy as np
import pytest
import torch

from sparse_mixture_experts_noisy_b200 import moe
from sparse_mixture_experts_noisy_b200.synth import WORKLOADS
from tests.gpu_util import Case, require_gpu, to_host_bits

pytestmark = pytest.mark.gpu

# Batches above 1024 tokens use the multi-block passes, i.e. the scratch
# array.  The larger batch (more blocks, more experts) goes first, so the
# smaller one that follows runs over the leftovers of a bigger call.
CALLS = [
    WORKLOADS["fine"].with_(N=5000, d=128, d_ff=64, E=16, k=3),
    WORKLOADS["mixtral"].with_(N=1500, d=256, d_ff=64),
]


def _dispatch_both(wl, seed):
    case = Case(wl, seed)
    topk, gates, _ = moe.moe_route(case.x, case.W_g, wl.k, b_g=case.b_g, noise=case.noise, sigma=wl.sigma)
    ref = moe.moe_dispatch(topk, case.x, wl.E, wl.cf)
    got = moe.moe_dispatch_noalloc(topk, case.x, wl.E, wl.cf)
    torch.cuda.synchronize()
    return ref, got


def _assert_same(got, ref):
    for key in ("slot", "counts", "offsets"):
        assert torch.equal(got[key], ref[key]), key
    kept = int(ref["offsets"][-1].item())
    assert kept > 0
    assert np.array_equal(to_host_bits(got["x_gathered"][:kept]), to_host_bits(ref["x_gathered"][:kept]))


def test_noalloc_dispatch_matches_workspace_dispatch_call_after_call():
    require_gpu()
    dropped = []
    for seed, wl in enumerate(CALLS):
        ref, first = _dispatch_both(wl, seed)
        _assert_same(first, ref)
        # the same batch again, straight after: byte for byte the same output
        _, again = _dispatch_both(wl, seed)
        _assert_same(again, ref)
        dropped.append(int((ref["slot"] < 0).sum().item()))
    assert dropped[1] > 0      # the +1 router bias overflows expert 0: drops are exercised
    # and the larger batch once more, after the smaller one
    ref, got = _dispatch_both(CALLS[0], 0)
    _assert_same(got, ref)


def test_noalloc_dispatch_rejects_batches_beyond_its_scratch():
    require_gpu()
    L = moe.load_library()
    # 2^22 tokens, k = 8, E = 256 needs far more than the fixed scratch; the
    # size check comes before anything touches the (dummy, aligned) pointers
    p = ctypes.c_void_p(1 << 20)
    code = L.moe_dispatch_noalloc(p, p, moe.MOE_BF16, 1 << 22, 64, 256, 8, math.inf, p, p, p, p, None)
    assert code == 1
    assert b"needs" in L.moe_last_error() and b"scratch" in L.moe_last_error()
