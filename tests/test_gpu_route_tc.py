"""The tensor-core router against the oracle (needs a B200).

bf16 tokens (d a multiple of 8, at most 160 experts) route on the tensor
cores at every batch size, with each fp32 router weight cut into three bf16
parts and K cut into up to 8 pieces summed by the CTAs of a cluster
("Mixture of Experts (MoE)
12段階極小ビジュアル解剖シミュレーター" STEP 2-6; "nanoMoEの深層解剖" slides
11-13: the router runs in fp32).  The bar is the one every router path meets:
logits within fp32 accumulation error of the oracle's exact dot products,
and, given the GPU's logits, the oracle's KeepTopK (ties to the lower expert
index) and softmax.

The shapes cover one and two MMA column chunks (3 * E_pad up to 480 rows of
B), odd expert counts, a K tail shorter than a 64-wide block, a last token
tile of one row, exact ties between experts, and the CUDA-core fallback above
160 experts or 32 choices."""
import numpy as np
import pytest
import torch

import oracle
from sparse_mixture_experts_noisy_b200 import moe
from sparse_mixture_experts_noisy_b200.synth import BF16, Workload, make_inputs
from tests.gpu_util import require_gpu, to_dev, values

pytestmark = pytest.mark.gpu


def _wl(name, N, d, E, k, sigma, wg_std=0.02, bias0=0.0):
    return Workload(name, BF16, N=N, d=d, E=E, d_ff=16, k=k, sigma=sigma, cf=1.0, wg_std=wg_std, bias0=bias0)


SHAPES = {
    "e8_mixtral_d": _wl("e8", N=1500, d=4096, E=8, k=2, sigma=0.0, bias0=1.0),
    "e8_decode": _wl("e8d", N=64, d=4096, E=8, k=2, sigma=0.0),
    "e8_one_token": _wl("e8one", N=1, d=1000, E=8, k=2, sigma=1.0, wg_std=0.05),
    "e64_fine_d": _wl("e64", N=2085, d=2048, E=64, k=6, sigma=1.0),
    "e5_odd_ktail": _wl("e5", N=1025, d=72, E=5, k=3, sigma=0.5, wg_std=0.3),
    "e33_k1": _wl("e33", N=1111, d=136, E=33, k=1, sigma=0.0, wg_std=0.1),
    "e96_two_chunks": _wl("e96", N=1300, d=520, E=96, k=4, sigma=1.0, wg_std=0.05),
    "e160_largest": _wl("e160", N=1200, d=256, E=160, k=8, sigma=0.0, wg_std=1.0),
    "e161_fallback": _wl("e161", N=1050, d=64, E=161, k=2, sigma=0.0, wg_std=1.0),
    "k33_fallback": _wl("k33", N=1100, d=64, E=40, k=33, sigma=0.5, wg_std=1.0),
    # enough tiles for the persistent form
    "e64_persistent": _wl("e64p", N=20000, d=2048, E=64, k=6, sigma=1.0),
    "e80_persistent": _wl("e80p", N=40000, d=1024, E=80, k=4, sigma=0.5, wg_std=0.05, bias0=0.5),
}


def _check(wl, inp, idx, gates, lg):
    ref_lg = oracle.router_logits(inp.x, inp.W_g, inp.b_g)
    absdot = np.abs(values(inp.x)) @ np.abs(inp.W_g.astype(np.float64)).T
    eps = 2.0 ** -24
    bound = (wl.d / 8 + 16) * eps * absdot + 2 * eps * np.abs(ref_lg) + 1e-30
    err = np.abs(lg.astype(np.float64) - ref_lg.astype(np.float64))
    assert np.all(err <= bound), f"logits off by up to {float(np.max(err / bound)):.3g} x the bound"
    ref_idx, ref_g = oracle.route_from_logits(lg, wl.k, inp.noise, wl.sigma)
    assert np.array_equal(idx, ref_idx), "top-k differs from the oracle on identical logits"
    np.testing.assert_allclose(gates, ref_g, rtol=0, atol=2e-6)


@pytest.mark.parametrize("name", sorted(SHAPES))
def test_router_against_oracle(name):
    require_gpu()
    wl = SHAPES[name]
    inp = make_inputs(wl, seed=21, weights=False)
    x, W_g, b_g, noise = to_dev(inp.x), to_dev(inp.W_g), to_dev(inp.b_g), to_dev(inp.noise)
    topk, gates, logits = moe.moe_route(x, W_g, wl.k, b_g=b_g, noise=noise, sigma=wl.sigma)
    torch.cuda.synchronize()
    _check(wl, inp, topk.cpu().numpy(), gates.cpu().numpy(), logits.cpu().numpy())
    # without the logits output: the same routing, bit for bit
    topk2, gates2, _ = moe.moe_route(x, W_g, wl.k, b_g=b_g, noise=noise, sigma=wl.sigma, want_logits=False)
    torch.cuda.synchronize()
    assert torch.equal(topk, topk2)
    assert torch.equal(gates.view(torch.int32), gates2.view(torch.int32))


def test_router_ties_go_to_lower_index():
    """Experts 2 and 6 (and 3 and 4) share router weights, so their logits are
    equal bit for bit; the lower index must be kept first."""
    require_gpu()
    wl = _wl("ties", N=1536, d=256, E=8, k=3, sigma=0.0, wg_std=0.1)
    inp = make_inputs(wl, seed=22, weights=False)
    inp.W_g[6] = inp.W_g[2]
    inp.W_g[4] = inp.W_g[3]
    x, W_g = to_dev(inp.x), to_dev(inp.W_g)
    topk, gates, logits = moe.moe_route(x, W_g, wl.k)
    torch.cuda.synchronize()
    lg = logits.cpu().numpy()
    assert np.array_equal(lg[:, 2].view(np.int32), lg[:, 6].view(np.int32))
    assert np.array_equal(lg[:, 3].view(np.int32), lg[:, 4].view(np.int32))
    idx = topk.cpu().numpy()
    _check(wl, inp, idx, gates.cpu().numpy(), lg)
    both = (idx == 2).any(1) & (idx == 6).any(1)
    pos2 = np.argmax(idx == 2, axis=1)
    pos6 = np.argmax(idx == 6, axis=1)
    assert np.all(pos2[both] < pos6[both])
    assert ((idx == 6).any(1) <= (idx == 2).any(1)).all(), "expert 6 kept without its tied twin 2"


FWD_CASES = {
    "clustered": Workload("fwd", BF16, N=2048, d=512, E=8, d_ff=256, k=2, sigma=1.0, cf=1.25, w_std=0.05),
    "persistent": Workload("fwdp", BF16, N=20000, d=2048, E=64, d_ff=128, k=6, sigma=1.0, cf=1.0, w_std=0.05),
}


@pytest.mark.parametrize("name", sorted(FWD_CASES))
def test_router_fused_forward_matches_staged(name):
    """moe_forward (router weights split once by a first pass, read by TMA)
    and moe_route (split inside the router kernel) give the same bits."""
    require_gpu()
    wl = FWD_CASES[name]
    inp = make_inputs(wl, seed=23)
    x, W_g, noise = to_dev(inp.x), to_dev(inp.W_g), to_dev(inp.noise)
    topk, gates, logits = moe.moe_route(x, W_g, wl.k, noise=noise, sigma=wl.sigma)
    _, inter = moe.moe_forward(x, W_g, to_dev(inp.W_up), to_dev(inp.W_down), wl.k, wl.cf, noise=noise,
                               sigma=wl.sigma, intermediates=True)
    torch.cuda.synchronize()
    assert torch.equal(inter["topk_idx"], topk)
    assert torch.equal(inter["gates"].view(torch.int32), gates.view(torch.int32))
    assert torch.equal(inter["logits"].view(torch.int32), logits.view(torch.int32))


BATCH_CASES = {
    "bf16_tensor_cores": _wl("bi_tc", N=3000, d=4096, E=8, k=2, sigma=1.0, bias0=1.0),
    "bf16_e64": _wl("bi_e64", N=2100, d=2048, E=64, k=6, sigma=1.0),
    "f32_cuda_cores": Workload("bi_f32", "f32", N=2100, d=1000, E=12, d_ff=16, k=3, sigma=0.5, cf=1.0,
                               wg_std=0.1),
    "bf16_cuda_cores": _wl("bi_odd", N=2100, d=36, E=5, k=2, sigma=0.0, wg_std=0.3),
    # the whole batch takes the persistent form, the slices the clustered one
    "bf16_persistent_e8": _wl("bi_p8", N=20000, d=4096, E=8, k=2, sigma=1.0, bias0=1.0),
    "bf16_persistent_e64": _wl("bi_p64", N=20000, d=2048, E=64, k=6, sigma=1.0),
}


@pytest.mark.parametrize("name", sorted(BATCH_CASES))
def test_router_batch_size_independent(name):
    """A token's logits, picks and gates do not depend on how many tokens
    share its call or where it sits: slices routed alone (one token, a
    64-token decode batch, the small-batch and large-batch kernels) equal the
    rows of the whole batch bit for bit."""
    require_gpu()
    wl = BATCH_CASES[name]
    inp = make_inputs(wl, seed=24, weights=False)
    x, W_g, b_g, noise = to_dev(inp.x), to_dev(inp.W_g), to_dev(inp.b_g), to_dev(inp.noise)
    topk, gates, logits = moe.moe_route(x, W_g, wl.k, b_g=b_g, noise=noise, sigma=wl.sigma)
    # even starts keep every slice 16-byte aligned (the ABI requires it)
    for a, b in ((6, 7), (100, 164), (0, 1000), (8, 1033), (2, min(2100, wl.N)), (2, wl.N - 1)):
        sl = slice(a, b)
        nz = None if noise is None else noise[sl].contiguous()
        t2, g2, l2 = moe.moe_route(x[sl].contiguous(), W_g, wl.k, b_g=b_g, noise=nz, sigma=wl.sigma)
        torch.cuda.synchronize()
        assert torch.equal(l2.view(torch.int32), logits[sl].view(torch.int32)), (a, b)
        assert torch.equal(t2, topk[sl]), (a, b)
        assert torch.equal(g2.view(torch.int32), gates[sl].view(torch.int32)), (a, b)


PRESPLIT_CASES = {
    "e8_d4096": _wl("pe8", N=20000, d=4096, E=8, k=2, sigma=1.0, bias0=1.0),
    "e24_odd_tiles": _wl("pe24", N=30001, d=512, E=24, k=3, sigma=0.5, wg_std=0.1),
    "e64_fine": _wl("pe64", N=32768, d=2048, E=64, k=6, sigma=1.0),
    # many picks per token: two groups' pick lists of 16 merged per token
    "e64_k16": _wl("pe64k", N=20000, d=512, E=64, k=16, sigma=0.5, wg_std=0.05),
    "e80": _wl("pe80", N=40000, d=1024, E=80, k=4, sigma=0.5, wg_std=0.05, bias0=0.5),
}


@pytest.mark.parametrize("name", sorted(PRESPLIT_CASES))
def test_router_pre_split_matches_in_kernel_split(name):
    """With a router workspace the weights are split once by a first pass and
    read by TMA (moe_forward's router); without one, the router splits them
    in-kernel.  Same bits, and the oracle's bar, on the persistent form with
    balanced tiles (an odd tile count among them)."""
    require_gpu()
    wl = PRESPLIT_CASES[name]
    inp = make_inputs(wl, seed=25, weights=False)
    x, W_g, b_g, noise = to_dev(inp.x), to_dev(inp.W_g), to_dev(inp.b_g), to_dev(inp.noise)
    ws = moe.route_workspace(wl.d, wl.E, x.device)
    t1, g1, l1 = moe.moe_route(x, W_g, wl.k, b_g=b_g, noise=noise, sigma=wl.sigma, status=ws)
    t2, g2, l2 = moe.moe_route(x, W_g, wl.k, b_g=b_g, noise=noise, sigma=wl.sigma)
    torch.cuda.synchronize()
    assert moe.check_status(ws) == (0, 0)
    assert torch.equal(l1.view(torch.int32), l2.view(torch.int32))
    assert torch.equal(t1, t2)
    assert torch.equal(g1.view(torch.int32), g2.view(torch.int32))
    _check(wl, inp, t1.cpu().numpy(), g1.cpu().numpy(), l1.cpu().numpy())


def test_router_larger_k_after_smaller_in_one_process():
    """The persistent router's shared memory grows with k (pick scratch and
    pick lists); a call with a larger k after a smaller one must still launch
    and route correctly (launch attributes are set once per device)."""
    require_gpu()
    for k in (2, 16, 4, 24):
        wl = _wl(f"kgrow{k}", N=20000, d=256, E=64, k=k, sigma=0.5, wg_std=0.1)
        inp = make_inputs(wl, seed=31 + k, weights=False)
        x, W_g, b_g, noise = to_dev(inp.x), to_dev(inp.W_g), to_dev(inp.b_g), to_dev(inp.noise)
        ws = moe.route_workspace(wl.d, wl.E, x.device)
        t, g, lg = moe.moe_route(x, W_g, wl.k, b_g=b_g, noise=noise, sigma=wl.sigma, status=ws)
        torch.cuda.synchronize()
        assert moe.check_status(ws) == (0, 0)
        _check(wl, inp, t.cpu().numpy(), g.cpu().numpy(), lg.cpu().numpy())
