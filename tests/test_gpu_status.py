"""Kernel status reporting (needs a B200).

A kernel whose bounded wait runs out ORs MOE_ERR_TIMEOUT's bit into the status
word; nothing but moe_check_status clears it.  So the report of a failed
launch must survive any number of later, clean calls on the same workspace,
and those later calls must still compute their results (the give-up signal
between a kernel's roles stays inside that kernel's CTA)."""
import pytest
import torch

from sparse_mixture_experts_noisy_b200 import moe
from sparse_mixture_experts_noisy_b200.synth import WORKLOADS
from tests.gpu_util import Case, require_gpu

pytestmark = pytest.mark.gpu

TIMEOUT = 6


def _small(name):
    base = {"mixtral": dict(N=700, d=256, d_ff=512), "decode": dict(N=64, d=512, d_ff=1024),
            "fine": dict(N=3000, d=256, d_ff=128, E=64, k=6)}[name]
    return WORKLOADS[name].with_(**base)


@pytest.mark.parametrize("name", ["mixtral", "decode", "fine"])
def test_timeout_report_survives_a_clean_forward(name):
    require_gpu()
    wl = _small(name)
    case = Case(wl, seed=3)
    layer = moe.MoELayer(case.W_g, case.W_up, case.W_down, wl.k, wl.cf, b_g=case.b_g, sigma=wl.sigma)
    y_ref = layer(case.x, noise=case.noise).clone()
    assert moe.check_status(layer.workspace) == (0, 0)
    moe.debug_wait_timeout(20000, layer.workspace)     # a wait that runs out after 20 ms
    y = layer(case.x, noise=case.noise)                # then a clean forward on the same workspace
    y2 = layer(case.x, noise=case.noise)
    torch.cuda.synchronize()
    # the clean forwards did their work in full despite the earlier failure
    assert torch.equal(y.view(torch.int16), y_ref.view(torch.int16))
    assert torch.equal(y2.view(torch.int16), y_ref.view(torch.int16))
    code, word = moe.check_status(layer.workspace)
    assert code == TIMEOUT and (word & 1), (code, hex(word))
    assert (word & 2) == 0                             # the CTA-local give-up bit never reaches the word
    assert moe.check_status(layer.workspace) == (0, 0)  # read once, then cleared


def test_expert_ffn_keeps_an_earlier_report():
    require_gpu()
    wl = _small("mixtral")
    case = Case(wl, seed=5)
    topk, gates, _ = moe.moe_route(case.x, case.W_g, wl.k, b_g=case.b_g)
    dsp = moe.moe_dispatch(topk, case.x, wl.E, wl.cf)
    ws = moe.new_workspace(moe.load_library().moe_expert_ffn_workspace_size(
        dsp["rows"], wl.d, wl.E, wl.d_ff, moe.MOE_BF16), case.x.device)
    moe.debug_wait_timeout(20000, ws)
    moe.moe_expert_ffn(dsp["x_gathered"], dsp["offsets"], dsp["counts"], case.W_up, case.W_down, ws=ws)
    code, _ = moe.check_status(ws)
    assert code == TIMEOUT
    moe.moe_expert_ffn(dsp["x_gathered"], dsp["offsets"], dsp["counts"], case.W_up, case.W_down, ws=ws)
    assert moe.check_status(ws) == (0, 0)


@pytest.mark.parametrize("name", ["mixtral", "fine"])
def test_router_reports_into_the_callers_word(name):
    require_gpu()
    wl = _small(name)
    case = Case(wl, seed=7)
    ws = moe.new_workspace(256, case.x.device)
    a = moe.moe_route(case.x, case.W_g, wl.k, b_g=case.b_g, noise=case.noise, sigma=wl.sigma, status=ws)
    assert moe.check_status(ws) == (0, 0)
    moe.debug_wait_timeout(20000, ws)
    b = moe.moe_route(case.x, case.W_g, wl.k, b_g=case.b_g, noise=case.noise, sigma=wl.sigma, status=ws)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])
    code, word = moe.check_status(ws)                  # the router did not clear the earlier report
    assert code == TIMEOUT and (word & 1)


def test_router_without_a_word_reports_into_the_librarys():
    require_gpu()
    wl = _small("fine")
    case = Case(wl, seed=9)
    moe.check_route_status()                           # start from a clear word
    moe.moe_route(case.x, case.W_g, wl.k, b_g=case.b_g, noise=case.noise, sigma=wl.sigma)
    assert moe.check_route_status() == (0, 0)
