"""The nanoMoE expert variant ("nanoMoEの深層解剖" slide 32: biases after each
projection, GELU in place of ReLU) on the GPU against the oracle (needs a B200).

Every FFN path is covered: CTA-pair prefill tiles, one-CTA tiles, the decode
plan (K splits summed in the ReLU/GELU pass and in the combine), and the
CUDA-core fp32 and unaligned-bf16 kernels."""
import numpy as np
import pytest
import torch

import oracle
from sparse_mixture_experts_noisy_b200 import moe
from sparse_mixture_experts_noisy_b200.synth import WORKLOADS, Workload, F32, BF16
from tests.gpu_util import Case, TOL, rel_err, require_gpu, to_host_bits, values

pytestmark = pytest.mark.gpu

W = WORKLOADS
SHAPES = {
    "prefill": W["mixtral"].with_(N=1536, d=512, d_ff=1024),
    "decode": W["decode"].with_(N=64, d=512, d_ff=1024),
    "f32": Workload("f32v", F32, N=300, d=40, E=6, d_ff=50, k=3, sigma=0.5, cf=0.8, w_std=0.3, wg_std=0.3),
    "bf16_unaligned": Workload("bf16v", BF16, N=200, d=36, E=5, d_ff=20, k=2, sigma=0.0, cf=1.0,
                               w_std=0.2, wg_std=0.3),
}


def _biases(wl, seed):
    rng = np.random.default_rng(1000 + seed)
    b_up = (0.5 * rng.standard_normal((wl.E, wl.d_ff))).astype(np.float32)
    b_down = (0.5 * rng.standard_normal((wl.E, wl.d))).astype(np.float32)
    return b_up, b_down


@pytest.mark.parametrize("act", [moe.ACT_GELU, moe.ACT_RELU])
@pytest.mark.parametrize("with_bias", [True, False])
@pytest.mark.parametrize("shape", sorted(SHAPES))
def test_variant_forward(shape, with_bias, act, monkeypatch):
    require_gpu()
    if act == moe.ACT_RELU and not with_bias:
        pytest.skip("the plain layer is covered by the main parity tests")
    wl = SHAPES[shape]
    case = Case(wl, seed=7)
    b_up, b_down = _biases(wl, 7) if with_bias else (None, None)
    bu = None if b_up is None else torch.from_numpy(b_up).cuda()
    bd = None if b_down is None else torch.from_numpy(b_down).cuda()
    y, inter = moe.moe_forward(case.x, case.W_g, case.W_up, case.W_down, wl.k, wl.cf, b_g=case.b_g,
                               noise=case.noise, sigma=wl.sigma, intermediates=True, act=act, b_up=bu,
                               b_down=bd)
    torch.cuda.synchronize()
    lg = inter["logits"].cpu().numpy()
    i = case.inp
    ref = oracle.forward(i.x, i.W_g, i.b_g, i.noise, wl.sigma, wl.k, wl.cf, i.W_up, i.W_down, logits=lg,
                         nthreads=8, act=act, b_up=b_up, b_down=b_down)
    assert np.array_equal(inter["slot"].cpu().numpy(), ref["slot"])
    err = rel_err(values(to_host_bits(y)), ref["y"])
    assert err <= TOL[wl.dtype], f"{shape}: {err:.3g}"


@pytest.mark.parametrize("shape", ["prefill", "decode"])
def test_variant_expert_ffn_rows(shape):
    """moe_expert_ffn_ex row by row against the oracle's expert variant."""
    require_gpu()
    wl = SHAPES[shape]
    case = Case(wl, seed=8)
    b_up, b_down = _biases(wl, 8)
    topk, gates, _ = moe.moe_route(case.x, case.W_g, wl.k, b_g=case.b_g, noise=case.noise, sigma=wl.sigma)
    d = moe.moe_dispatch(topk, case.x, wl.E, wl.cf)
    out = moe.moe_expert_ffn(d["x_gathered"], d["offsets"], d["counts"], case.W_up, case.W_down,
                             act=moe.ACT_GELU, b_up=torch.from_numpy(b_up).cuda(),
                             b_down=torch.from_numpy(b_down).cuda())
    torch.cuda.synchronize()
    slot = d["slot"].cpu().numpy()
    offs = d["offsets"].cpu().numpy()
    tk = topk.cpu().numpy()
    og = values(to_host_bits(out))
    i = case.inp
    checked = 0
    for t in range(0, wl.N, max(1, wl.N // 40)):
        for j in range(wl.k):
            if slot[t, j] < 0:
                continue
            r = offs[tk[t, j]] + slot[t, j]
            _, o = oracle.expert_ffn_ex(i.x, i.W_up, i.W_down, t, tk[t, j], act=oracle.ACT_GELU, b_up=b_up,
                                        b_down=b_down)
            assert rel_err(og[r], o) <= TOL[wl.dtype]
            checked += 1
    assert checked >= 20


def test_variant_one_cta_tiles(monkeypatch):
    """The one-CTA prefill tiles (selected when CTA pairs are switched off in a
    fresh process) carry the same epilogue; run them through a child process."""
    require_gpu()
    import subprocess
    import sys
    import os
    code = (
        "import numpy as np, torch, oracle;"
        "from sparse_mixture_experts_noisy_b200 import moe;"
        "from tests.test_gpu_variant import SHAPES, _biases;"
        "from tests.gpu_util import Case, TOL, rel_err, to_host_bits, values;"
        "wl=SHAPES['prefill']; c=Case(wl,seed=5); bu,bd=_biases(wl,5);"
        "y,it=moe.moe_forward(c.x,c.W_g,c.W_up,c.W_down,wl.k,wl.cf,b_g=c.b_g,intermediates=True,"
        "act=moe.ACT_GELU,b_up=torch.from_numpy(bu).cuda(),b_down=torch.from_numpy(bd).cuda());"
        "torch.cuda.synchronize(); i=c.inp;"
        "ref=oracle.forward(i.x,i.W_g,i.b_g,None,0.0,wl.k,wl.cf,i.W_up,i.W_down,logits=it['logits'].cpu().numpy(),"
        "nthreads=8,act=2,b_up=bu,b_down=bd);"
        "e=rel_err(values(to_host_bits(y)),ref['y']); print('err',e); assert e<=TOL['bf16']"
    )
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, MOE_TC_PAIR="0", PYTHONPATH=root)
    r = subprocess.run([sys.executable, "-c", code], cwd=root, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
