"""moe_combine on its own (needs a B200): y[t] = sum over kept choices j of
gate[t, j] * out[offsets[e] + slot[t, j]], in fp32, no renormalisation
("Mixture of Experts (MoE) 12段階極小ビジュアル解剖シミュレーター" STEP 11-12;
"nanoMoEの深層解剖" slides 38-40: a dropped pair has weight 0).

Every large-batch kernel variant (1 to 8 choices per token) and the
small-batch kernel run on the same rows; they must agree bit for bit, and
with the sum written out in float64 to within one bf16 rounding of y."""
import numpy as np
import pytest
import torch

from sparse_mixture_experts_noisy_b200 import moe
from sparse_mixture_experts_noisy_b200.synth import bf16_bits_to_f32, f32_to_bf16_bits
from tests.gpu_util import require_gpu

pytestmark = pytest.mark.gpu


def _case(k, N=2100, d=520, E=12, cf=0.9, seed=0):
    rng = np.random.default_rng(100 + k)
    scores = rng.standard_normal((N, E))
    topk = np.argsort(-scores, axis=1, kind="stable")[:, :k].astype(np.int32)
    g = rng.random((N, k)).astype(np.float32)
    x = torch.zeros((N, d), dtype=torch.bfloat16, device="cuda")
    tk = torch.from_numpy(topk).cuda()
    disp = moe.moe_dispatch(tk, x, E, cf)  # slots, offsets, with drops at cf < 1
    rows = disp["rows"]
    out = f32_to_bf16_bits(rng.standard_normal((rows, d)).astype(np.float32))
    out_t = torch.from_numpy(out.view(np.int16)).cuda().view(torch.bfloat16)
    return tk, torch.from_numpy(g).cuda(), disp, out_t, out


@pytest.mark.parametrize("k,d", [(1, 520), (2, 520), (3, 520), (4, 520), (5, 520), (6, 520), (7, 520), (8, 520),
                                 (10, 520), (2, 36)])
def test_combine_variants(k, d):
    """k <= 8 with 16-byte rows: the warp kernel; k = 10 or d = 36 (rows not
    16-byte multiples): the per-chunk kernel."""
    require_gpu()
    tk, g, disp, out_t, out = _case(k, d=d)
    y = moe.moe_combine(out_t, disp["slot"], tk, disp["offsets"], g)
    torch.cuda.synchronize()
    yb = y.view(torch.int16).cpu().numpy().view(np.uint16)
    # reference sum in float64 on the exact inputs
    slot = disp["slot"].cpu().numpy()
    offs = disp["offsets"].cpu().numpy()
    tkn = tk.cpu().numpy()
    gn = g.cpu().numpy().astype(np.float64)
    o64 = bf16_bits_to_f32(out).astype(np.float64)
    N, d = yb.shape
    ref = np.zeros((N, d))
    for j in range(k):
        kept = slot[:, j] >= 0
        r = offs[tkn[kept, j]] + slot[kept, j]
        ref[kept] += gn[kept, j, None] * o64[r]
    got = bf16_bits_to_f32(yb).astype(np.float64)
    # one bf16 rounding of y plus fp32 accumulation
    tol = 2.0 ** -8 * np.abs(ref) + 1e-6 * np.abs(gn).sum(1, keepdims=True) * np.abs(o64).max()
    assert np.all(np.abs(got - ref) <= tol)
    assert np.array_equal(got[(slot < 0).all(1)], np.zeros(((slot < 0).all(1).sum(), d)))
    # the small-batch kernel on the first 100 tokens gives the same bits
    y_small = moe.moe_combine(out_t, disp["slot"][:100].contiguous(), tk[:100].contiguous(), disp["offsets"],
                              g[:100].contiguous())
    torch.cuda.synchronize()
    assert torch.equal(y_small.view(torch.int16), y[:100].view(torch.int16))
