"""The five workloads at full size, in the launch configuration the benchmark
times (one moe_forward call), against the oracle (needs a B200).

Routing is checked bit-exactly over every token (the oracle replays the GPU's
fp32 logits).  The output is checked on tokens the oracle computes one by one:
  - for every expert, the tokens of its first and last kept row and of the
    first and last row of every 128-row block of its rows, so every tile of
    the expert GEMMs (128-row tiles, 256-row pair tiles, and the tiles whose
    last rows belong to the next expert) contributes checked rows;
  - a seeded random sample, the first and last token, and tokens with dropped
    choices.
Each checked row must meet the max-normalised bar and, for bf16, the
per-element rounding model (tests/gpu_util.py)."""
import numpy as np
import pytest
import torch

from sparse_mixture_experts_noisy_b200.synth import WORKLOADS
from tests.gpu_util import (Case, TOL, bf16_error_sigma, check_elementwise_bf16, check_routing, rel_err,
                            require_gpu, to_host_bits, values)

pytestmark = pytest.mark.gpu

SAMPLE = {"toy": None, "nano": 384, "mixtral": 48, "fine": 256, "decode": None}
BLOCK = 128


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def tile_tokens(idx, slot, counts):
    """Tokens owning the first and last row of every expert and of every
    BLOCK-row block of each expert's kept rows."""
    E = len(counts)
    owner = [dict() for _ in range(E)]
    ts, js = np.nonzero(slot >= 0)
    for t, j in zip(ts.tolist(), js.tolist()):
        owner[idx[t, j]][int(slot[t, j])] = t
    picked = set()
    for e in range(E):
        c = int(counts[e])
        if c == 0:
            continue
        rows = {0, c - 1}
        for b in range(0, c, BLOCK):
            rows.add(b)
            rows.add(min(c, b + BLOCK) - 1)
        picked |= {owner[e][r] for r in rows}
    return picked


@pytest.mark.parametrize("name", ["toy", "nano", "mixtral", "fine", "decode"])
def test_full_size(name):
    wl = WORKLOADS[name]
    case = Case(wl, seed=0)
    y, inter = case.forward()
    torch.cuda.synchronize()
    lg, idx, g, slot, counts = check_routing(case, inter)
    n = SAMPLE[name]
    if n is None or n >= wl.N:
        tokens = np.arange(wl.N)
    else:
        rng = np.random.default_rng(123)
        tokens = set(rng.choice(wl.N, size=n, replace=False).tolist()) | {0, wl.N - 1}
        dropped_any = np.where(np.any(slot < 0, axis=1))[0]
        if len(dropped_any):
            tokens |= set(dropped_any[:8].tolist())
        tokens |= tile_tokens(idx, slot, counts)
        tokens = np.array(sorted(tokens))
    ref = case.oracle_from_logits(lg, tokens)
    yh = values(to_host_bits(y))[tokens]
    err = rel_err(yh, ref["y"])
    assert err <= TOL[wl.dtype], f"{name}: output error {err:.3g}"
    if wl.dtype == "bf16":
        sig = bf16_error_sigma(case.inp, wl, tokens, idx, g, slot, ref["y"])
        worst = check_elementwise_bf16(yh, ref["y"], sig, name)
        print(f"{name}: {len(tokens)} tokens checked, max rel err {err:.3g}, worst element {worst:.2f} sigma")
    if name == "mixtral":
        assert np.sum(slot < 0) > 0, "the +1 router bias on expert 0 should overflow its capacity"
        assert counts[0] == 5120
