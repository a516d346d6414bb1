"""Run the layer forward a few times on one workload (for profilers).

    python -m sparse_mixture_experts_noisy_b200.run_case --workload mixtral [--N 8192] [--iters 3]

Generates the workload's seeded inputs, calls moe_forward `iters` times on
cuda:0, synchronises, checks the kernels' status word and prints the routing
load.  Sizes can be overridden to make a smaller case of the same shape.
"""
from __future__ import annotations

import argparse
import sys

import numpy as np
import torch

from sparse_mixture_experts_noisy_b200 import moe
from sparse_mixture_experts_noisy_b200.synth import WORKLOADS, make_inputs


def to_dev(a):
    if a is None:
        return None
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="mixtral", choices=sorted(WORKLOADS))
    ap.add_argument("--N", type=int)
    ap.add_argument("--d", type=int)
    ap.add_argument("--d_ff", type=int)
    ap.add_argument("--iters", type=int, default=3)
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--staged", action="store_true", help="call moe_expert_ffn alone after one forward")
    a = ap.parse_args(argv)
    wl = WORKLOADS[a.workload]
    over = {k: v for k, v in (("N", a.N), ("d", a.d), ("d_ff", a.d_ff)) if v is not None}
    if over:
        wl = wl.with_(**over)
    inp = make_inputs(wl, a.seed)
    x, W_g, b_g, noise, W_up, W_down = (to_dev(v) for v in (inp.x, inp.W_g, inp.b_g, inp.noise,
                                                             inp.W_up, inp.W_down))
    layer = moe.MoELayer(W_g, W_up, W_down, wl.k, wl.cf, b_g=b_g, sigma=wl.sigma, max_tokens=wl.N)
    y = torch.empty_like(x)
    for _ in range(a.iters):
        layer(x, noise=noise, y=y)
    torch.cuda.synchronize()
    code, word = moe.check_status(layer.workspace)
    if code != 0:
        print(f"status {code} 0x{word:08x}", file=sys.stderr)
        return 1
    if a.staged:
        topk, gates, _ = moe.moe_route(x, W_g, wl.k, b_g=b_g, noise=noise, sigma=wl.sigma, want_logits=False)
        d = moe.moe_dispatch(topk, x, wl.E, wl.cf)
        for _ in range(a.iters):
            moe.moe_expert_ffn(d["x_gathered"], d["offsets"], d["counts"], W_up, W_down)
        torch.cuda.synchronize()
    _, inter = moe.moe_forward(x, W_g, W_up, W_down, wl.k, wl.cf, b_g=b_g, noise=noise, sigma=wl.sigma,
                               intermediates=True)
    torch.cuda.synchronize()
    counts = inter["counts"].cpu().numpy()
    print(f"{wl.name}: N={wl.N} d={wl.d} E={wl.E} d_ff={wl.d_ff} k={wl.k} kept={int(counts.sum())} "
          f"counts={counts.tolist()}")
    return 0


if __name__ == "__main__":
    sys.exit(main())
