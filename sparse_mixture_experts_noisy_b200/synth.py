"""Seeded synthetic inputs for the sparse noisy top-k MoE layer.

This module only draws random numbers and rounds them to the storage type.
It holds none of the layer's arithmetic, so the CUDA path and the CPU
oracle can both take their inputs from here without sharing any of the
method.

Workloads (shapes and value distributions follow the problem statement of
the MoE pages: the single-token walkthrough "Mixture of Experts (MoE)
12段階極小ビジュアル解剖シミュレーター", its input vector x = [1.20, -0.40,
-0.80] with k = 2 and sigma = 0, and the nanoMoE slides "nanoMoEの深層解剖",
slides 11-14 for the router and capacity settings):

  toy     fp32  N=8     d=3    E=4  d_ff=4     k=2  sigma=0  cf=inf
  nano    bf16  N=8192  d=768  E=8  d_ff=3072  k=2  sigma=0  cf=1.25
  mixtral bf16  N=16384 d=4096 E=8  d_ff=14336 k=2  sigma=0  cf=1.25, b_g[0]=+1
  fine    bf16  N=32768 d=2048 E=64 d_ff=1408  k=6  sigma=1  cf=1.0
  decode  bf16  N=64    d=4096 E=8  d_ff=14336 k=2  sigma=0  cf=inf

Recipe: numpy ``default_rng(seed + offset).standard_normal`` in float64,
scaled by the workload's standard deviation, rounded to float32, then to
bfloat16 (round to nearest even) where the workload stores bf16.  Offsets:
x +0, W_g +1, W_up +2, W_down +3, noise eps +4.  The router weight W_g, its
bias and the noise are always float32.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import numpy as np

F32 = "f32"
BF16 = "bf16"

_CHUNK = 1 << 22  # values drawn per call; the stream is the same for any chunking


@dataclass(frozen=True)
class Workload:
    name: str
    dtype: str
    N: int
    d: int
    E: int
    d_ff: int
    k: int
    sigma: float
    cf: float
    x_std: float = 1.0
    w_std: float = 0.02
    wg_std: float = 0.02
    bias0: float = 0.0          # router bias on expert 0 (others 0); 0 means no bias tensor
    fix_token0: tuple = ()      # explicit values for x[0]
    note: str = ""

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    "toy": Workload("toy", F32, N=8, d=3, E=4, d_ff=4, k=2, sigma=0.0, cf=math.inf,
                    x_std=1.0, w_std=1.0, wg_std=1.0, fix_token0=(1.20, -0.40, -0.80),
                    note="single-token walkthrough sizes, batched B=2,T=4"),
    "nano": Workload("nano", BF16, N=8192, d=768, E=8, d_ff=3072, k=2, sigma=0.0, cf=1.25,
                     x_std=1.0, w_std=0.02, wg_std=1.0 / math.sqrt(768.0),
                     note="nanoMoE scale B=8,T=1024"),
    "mixtral": Workload("mixtral", BF16, N=16384, d=4096, E=8, d_ff=14336, k=2, sigma=0.0,
                        cf=1.25, x_std=1.0, w_std=0.02, wg_std=0.02, bias0=1.0,
                        note="Mixtral-shaped layer, router bias +1 on expert 0"),
    "fine": Workload("fine", BF16, N=32768, d=2048, E=64, d_ff=1408, k=6, sigma=1.0, cf=1.0,
                     x_std=1.0, w_std=0.02, wg_std=0.02,
                     note="fine-grained noisy routing, supplied eps ~ N(0,1)"),
    "decode": Workload("decode", BF16, N=64, d=4096, E=8, d_ff=14336, k=2, sigma=0.0,
                       cf=math.inf, x_std=1.0, w_std=0.02, wg_std=0.02,
                       note="64-token decode, weight streaming"),
}


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (nearest, ties to even); returns the uint16 bit patterns."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = u + 0x7FFF + ((u >> 16) & 1)
    return (u >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bit patterns to float32."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def normal_f32(seed: int, shape, std: float) -> np.ndarray:
    """std * N(0,1) drawn in float64 from default_rng(seed), rounded to float32."""
    rng = np.random.default_rng(seed)
    n = int(np.prod(shape)) if len(shape) else 1
    out = np.empty(n, dtype=np.float32)
    for s in range(0, n, _CHUNK):
        m = min(_CHUNK, n - s)
        v = rng.standard_normal(m)
        if std != 1.0:
            v *= std
        out[s:s + m] = v
    return out.reshape(shape)


def _store(a32: np.ndarray, dtype: str) -> np.ndarray:
    return f32_to_bf16_bits(a32) if dtype == BF16 else a32


@dataclass
class Inputs:
    """Host copies of one layer call's inputs.

    Arrays of the workload's storage type hold float32 values (fp32) or
    uint16 bfloat16 bit patterns (bf16)."""
    wl: Workload
    seed: int
    x: np.ndarray            # [N, d]
    W_g: np.ndarray          # [E, d] float32
    b_g: np.ndarray | None   # [E] float32
    noise: np.ndarray | None # [N, E] float32
    W_up: np.ndarray         # [E, d_ff, d]
    W_down: np.ndarray       # [E, d, d_ff]
    extra: dict = field(default_factory=dict)


def make_x(wl: Workload, seed: int = 0) -> np.ndarray:
    x = normal_f32(seed, (wl.N, wl.d), wl.x_std)
    if wl.fix_token0 and wl.N > 0:
        x[0, :len(wl.fix_token0)] = np.asarray(wl.fix_token0, dtype=np.float32)
    return _store(x, wl.dtype)


def make_noise(wl: Workload, seed: int = 0) -> np.ndarray | None:
    if wl.sigma == 0.0:
        return None
    return normal_f32(seed + 4, (wl.N, wl.E), 1.0)


def make_inputs(wl: Workload | str, seed: int = 0, weights: bool = True) -> Inputs:
    if isinstance(wl, str):
        wl = WORKLOADS[wl]
    x = make_x(wl, seed)
    W_g = normal_f32(seed + 1, (wl.E, wl.d), wl.wg_std)
    b_g = None
    if wl.bias0 != 0.0:
        b_g = np.zeros(wl.E, dtype=np.float32)
        b_g[0] = wl.bias0
    noise = make_noise(wl, seed)
    if weights:
        W_up = _store(normal_f32(seed + 2, (wl.E, wl.d_ff, wl.d), wl.w_std), wl.dtype)
        W_down = _store(normal_f32(seed + 3, (wl.E, wl.d, wl.d_ff), wl.w_std), wl.dtype)
    else:
        W_up = W_down = None
    return Inputs(wl, seed, x, W_g, b_g, noise, W_up, W_down)


def as_f64(a: np.ndarray, dtype: str) -> np.ndarray:
    """Exact float64 values of an array stored as fp32 or bf16 bits."""
    if dtype == BF16:
        return bf16_bits_to_f32(a).astype(np.float64)
    return np.asarray(a, dtype=np.float32).astype(np.float64)
