"""ctypes wrapper around the plain C oracle (``moe_oracle.c``).

TEST INFRASTRUCTURE ONLY.  Each function mirrors one step of the layer as
the MoE pages define it ("Mixture of Experts (MoE) 12段階極小ビジュアル解剖
シミュレーター", STEP 2-12; "nanoMoEの深層解剖", slides 11-40).  The C file
holds the arithmetic; this file only marshals numpy arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

ORACLE_F32 = 0
ORACLE_BF16 = 1

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "_build", "libmoe_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, no FMA contraction)."""
    os.makedirs(os.path.dirname(_LIB), exist_ok=True)
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
                               "-fPIC", "-shared", "-o", tmp, _SRC, "-lm", "-lpthread"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            I64, I32, F32, F64 = ctypes.c_int64, ctypes.c_int, ctypes.c_float, ctypes.c_double
            lib.oracle_router_logits.argtypes = [P, I32, P, P, I64, I32, I32, P]
            lib.oracle_router_logits.restype = None
            lib.oracle_route_from_logits.argtypes = [P, P, F32, I64, I32, I32, P, P, P]
            lib.oracle_route_from_logits.restype = None
            lib.oracle_capacity.argtypes = [I64, I32, I32, F64]
            lib.oracle_capacity.restype = I64
            lib.oracle_assign_slots.argtypes = [P, I64, I32, I32, I64, P, P]
            lib.oracle_assign_slots.restype = None
            lib.oracle_load_stats.argtypes = [P, P, I64, I32, I32, I64, P, P, P]
            lib.oracle_load_stats.restype = None
            lib.oracle_backward.argtypes = [P, I32, P, P, P, P, P, P, P, I64, I32, I32, I32, I32, P, P, P, P, P, P]
            lib.oracle_backward.restype = None
            lib.oracle_backward_sampled.argtypes = [P, I32, P, P, P, P, P, P, P, I64, I32, I32, I32, I32, P,
                                                    P, I64, P, I64, I32, P, P, P, P, P]
            lib.oracle_backward_sampled.restype = None
            lib.oracle_expert_ffn.argtypes = [P, I32, P, P, I64, I32, I32, I32, P, P]
            lib.oracle_expert_ffn.restype = None
            lib.oracle_ffn_combine.argtypes = [P, I32, P, P, P, P, P, I32, I32, I32, P, I64, P, I32]
            lib.oracle_ffn_combine.restype = None
            lib.oracle_expert_ffn_ex.argtypes = [P, I32, P, P, P, P, I32, I64, I32, I32, I32, P, P]
            lib.oracle_expert_ffn_ex.restype = None
            lib.oracle_ffn_combine_ex.argtypes = [P, I32, P, P, P, P, I32, P, P, P, I32, I32, I32, P, I64, P, I32]
            lib.oracle_ffn_combine_ex.restype = None
            _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _dt(a: np.ndarray) -> int:
    if a.dtype == np.uint16:
        return ORACLE_BF16
    if a.dtype == np.float32:
        return ORACLE_F32
    raise TypeError(f"oracle inputs are float32 or bf16 bit patterns (uint16), got {a.dtype}")


def capacity(N: int, E: int, k: int, cf: float) -> int:
    return int(_load().oracle_capacity(N, E, k, float(cf)))


def router_logits(x, W_g, b_g=None):
    """s_raw [N,E] fp32 (STEP 2; slide 11, fp32 router)."""
    x = np.ascontiguousarray(x)
    W_g = np.ascontiguousarray(W_g, dtype=np.float32)
    N, d = x.shape
    E = W_g.shape[0]
    out = np.empty((N, E), dtype=np.float32)
    bg = None if b_g is None else np.ascontiguousarray(b_g, dtype=np.float32)
    _load().oracle_router_logits(_ptr(x), _dt(x), _ptr(W_g), _ptr(bg), N, d, E, _ptr(out))
    return out


def route_from_logits(s_raw, k, noise=None, sigma=0.0, return_scores=False):
    """(topk_idx [N,k] int32, gates [N,k] fp32[, s [N,E]]) (STEP 3-6; slides 12-13)."""
    s_raw = np.ascontiguousarray(s_raw, dtype=np.float32)
    N, E = s_raw.shape
    nz = None if noise is None else np.ascontiguousarray(noise, dtype=np.float32)
    idx = np.empty((N, k), dtype=np.int32)
    g = np.empty((N, k), dtype=np.float32)
    s = np.empty((N, E), dtype=np.float32) if return_scores else None
    _load().oracle_route_from_logits(_ptr(s_raw), _ptr(nz), float(sigma), N, E, k,
                                     _ptr(idx), _ptr(g), _ptr(s))
    return (idx, g, s) if return_scores else (idx, g)


def assign_slots(topk_idx, E, C):
    """(slot [N,k] int32 with -1 = dropped, counts [E] int32) (slides 14-23)."""
    topk_idx = np.ascontiguousarray(topk_idx, dtype=np.int32)
    N, k = topk_idx.shape
    slot = np.empty((N, k), dtype=np.int32)
    counts = np.empty(E, dtype=np.int32)
    _load().oracle_assign_slots(_ptr(topk_idx), N, E, k, int(C), _ptr(slot), _ptr(counts))
    return slot, counts


def _mask(relu_mask, N, k, d_ff):
    if relu_mask is None:
        return None
    m = np.ascontiguousarray(relu_mask, dtype=np.uint8)
    assert m.shape == (N, k, d_ff)
    return m


def backward(x, W_g, W_up, W_down, s, topk_idx, slot, dy, relu_mask=None):
    """Gradients of L = sum(dy * y) for a given routing (STEP 6 and STEP 11):
    dict(dx [N,d], dW_g [E,d], db_g [E], dW_up [E,d_ff,d], dW_down [E,d,d_ff]), float64.
    s [N,E] float32: the noisy scores the gates came from (route_from_logits' s_noisy).
    relu_mask [N,k,d_ff] (optional): ReLU decisions of the kept pairs to replay."""
    x = np.ascontiguousarray(x)
    W_g = np.ascontiguousarray(W_g, dtype=np.float32)
    W_up = np.ascontiguousarray(W_up)
    W_down = np.ascontiguousarray(W_down)
    s = np.ascontiguousarray(s, dtype=np.float32)
    topk_idx = np.ascontiguousarray(topk_idx, dtype=np.int32)
    slot = np.ascontiguousarray(slot, dtype=np.int32)
    dy = np.ascontiguousarray(dy, dtype=np.float64)
    N, d = x.shape
    E, d_ff, _ = W_up.shape
    k = topk_idx.shape[1]
    out = dict(dx=np.empty((N, d)), dW_g=np.empty((E, d)), db_g=np.empty(E), dW_up=np.empty((E, d_ff, d)),
               dW_down=np.empty((E, d, d_ff)))
    mk = _mask(relu_mask, N, k, d_ff)
    _load().oracle_backward(_ptr(x), _dt(x), _ptr(W_g), _ptr(W_up), _ptr(W_down), _ptr(s), _ptr(topk_idx),
                            _ptr(slot), _ptr(dy), N, d, E, d_ff, k, _ptr(mk), _ptr(out["dx"]), _ptr(out["dW_g"]),
                            _ptr(out["db_g"]), _ptr(out["dW_up"]), _ptr(out["dW_down"]))
    return out


def backward_sampled(x, W_g, W_up, W_down, s, topk_idx, slot, dy, tokens, ef, relu_mask=None, nthreads=1):
    """oracle_backward at listed places: dict(dx_rows [len(tokens), d],
    dW_up_rows [len(ef), d] (dW_up[e, f, :]), dW_down_cols [len(ef), d]
    (dW_down[e, :, f]), dW_g [E, d], db_g [E]), float64; ef: [(e, f), ...]."""
    x = np.ascontiguousarray(x)
    W_g = np.ascontiguousarray(W_g, dtype=np.float32)
    W_up = np.ascontiguousarray(W_up)
    W_down = np.ascontiguousarray(W_down)
    s = np.ascontiguousarray(s, dtype=np.float32)
    topk_idx = np.ascontiguousarray(topk_idx, dtype=np.int32)
    slot = np.ascontiguousarray(slot, dtype=np.int32)
    dy = np.ascontiguousarray(dy, dtype=np.float64)
    tokens = np.ascontiguousarray(tokens, dtype=np.int64)
    ef = np.ascontiguousarray(np.asarray(ef, dtype=np.int32).reshape(-1, 2))
    N, d = x.shape
    E, d_ff, _ = W_up.shape
    k = topk_idx.shape[1]
    mk = _mask(relu_mask, N, k, d_ff)
    out = dict(dx_rows=np.empty((len(tokens), d)), dW_up_rows=np.empty((len(ef), d)),
               dW_down_cols=np.empty((len(ef), d)), dW_g=np.empty((E, d)), db_g=np.empty(E))
    _load().oracle_backward_sampled(_ptr(x), _dt(x), _ptr(W_g), _ptr(W_up), _ptr(W_down), _ptr(s),
                                    _ptr(topk_idx), _ptr(slot), _ptr(dy), N, d, E, d_ff, k, _ptr(mk),
                                    _ptr(tokens), len(tokens), _ptr(ef), len(ef), int(nthreads),
                                    _ptr(out["dx_rows"]), _ptr(out["dW_g"]), _ptr(out["db_g"]),
                                    _ptr(out["dW_up_rows"]), _ptr(out["dW_down_cols"]))
    return out


def load_stats(topk_idx, E, C, gates=None):
    """(load [E] int32, used [E] int32, importance [E] float64 or None): per-expert
    choices before the capacity cut, min(load, C) (slide 14's used_capacity),
    and the gate mass in units of 2^-32 summed exactly."""
    topk_idx = np.ascontiguousarray(topk_idx, dtype=np.int32)
    N, k = topk_idx.shape
    load = np.empty(E, dtype=np.int32)
    used = np.empty(E, dtype=np.int32)
    imp = np.empty(E, dtype=np.float64) if gates is not None else None
    g = None if gates is None else np.ascontiguousarray(gates, dtype=np.float32)
    _load().oracle_load_stats(_ptr(topk_idx), _ptr(g), N, E, k, int(C), _ptr(load), _ptr(used), _ptr(imp))
    return load, used, imp


def expert_ffn(x, W_up, W_down, t, e):
    """(h [d_ff], o [d]) in float64 for token t through expert e (STEP 8-10)."""
    x = np.ascontiguousarray(x)
    W_up = np.ascontiguousarray(W_up)
    W_down = np.ascontiguousarray(W_down)
    _, d = x.shape
    d_ff = W_up.shape[1]
    h = np.empty(d_ff, dtype=np.float64)
    o = np.empty(d, dtype=np.float64)
    _load().oracle_expert_ffn(_ptr(x), _dt(x), _ptr(W_up), _ptr(W_down), int(t), int(e), d, d_ff,
                              _ptr(h), _ptr(o))
    return h, o


ACT_RELU, ACT_GELU = 1, 2


def expert_ffn_ex(x, W_up, W_down, t, e, act=ACT_RELU, b_up=None, b_down=None):
    """(h, o) for the nanoMoE expert variant (slide 32): optional biases, ReLU or GELU."""
    x = np.ascontiguousarray(x)
    W_up = np.ascontiguousarray(W_up)
    W_down = np.ascontiguousarray(W_down)
    _, d = x.shape
    d_ff = W_up.shape[1]
    h = np.empty(d_ff, dtype=np.float64)
    o = np.empty(d, dtype=np.float64)
    bu = None if b_up is None else np.ascontiguousarray(b_up, dtype=np.float32)
    bd = None if b_down is None else np.ascontiguousarray(b_down, dtype=np.float32)
    _load().oracle_expert_ffn_ex(_ptr(x), _dt(x), _ptr(W_up), _ptr(W_down), _ptr(bu), _ptr(bd), int(act),
                                 int(t), int(e), d, d_ff, _ptr(h), _ptr(o))
    return h, o


def ffn_combine(x, W_up, W_down, topk_idx, gates, slot, tokens=None, nthreads=1, act=ACT_RELU,
                b_up=None, b_down=None):
    """y rows (float64) for the listed tokens (STEP 11-12; slides 38-40)."""
    x = np.ascontiguousarray(x)
    W_up = np.ascontiguousarray(W_up)
    W_down = np.ascontiguousarray(W_down)
    topk_idx = np.ascontiguousarray(topk_idx, dtype=np.int32)
    gates = np.ascontiguousarray(gates, dtype=np.float32)
    slot = np.ascontiguousarray(slot, dtype=np.int32)
    N, d = x.shape
    d_ff = W_up.shape[1]
    k = topk_idx.shape[1]
    if tokens is None:
        tokens = np.arange(N, dtype=np.int64)
    tokens = np.ascontiguousarray(tokens, dtype=np.int64)
    y = np.empty((len(tokens), d), dtype=np.float64)
    bu = None if b_up is None else np.ascontiguousarray(b_up, dtype=np.float32)
    bd = None if b_down is None else np.ascontiguousarray(b_down, dtype=np.float32)
    _load().oracle_ffn_combine_ex(_ptr(x), _dt(x), _ptr(W_up), _ptr(W_down), _ptr(bu), _ptr(bd), int(act),
                                  _ptr(topk_idx), _ptr(gates), _ptr(slot), d, d_ff, k, _ptr(tokens),
                                  len(tokens), _ptr(y), int(nthreads))
    return y


def forward(x, W_g, b_g, noise, sigma, k, cf, W_up, W_down, logits=None, tokens=None,
            nthreads=1, act=ACT_RELU, b_up=None, b_down=None):
    """The whole layer.  ``logits`` (optional) replaces the oracle's own s_raw,
    so routing can be replayed from another implementation's fp32 logits.
    Returns a dict with every intermediate."""
    N = x.shape[0]
    E = W_g.shape[0]
    s_raw = router_logits(x, W_g, b_g) if logits is None else np.asarray(logits, np.float32)
    topk_idx, gates = route_from_logits(s_raw, k, noise, sigma)
    C = capacity(N, E, k, cf)
    slot, counts = assign_slots(topk_idx, E, C)
    y = ffn_combine(x, W_up, W_down, topk_idx, gates, slot, tokens, nthreads, act, b_up, b_down)
    return dict(s_raw=s_raw, topk_idx=topk_idx, gates=gates, C=C, slot=slot, counts=counts,
                y=y, tokens=tokens)
