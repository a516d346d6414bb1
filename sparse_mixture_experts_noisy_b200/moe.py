"""Python binding of libmoe.so (include/moe.h): argument marshalling only.

Every step of the layer runs in the library's CUDA kernels; torch provides
device memory and the stream.  There is no fallback: if the library is not
built, or no CUDA device is present, the calls raise.
"""
from __future__ import annotations

import ctypes
import math
import os
import threading

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "_lib", "libmoe.so")

MOE_F32, MOE_BF16 = 0, 1
ACT_RELU, ACT_GELU = 1, 2
STATUS_NAMES = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED", 3: "MOE_ERR_WORKSPACE",
                4: "MOE_ERR_CUDA", 5: "MOE_ERR_DEVICE_CHECK", 6: "MOE_ERR_TIMEOUT"}

EXPORTS = ("moe_capacity", "moe_gathered_rows", "moe_route", "moe_route_ex", "moe_route_workspace_size",
           "moe_check_route_status",
           "moe_dispatch_workspace_size", "moe_dispatch", "moe_dispatch_noalloc",
           "moe_shard_workspace_size", "moe_shard_count", "moe_shard_base", "moe_shard_dispatch",
           "moe_expert_ffn_workspace_size", "moe_expert_ffn", "moe_expert_ffn_ex", "moe_expert_ffn_train",
           "moe_backward_workspace_size", "moe_backward", "moe_combine",
           "moe_load_stats_workspace_size", "moe_load_stats",
           "moe_workspace_size", "moe_forward", "moe_forward_ex", "moe_forward_launches",
           "moe_set_fused_small_batch", "moe_check_status", "moe_debug_wait_timeout", "moe_num_sms", "moe_last_error")


class MoeError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{STATUS_NAMES.get(code, code)}: {msg}")
        self.code = code


_lock = threading.Lock()
_lib = None


def load_library(path: str = LIB_PATH):
    """Load libmoe.so and declare its signatures.  Raises if it is missing."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(path):
            raise ImportError(f"libmoe.so not built at {path}; run `python -m "
                              "sparse_mixture_experts_noisy_b200.build` (there is no CPU fallback)")
        L = ctypes.CDLL(path)
        P, I, I64, U32, F, D, SZ = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_uint32,
                                    ctypes.c_float, ctypes.c_double, ctypes.c_size_t)
        sig = {
            "moe_capacity": (I64, [I64, I, I, D]),
            "moe_gathered_rows": (I64, [I64, I, I, D]),
            "moe_route": (I, [P, I, P, P, P, F, I64, I, I, I, P, P, P, P]),
            "moe_route_ex": (I, [P, I, P, P, P, F, I64, I, I, I, P, P, P, P, SZ, P]),
            "moe_route_workspace_size": (SZ, [I, I]),
            "moe_check_route_status": (I, [P, ctypes.POINTER(U32)]),
            "moe_dispatch_workspace_size": (SZ, [I64, I, I]),
            "moe_dispatch": (I, [P, P, I, I64, I, I, I, D, P, P, P, P, P, SZ, P]),
            "moe_dispatch_noalloc": (I, [P, P, I, I64, I, I, I, D, P, P, P, P, P]),
            "moe_load_stats_workspace_size": (SZ, []),
            "moe_load_stats": (I, [P, P, I64, I, I, D, P, P, P, P, SZ, P]),
            "moe_shard_workspace_size": (SZ, [I64, I, I]),
            "moe_shard_count": (I, [P, I64, I, I, P, P, SZ, P]),
            "moe_shard_base": (I, [P, I, I, I, I, P, P]),
            "moe_shard_dispatch": (I, [P, P, I, I64, I, I, I, I64, P, P, P, P, P, P, P, SZ, P]),
            "moe_expert_ffn_workspace_size": (SZ, [I64, I, I, I, I]),
            "moe_expert_ffn": (I, [P, P, P, P, P, I, I64, I, I, I, P, P, SZ, P]),
            "moe_expert_ffn_ex": (I, [P, P, P, P, P, I, I64, I, I, I, I, P, P, P, P, SZ, P]),
            "moe_expert_ffn_train": (I, [P, P, P, P, P, I, I64, I, I, I, P, P, P, SZ, P]),
            "moe_backward_workspace_size": (SZ, [I64, I, I, I, I, I64, I]),
            "moe_backward": (I, [P, I, P, P, P, I64, I, I, I, I, I64, P, P, P, P, P, P, P, P, P, P, P, P, P, P,
                                 P, SZ, P]),
            "moe_combine": (I, [P, P, P, P, P, I, I64, I, I, P, P]),
            "moe_workspace_size": (SZ, [I64, I, I, I, I, D, I]),
            "moe_forward": (I, [P, I, P, P, P, F, I64, I, I, I, I, D, P, P, P, P, P, P, P, P, P, SZ, P]),
            "moe_forward_ex": (I, [P, I, P, P, P, F, I64, I, I, I, I, D, P, P, I, P, P, P, P, P, P, P, P, P, SZ,
                                   P]),
            "moe_forward_launches": (I, [I64, I, I, I, I, D, I]),
            "moe_set_fused_small_batch": (I, [I]),
            "moe_check_status": (I, [P, P, ctypes.POINTER(U32)]),
            "moe_debug_wait_timeout": (I, [U32, P, SZ, P]),
            "moe_num_sms": (I, []),
            "moe_last_error": (ctypes.c_char_p, []),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
        return L


def _check(code: int):
    if code != 0:
        raise MoeError(code, load_library().moe_last_error().decode())


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return MOE_BF16
    if t.dtype == torch.float32:
        return MOE_F32
    raise TypeError(f"storage type must be float32 or bfloat16, got {t.dtype}")


def _stream(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _cuda(t, name):
    if t is None:
        return
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _cf(cf) -> float:
    return math.inf if cf is None else float(cf)


def capacity(N: int, E: int, k: int, cf) -> int:
    return int(load_library().moe_capacity(N, E, k, _cf(cf)))


def gathered_rows(N: int, E: int, k: int, cf) -> int:
    return int(load_library().moe_gathered_rows(N, E, k, _cf(cf)))


def num_sms() -> int:
    return int(load_library().moe_num_sms())


def new_workspace(nbytes, device):
    """A device workspace whose status word (first 4 bytes) starts at zero."""
    ws = torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)
    ws[:256].zero_()
    return ws


def route_workspace(d, E, device):
    """A workspace with which moe_route takes moe_forward's router path."""
    return new_workspace(load_library().moe_route_workspace_size(d, E), device)


def moe_route(x, W_g, k, b_g=None, noise=None, sigma=0.0, want_logits=True, stream=None, status=None):
    """-> (topk_idx [N,k] int32, gates [N,k] fp32, logits [N,E] fp32 or None).
    status (a workspace, nullable): its first 4 bytes record a router timeout
    (read them with check_status); None records into the library's own word
    (check_route_status).  A workspace from route_workspace() also selects the
    pre-split router of moe_forward."""
    L = load_library()
    for t, n in ((x, "x"), (W_g, "W_g"), (b_g, "b_g"), (noise, "noise")):
        _cuda(t, n)
    N, d = x.shape
    E = W_g.shape[0]
    dev = x.device
    topk = torch.empty((N, k), dtype=torch.int32, device=dev)
    gates = torch.empty((N, k), dtype=torch.float32, device=dev)
    logits = torch.empty((N, E), dtype=torch.float32, device=dev) if want_logits else None
    _cuda(status, "status")
    _check(L.moe_route_ex(_p(x), _dt(x), _p(W_g), _p(b_g), _p(noise), float(sigma), N, d, E, k,
                          _p(logits), _p(topk), _p(gates), _p(status), 0 if status is None else status.numel(),
                          _stream(stream)))
    return topk, gates, logits


def check_route_status(stream=None):
    """Read/clear the library's router status word (moe_route without one) -> (code, raw word)."""
    word = ctypes.c_uint32(0)
    code = load_library().moe_check_route_status(_stream(stream), ctypes.byref(word))
    return int(code), int(word.value)


def moe_dispatch(topk_idx, x, E, cf, stream=None):
    """-> dict(slot, counts, offsets, x_gathered, rows, C)."""
    L = load_library()
    _cuda(topk_idx, "topk_idx")
    _cuda(x, "x")
    N, d = x.shape
    k = topk_idx.shape[1]
    dev = x.device
    rows = L.moe_gathered_rows(N, E, k, _cf(cf))
    if rows < 0:
        raise MoeError(1, "invalid capacity arguments")
    slot = torch.empty((N, k), dtype=torch.int32, device=dev)
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    xg = torch.empty((rows, d), dtype=x.dtype, device=dev)
    wsb = L.moe_dispatch_workspace_size(N, E, k)
    ws = torch.empty(max(wsb, 256), dtype=torch.uint8, device=dev)
    _check(L.moe_dispatch(_p(topk_idx), _p(x), _dt(x), N, d, E, k, _cf(cf), _p(slot), _p(counts),
                          _p(offsets), _p(xg), _p(ws), ws.numel(), _stream(stream)))
    return dict(slot=slot, counts=counts, offsets=offsets, x_gathered=xg, rows=rows,
                C=capacity(N, E, k, cf))


def moe_dispatch_noalloc(topk_idx, x, E, cf, stream=None):
    """moe_dispatch for callers that cannot allocate device memory at dispatch
    time: the library's fixed scratch array replaces the workspace.  The
    output tensors here are allocated by torch for convenience; a caller
    without an allocator passes its own buffers to the C entry point.
    -> dict(slot, counts, offsets, x_gathered, rows, C)."""
    L = load_library()
    _cuda(topk_idx, "topk_idx")
    _cuda(x, "x")
    N, d = x.shape
    k = topk_idx.shape[1]
    dev = x.device
    rows = L.moe_gathered_rows(N, E, k, _cf(cf))
    if rows < 0:
        raise MoeError(1, "invalid capacity arguments")
    slot = torch.empty((N, k), dtype=torch.int32, device=dev)
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    xg = torch.empty((rows, d), dtype=x.dtype, device=dev)
    _check(L.moe_dispatch_noalloc(_p(topk_idx), _p(x), _dt(x), N, d, E, k, _cf(cf), _p(slot), _p(counts),
                                  _p(offsets), _p(xg), _stream(stream)))
    return dict(slot=slot, counts=counts, offsets=offsets, x_gathered=xg, rows=rows,
                C=capacity(N, E, k, cf))


def moe_shard_count(topk_idx, E, ws, stream=None):
    """This shard's [k, E] int32 counts of j-th choices per expert (device).
    `ws` (from shard_workspace) must then go, untouched, to moe_shard_dispatch."""
    L = load_library()
    N, k = topk_idx.shape
    counts_je = torch.empty((k, E), dtype=torch.int32, device=topk_idx.device)
    _check(L.moe_shard_count(_p(topk_idx), N, E, k, _p(counts_je), _p(ws), ws.numel(), _stream(stream)))
    return counts_je


def shard_workspace(N_local, E, k, device):
    n = load_library().moe_shard_workspace_size(N_local, E, k)
    return torch.empty(max(n, 256), dtype=torch.uint8, device=device)


def moe_shard_base(all_counts, rank, stream=None):
    """all_counts [G, k, E] int32 (device, rank order) -> base [k, E] int32."""
    L = load_library()
    G, k, E = all_counts.shape
    base = torch.empty((k, E), dtype=torch.int32, device=all_counts.device)
    _check(L.moe_shard_base(_p(all_counts.contiguous()), G, rank, E, k, _p(base), _stream(stream)))
    return base


def moe_shard_dispatch(topk_idx, x, E, C, counts_je, base, ws, stream=None):
    """-> dict(slot, counts, offsets, x_gathered, rows) for this shard."""
    L = load_library()
    N, d = x.shape
    k = topk_idx.shape[1]
    dev = x.device
    rows = (N * k + 127) // 128 * 128
    slot = torch.empty((N, k), dtype=torch.int32, device=dev)
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    xg = torch.empty((rows, d), dtype=x.dtype, device=dev)
    _check(L.moe_shard_dispatch(_p(topk_idx), _p(x), _dt(x), N, d, E, k, int(C), _p(counts_je), _p(base),
                                _p(slot), _p(counts), _p(offsets), _p(xg), _p(ws), ws.numel(), _stream(stream)))
    return dict(slot=slot, counts=counts, offsets=offsets, x_gathered=xg, rows=rows)


def moe_expert_ffn(x_gathered, offsets, counts, W_up, W_down, stream=None, ws=None, out=None, act=ACT_RELU,
                   b_up=None, b_down=None):
    """-> out_gathered [rows, d] (rows outside the kept ranges unspecified).
    act/b_up/b_down select the nanoMoE expert variant (GELU, biases)."""
    L = load_library()
    for t, n in ((x_gathered, "x_gathered"), (offsets, "offsets"), (counts, "counts"), (W_up, "W_up"),
                 (W_down, "W_down")):
        _cuda(t, n)
    rows, d = x_gathered.shape
    E, d_ff, _ = W_up.shape
    dt = _dt(x_gathered)
    wsb = L.moe_expert_ffn_workspace_size(rows, d, E, d_ff, dt)
    if ws is None:
        ws = new_workspace(wsb, x_gathered.device)
    if out is None:
        out = torch.empty((rows, d), dtype=x_gathered.dtype, device=x_gathered.device)
    for t, n in ((b_up, "b_up"), (b_down, "b_down")):
        _cuda(t, n)
    _check(L.moe_expert_ffn_ex(_p(x_gathered), _p(offsets), _p(counts), _p(W_up), _p(W_down), dt, rows, d,
                               d_ff, E, int(act), _p(b_up), _p(b_down), _p(out), _p(ws), ws.numel(),
                               _stream(stream)))
    return out


def moe_expert_ffn_train(x_gathered, offsets, counts, W_up, W_down, stream=None, ws=None):
    """Expert FFN that keeps the hidden activations for the backward.
    -> (out_gathered [rows, d], H [rows, d_ff])."""
    L = load_library()
    for t, n in ((x_gathered, "x_gathered"), (offsets, "offsets"), (counts, "counts"), (W_up, "W_up"),
                 (W_down, "W_down")):
        _cuda(t, n)
    rows, d = x_gathered.shape
    E, d_ff, _ = W_up.shape
    dt = _dt(x_gathered)
    if ws is None:
        ws = new_workspace(L.moe_expert_ffn_workspace_size(rows, d, E, d_ff, dt), x_gathered.device)
    out = torch.empty((rows, d), dtype=x_gathered.dtype, device=x_gathered.device)
    H = torch.empty((rows, d_ff), dtype=x_gathered.dtype, device=x_gathered.device)
    _check(L.moe_expert_ffn_train(_p(x_gathered), _p(offsets), _p(counts), _p(W_up), _p(W_down), dt, rows, d, d_ff,
                                  E, _p(out), _p(H), _p(ws), ws.numel(), _stream(stream)))
    return out, H


def moe_backward(x, W_g, W_up, W_down, k, topk_idx, gates, slot, offsets, counts, x_gathered, H, out_gathered, dy,
                 stream=None, ws=None):
    """Gradients of sum(dy * y) for the routing of a staged forward.
    -> dict(dx [N, d] of x's dtype, dW_g [E, d], db_g [E], dW_up [E, d_ff, d], dW_down [E, d, d_ff] fp32)."""
    L = load_library()
    for t, n in ((x, "x"), (W_g, "W_g"), (W_up, "W_up"), (W_down, "W_down"), (topk_idx, "topk_idx"),
                 (gates, "gates"), (slot, "slot"), (offsets, "offsets"), (counts, "counts"),
                 (x_gathered, "x_gathered"), (H, "H"), (out_gathered, "out_gathered"), (dy, "dy")):
        _cuda(t, n)
    N, d = x.shape
    E, d_ff, _ = W_up.shape
    rows = x_gathered.shape[0]
    dt = _dt(x)
    dev = x.device
    if ws is None:
        ws = new_workspace(L.moe_backward_workspace_size(N, d, E, d_ff, k, rows, dt), dev)
    out = dict(dx=torch.empty((N, d), dtype=x.dtype, device=dev),
               dW_g=torch.empty((E, d), dtype=torch.float32, device=dev),
               db_g=torch.empty(E, dtype=torch.float32, device=dev),
               dW_up=torch.empty((E, d_ff, d), dtype=torch.float32, device=dev),
               dW_down=torch.empty((E, d, d_ff), dtype=torch.float32, device=dev))
    _check(L.moe_backward(_p(x), dt, _p(W_g), _p(W_up), _p(W_down), N, d, E, d_ff, k, rows, _p(topk_idx),
                          _p(gates), _p(slot), _p(offsets), _p(counts), _p(x_gathered), _p(H), _p(out_gathered),
                          _p(dy), _p(out["dx"]), _p(out["dW_g"]), _p(out["db_g"]), _p(out["dW_up"]),
                          _p(out["dW_down"]), _p(ws), ws.numel(), _stream(stream)))
    out["ws"] = ws
    return out


def moe_combine(out_gathered, slot, topk_idx, offsets, gates, stream=None, y=None):
    """-> y [N, d]."""
    L = load_library()
    N, k = slot.shape
    d = out_gathered.shape[1]
    if y is None:
        y = torch.empty((N, d), dtype=out_gathered.dtype, device=out_gathered.device)
    _check(L.moe_combine(_p(out_gathered), _p(slot), _p(topk_idx), _p(offsets), _p(gates),
                         _dt(out_gathered), N, d, k, _p(y), _stream(stream)))
    return y


def moe_load_stats(topk_idx, E, cf, gates=None, stream=None):
    """Per-expert load of a routed batch (slide 14's used_capacity and more).
    -> dict(load [E] int32, used [E] int32, importance [E] float64 or None)."""
    L = load_library()
    _cuda(topk_idx, "topk_idx")
    _cuda(gates, "gates")
    N, k = topk_idx.shape
    dev = topk_idx.device
    load = torch.empty(E, dtype=torch.int32, device=dev)
    used = torch.empty(E, dtype=torch.int32, device=dev)
    imp = torch.empty(E, dtype=torch.float64, device=dev) if gates is not None else None
    ws = torch.empty(max(int(L.moe_load_stats_workspace_size()), 256), dtype=torch.uint8, device=dev)
    _check(L.moe_load_stats(_p(topk_idx), _p(gates), N, E, k, _cf(cf), _p(load), _p(used), _p(imp), _p(ws),
                            ws.numel(), _stream(stream)))
    return dict(load=load, used=used, importance=imp)


def workspace_size(N, d, E, d_ff, k, cf, dtype) -> int:
    dt = MOE_BF16 if dtype == torch.bfloat16 else MOE_F32
    return int(load_library().moe_workspace_size(N, d, E, d_ff, k, _cf(cf), dt))


def forward_launches(N, d, E, d_ff, k, cf, dtype) -> int:
    dt = MOE_BF16 if dtype == torch.bfloat16 else MOE_F32
    return int(load_library().moe_forward_launches(N, d, E, d_ff, k, _cf(cf), dt))


def set_fused_small_batch(on: bool | None) -> bool:
    """Select (True/False) or query (None) the single-launch small-batch layer
    for this process; returns the previous setting."""
    return bool(load_library().moe_set_fused_small_batch(-1 if on is None else int(bool(on))))


def moe_forward(x, W_g, W_up, W_down, k, cf, b_g=None, noise=None, sigma=0.0, y=None, ws=None,
                intermediates=False, stream=None, act=ACT_RELU, b_up=None, b_down=None):
    """The whole layer.  -> y, or (y, dict of logits/topk_idx/gates/slot/counts).
    act/b_up/b_down select the nanoMoE expert variant (GELU, biases)."""
    L = load_library()
    for t, n in ((x, "x"), (W_g, "W_g"), (W_up, "W_up"), (W_down, "W_down"), (b_g, "b_g"),
                 (noise, "noise"), (b_up, "b_up"), (b_down, "b_down")):
        _cuda(t, n)
    N, d = x.shape
    E, d_ff, _ = W_up.shape
    dev = x.device
    wsb = workspace_size(N, d, E, d_ff, k, cf, x.dtype)
    if wsb == 0:
        raise MoeError(1, "invalid layer arguments")
    if ws is None:
        ws = new_workspace(wsb, dev)
    if y is None:
        y = torch.empty((N, d), dtype=x.dtype, device=dev)
    inter = None
    if intermediates:
        inter = dict(logits=torch.empty((N, E), dtype=torch.float32, device=dev),
                     topk_idx=torch.empty((N, k), dtype=torch.int32, device=dev),
                     gates=torch.empty((N, k), dtype=torch.float32, device=dev),
                     slot=torch.empty((N, k), dtype=torch.int32, device=dev),
                     counts=torch.empty(E, dtype=torch.int32, device=dev))
    g = (lambda n: _p(inter[n])) if inter else (lambda n: None)
    _check(L.moe_forward_ex(_p(x), _dt(x), _p(W_g), _p(b_g), _p(noise), float(sigma), N, d, E, d_ff, k,
                            _cf(cf), _p(W_up), _p(W_down), int(act), _p(b_up), _p(b_down), _p(y),
                            g("logits"), g("topk_idx"), g("gates"), g("slot"), g("counts"), _p(ws),
                            ws.numel(), _stream(stream)))
    return (y, inter) if intermediates else y


def check_status(ws, stream=None):
    """Synchronise and read/clear a workspace's status word -> (code, raw word)."""
    L = load_library()
    word = ctypes.c_uint32(0)
    code = L.moe_check_status(_p(ws), _stream(stream), ctypes.byref(word))
    return int(code), int(word.value)


def debug_wait_timeout(timeout_us: int, ws, stream=None):
    _check(load_library().moe_debug_wait_timeout(int(timeout_us), _p(ws), ws.numel(), _stream(stream)))


class MoELayer:
    """Weights resident on the device plus a reusable workspace; __call__ runs
    moe_forward on the current stream without allocating."""

    def __init__(self, W_g, W_up, W_down, k, cf, b_g=None, sigma=0.0, max_tokens=None, act=ACT_RELU,
                 b_up=None, b_down=None):
        self.W_g, self.W_up, self.W_down, self.b_g = W_g, W_up, W_down, b_g
        self.act, self.b_up, self.b_down = int(act), b_up, b_down
        self.k, self.cf, self.sigma = int(k), cf, float(sigma)
        self.E, self.d_ff, self.d = W_up.shape
        self._ws = None
        self._ws_tokens = -1
        if max_tokens is not None:
            self._reserve(max_tokens, W_up.dtype)

    def _reserve(self, N, dtype):
        need = workspace_size(N, self.d, self.E, self.d_ff, self.k, self.cf, dtype)
        if self._ws is None or self._ws.numel() < need:
            self._ws = new_workspace(need, self.W_up.device)
        self._ws_tokens = N

    @property
    def workspace(self):
        return self._ws

    def __call__(self, x, noise=None, y=None, stream=None):
        if self._ws is None or x.shape[0] != self._ws_tokens:
            self._reserve(x.shape[0], x.dtype)
        return moe_forward(x, self.W_g, self.W_up, self.W_down, self.k, self.cf, b_g=self.b_g,
                           noise=noise, sigma=self.sigma, y=y, ws=self._ws, stream=stream, act=self.act,
                           b_up=self.b_up, b_down=self.b_down)


class GraphedForward:
    """moe_forward captured once in a CUDA graph over static buffers.

    The library launches every kernel of the layer on the capturing stream and
    allocates nothing, so the whole forward replays as one graph launch.  Copy
    new inputs into `.x` (and `.noise`) before `replay()`; the output lands in
    `.y`.  The graph bakes in the buffers' addresses: keep this object (and
    the layer's weights and workspace) alive while replaying."""

    def __init__(self, layer: MoELayer, x, noise=None):
        self.layer = layer
        self.x = x
        self.noise = noise
        self.y = torch.empty_like(x)
        layer._reserve(x.shape[0], x.dtype)
        side = torch.cuda.Stream(device=x.device)
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            layer(x, noise=noise, y=self.y)   # first call outside the capture
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize(x.device)
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            layer(x, noise=noise, y=self.y)

    def replay(self):
        self.graph.replay()
        return self.y


class HostPipeline:
    """The layer over a stream of batches that live in (pinned) host memory.

    Two graphed forwards over two sets of device buffers alternate.  Batch i's
    inputs are copied in on one stream, its forward replays on the current
    stream, and its output is copied out on a third, with events between them,
    so the copy of batch i+1 in and of batch i-1 out overlap the forward of
    batch i.  `submit(x_h, y_h, noise_h)` enqueues one batch (x_h, noise_h
    pinned host inputs, y_h the pinned host output); `synchronize()` waits for
    all of them.  Host buffers must stay untouched until their batch is done."""

    def __init__(self, layer: MoELayer, x_example, noise_example=None):
        dev = x_example.device
        self.graphs = []
        for _ in range(2):
            xb = torch.empty_like(x_example)
            nb = None if noise_example is None else torch.empty_like(noise_example)
            if nb is not None:
                nb.copy_(noise_example)
            xb.copy_(x_example)
            self.graphs.append(GraphedForward(layer, xb, nb))
        self.s_in = torch.cuda.Stream(device=dev)
        self.s_out = torch.cuda.Stream(device=dev)
        self.h2d = [torch.cuda.Event() for _ in range(2)]
        self.done = [torch.cuda.Event() for _ in range(2)]
        self.d2h = [torch.cuda.Event() for _ in range(2)]
        self.used = [False, False]
        self.i = 0

    def submit(self, x_h, y_h, noise_h=None):
        b = self.i & 1
        g = self.graphs[b]
        comp = torch.cuda.current_stream()
        with torch.cuda.stream(self.s_in):
            if self.used[b]:
                self.s_in.wait_event(self.done[b])   # the forward of batch i-2 has read these inputs
            g.x.copy_(x_h, non_blocking=True)
            if noise_h is not None:
                g.noise.copy_(noise_h, non_blocking=True)
            self.h2d[b].record(self.s_in)
        comp.wait_event(self.h2d[b])
        if self.used[b]:
            comp.wait_event(self.d2h[b])             # batch i-2's output has left these buffers
        g.replay()
        self.done[b].record(comp)
        with torch.cuda.stream(self.s_out):
            self.s_out.wait_event(self.done[b])
            y_h.copy_(g.y, non_blocking=True)
            self.d2h[b].record(self.s_out)
        self.used[b] = True
        self.i += 1

    def synchronize(self):
        for b in range(2):
            if self.used[b]:
                self.d2h[b].synchronize()
