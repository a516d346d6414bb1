"""The C-ABI library on the host: it loads, exports every call include/moe.h
declares, and rejects bad arguments before launching anything (CPU only)."""
import ctypes
import math
import os
import re
import subprocess
import sys

import pytest

from sparse_mixture_experts_noisy_b200 import moe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    from sparse_mixture_experts_noisy_b200.build import build
    build()
    return moe.load_library()


def header_names():
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    return sorted(set(re.findall(r"MOE_API\s+[\w\s\*]*?\b(moe_\w+)\s*\(", src)))


def test_header_declares_the_binding_exports():
    assert header_names() == sorted(moe.EXPORTS)


def test_library_exports_every_declared_symbol(L):
    for name in header_names():
        assert hasattr(L, name), name
    # nothing beyond the C ABI is exported
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", moe.LIB_PATH], capture_output=True, text=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    assert exported == set(header_names())


def test_capacity_matches_the_oracle_formula(L):
    import oracle
    for N, E, k, cf in [(8192, 8, 2, 1.25), (16384, 8, 2, 1.25), (32768, 64, 6, 1.0), (64, 8, 2, math.inf),
                        (10, 3, 2, 1.0), (4, 3, 2, 100.0), (0, 4, 2, 1.0), (7, 5, 5, 0.3)]:
        assert moe.capacity(N, E, k, cf) == oracle.capacity(N, E, k, cf)
    assert moe.capacity(4, 3, 2, 0.0) == -1
    assert moe.capacity(4, 3, 2, float("nan")) == -1
    assert moe.capacity(4, 3, 4, 1.0) == -1


def test_gathered_rows(L):
    # min(N*k, E*C) rounded up to 128
    assert moe.gathered_rows(16384, 8, 2, 1.25) == 32768
    assert moe.gathered_rows(64, 8, 2, math.inf) == 128
    assert moe.gathered_rows(32768, 64, 6, 1.0) == 196608
    assert moe.gathered_rows(1000, 8, 2, 0.5) == 1024   # C = 125, E*C = 1000
    assert moe.gathered_rows(0, 8, 2, 1.0) == 0


def _err(L):
    return L.moe_last_error().decode()


def test_route_rejects_bad_shapes_without_launching(L):
    P = ctypes.c_void_p
    assert L.moe_route(None, 1, None, None, None, 0.0, 4, 8, 4, 5, None, None, None, None) == 1
    assert "k must be" in _err(L)
    assert L.moe_route(None, 1, None, None, None, 0.0, 4, 8, 300, 2, None, None, None, None) == 1
    assert L.moe_route(None, 7, None, None, None, 0.0, 4, 8, 4, 2, None, None, None, None) == 1
    assert L.moe_route(None, 1, None, None, None, 0.0, 4, 8, 4, 2, None, None, None, None) == 1
    assert "x must not be NULL" in _err(L)
    # misaligned pointer
    assert L.moe_route(P(0x1001), 1, P(0x2000), None, None, 0.0, 4, 8, 4, 2, None, P(0x3000), P(0x4000),
                       None) == 1
    assert "16-byte aligned" in _err(L)
    assert L.moe_route(P(0x1000), 1, P(0x2000), None, None, float("nan"), 4, 8, 4, 2, None, P(0x3000),
                       P(0x4000), None) == 1


def test_dispatch_rejects_bad_capacity_and_workspace(L):
    P = ctypes.c_void_p
    a = P(0x10000)
    assert L.moe_dispatch(a, a, 1, 16, 8, 4, 2, 0.0, a, a, a, a, a, 1 << 20, None) == 1
    assert "capacity factor" in _err(L)
    assert L.moe_dispatch(a, a, 1, 16, 8, 4, 2, float("nan"), a, a, a, a, a, 1 << 20, None) == 1
    assert L.moe_dispatch(a, a, 1, 16, 8, 4, 2, 1.0, a, a, a, a, a, 8, None) == 3
    assert "workspace" in _err(L)
    assert L.moe_dispatch(a, a, 1, 16, 8, 4, 2, 1.0, a, a, a, a, None, 1 << 20, None) == 3


def test_expert_ffn_and_forward_reject_bad_arguments(L):
    P = ctypes.c_void_p
    a = P(0x10000)
    assert L.moe_expert_ffn(a, a, a, a, a, 1, 100, 8, 16, 4, a, a, 1 << 30, None) == 1   # rows % 128
    assert "multiple of 128" in _err(L)
    assert L.moe_expert_ffn(a, a, a, a, a, 1, 128, 8, 16, 4, a, a, 16, None) == 3
    assert L.moe_forward(a, 1, a, None, None, 0.0, 16, 8, 4, 16, 2, -1.0, a, a, a, None, None, None, None,
                         None, a, 1 << 30, None) == 1
    assert L.moe_forward(a, 1, a, None, None, 0.0, 16, 8, 4, 16, 2, 1.0, a, a, a, None, None, None, None,
                         None, a, 64, None) == 3
    assert L.moe_forward(a, 1, a, None, None, float("inf"), 16, 8, 4, 16, 2, 1.0, a, a, a, None, None, None,
                         None, None, a, 1 << 30, None) == 1
    assert L.moe_check_status(None, None, None) == 1
    assert L.moe_debug_wait_timeout(10, None, 0, None) == 3
    assert L.moe_debug_wait_timeout(0, a, 4096, None) == 1


def test_load_stats_rejects_bad_arguments(L):
    P = ctypes.c_void_p
    a = P(0x10000)
    ws = int(L.moe_load_stats_workspace_size())
    assert ws >= 256 * 12
    assert L.moe_load_stats(a, None, 16, 300, 2, 1.0, a, a, None, a, ws, None) == 1   # E > 256
    assert L.moe_load_stats(a, None, 16, 4, 5, 1.0, a, a, None, a, ws, None) == 1     # k > E
    assert L.moe_load_stats(a, None, 16, 4, 2, 0.0, a, a, None, a, ws, None) == 1     # cf
    assert "capacity factor" in _err(L)
    assert L.moe_load_stats(a, None, 16, 4, 2, 1.0, None, a, None, a, ws, None) == 1  # load NULL
    assert L.moe_load_stats(a, P(0x10004), 16, 4, 2, 1.0, a, a, None, a, ws, None) == 1  # misaligned gates
    assert L.moe_load_stats(a, None, 16, 4, 2, 1.0, a, a, None, a, 8, None) == 3       # workspace
    assert "workspace" in _err(L)


def test_workspace_sizes_are_monotone(L):
    s1 = L.moe_workspace_size(1024, 256, 8, 512, 2, 1.25, 1)
    s2 = L.moe_workspace_size(2048, 256, 8, 512, 2, 1.25, 1)
    assert 0 < s1 < s2
    assert L.moe_workspace_size(1024, 256, 8, 512, 9, 1.25, 1) == 0
    assert L.moe_dispatch_workspace_size(1000, 8, 2) >= 4 * 4 * 2 * 8


def test_product_path_fails_loudly_without_the_library(tmp_path, monkeypatch):
    monkeypatch.setattr(moe, "_lib", None)
    with pytest.raises(ImportError):
        moe.load_library(str(tmp_path / "missing.so"))


def test_fused_small_batch_off_by_default():
    code = ("import sys; sys.path.insert(0, {root!r}); from sparse_mixture_experts_noisy_b200 import moe; "
            "print(int(moe.set_fused_small_batch(None)))")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = {k: v for k, v in os.environ.items() if k != "MOE_FUSED_DECODE"}
    r = subprocess.run([sys.executable, "-c", code.format(root=root)], cwd=root, env=env, capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == "0"

