"""Plant plausible mistakes in copies of the oracle and check that the pins
catch every one of them (CPU only).

Each mutant is the oracle's C source with one textual change, compiled to a
temporary library and swapped in for the duration of the pin checks."""
import ctypes
import os
import subprocess

import pytest

import oracle.oracle as O
from tests import oracle_pins as P

MUTANTS = {
    "slots_token_major": (
        "for (int j = 0; j < k; ++j) {\n        for (int64_t t = 0; t < N; ++t) {",
        "for (int64_t t = 0; t < N; ++t) {\n        for (int j = 0; j < k; ++j) {"),
    "noise_dropped": ("v = v + scaled;", "v = v + 0.0f * scaled;"),
    "noise_fused": ("float scaled = sigma * noise[(size_t)t * E + e];\n                v = v + scaled;",
                    "v = fmaf(sigma, noise[(size_t)t * E + e], v);"),
    "ties_to_higher_index": ("return (ia < ib) ? -1 : (ia > ib);", "return (ia > ib) ? -1 : (ia < ib);"),
    "ascending_scores": ("if (sa > sb) return -1;\n    if (sa < sb) return 1;",
                         "if (sa < sb) return -1;\n    if (sa > sb) return 1;"),
    "softmax_over_all_experts": ("for (int j = 0; j < k; ++j)\n            denom += exp((double)s[idx[j]]",
                                 "for (int j = 0; j < E; ++j)\n            denom += exp((double)s[idx[j]]"),
    "relu_missing": ("h[f] = z > 0.0 ? z : 0.0;", "h[f] = z;"),
    "w_up_transposed": ("z += elem(W_up, dt, wrow + i)",
                        "z += elem(W_up, dt, (size_t)e * d_ff * d + (size_t)i * d_ff + f)"),
    "w_down_transposed": ("acc += elem(W_down, dt, wrow + f)",
                          "acc += elem(W_down, dt, (size_t)e * d * d_ff + (size_t)f * d + i)"),
    "capacity_off_by_one": ("(place < C) ? (int32_t)place : -1", "(place <= C) ? (int32_t)place : -1"),
    "dropped_pairs_contribute": ("if (jb->slot[(size_t)t * jb->k + j] < 0)\n                continue;", ""),
    "capacity_floor": ("double c = ceil(", "double c = floor("),
    "bf16_decode_shift": ("<< 16;", "<< 15;"),
    "counts_include_drops": ("counts[e] = (int32_t)(queue[e] < C ? queue[e] : C);",
                             "counts[e] = (int32_t)queue[e];"),
    "bias_dropped": ("s = s + b_g[e];", "s = s + 0.0f * b_g[e];"),
    "gate_not_applied": ("yt[i] += g * o[i];", "yt[i] += o[i];"),
    "gelu_as_relu": ("if (act == 2)\n            h[f] = 0.5 * z * (1.0 + erf(z / sqrt(2.0)));",
                     "if (act == 3)\n            h[f] = 0.5 * z * (1.0 + erf(z / sqrt(2.0)));"),
    "gelu_unscaled_erf": ("erf(z / sqrt(2.0))", "erf(z)"),
    "up_bias_dropped": ("z += (double)b_up[(size_t)e * d_ff + f];", "z += 0.0 * b_up[(size_t)e * d_ff + f];"),
    "down_bias_dropped": ("acc += (double)b_down[(size_t)e * d + i];", "acc += 0.0 * b_down[(size_t)e * d + i];"),
    "softmax_not_shifted_sign": ("denom += exp((double)s[idx[j]] - top);",
                                 "denom += exp(top - (double)s[idx[j]]);"),
    "used_not_capped": ("used[e] = (int32_t)(q[e] < C ? q[e] : C);", "used[e] = (int32_t)q[e];"),
    "load_counts_once_per_token": ("            q[e] += 1;\n", "            q[e] += (j == 0);\n"),
    "bwd_relu_mask_missing": ("                dz[f] = (mk ? (mk[f] != 0) : (z[f] > 0.0)) ? acc : 0.0;",
                              "                dz[f] = acc;"),
    "bwd_mask_not_replayed_in_h": ("const int on = mk ? (mk[f] != 0) : (acc > 0.0);", "const int on = (acc > 0.0);"),
    "bwd_sampled_dx_relu_missing": ("dz[f] = relu_on(c, t, j, f, z[f]) ? acc : 0.0;", "dz[f] = acc;"),
    "bwd_sampled_weight_rows_ungated": ("                    const double d_o = gj * dyt[i];\n                    wd[i]",
                                        "                    const double d_o = dyt[i];\n                    wd[i]"),
    "bwd_sampled_router_term_missing": ("                dxt[i] += dsj * (double)c->W_g[(size_t)e * d + i];",
                                        "                dxt[i] += 0.0 * c->W_g[(size_t)e * d + i];"),
    "bwd_softmax_not_coupled": ("            const double ds = g[j] * (dg[j] - sum);",
                                "            const double ds = g[j] * dg[j];"),
    "bwd_dropped_choices_skipped": ("            const int e = ti[j];\n            db_g[e] += ds;",
                                    "            const int e = ti[j];\n            if (slot[(size_t)t * k + j] < 0)\n"
                                    "                continue;\n            db_g[e] += ds;"),
    "bwd_router_to_x_missing": ("                dxt[i] += ds * (double)W_g[(size_t)e * d + i];", ""),
    "bwd_dW_up_transposed": ("dW_up[((size_t)e * d_ff + f) * d + i] += dz[f] * elem(x, dt, (size_t)t * d + i);",
                             "dW_up[((size_t)e * d + i) * d_ff + f] += dz[f] * elem(x, dt, (size_t)t * d + i);"),
    "gate_mass_truncated": ("mass[e] += llrint(ldexp((double)gates[(size_t)t * k + j], 32));",
                            "mass[e] += (int64_t)ldexp((double)gates[(size_t)t * k + j], 32);"),
}


def _build_mutant(tmp_path, name, old, new):
    src = open(O._SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    path = tmp_path / f"{name}.c"
    path.write_text(src.replace(old, new))
    lib = tmp_path / f"lib{name}.so"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fPIC", "-shared",
                           "-o", str(lib), str(path), "-lm", "-lpthread"])
    return str(lib)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(tmp_path, name):
    old, new = MUTANTS[name]
    lib_path = _build_mutant(tmp_path, name, old, new)
    O._load()
    saved = O._lib
    try:
        mutant = ctypes.CDLL(lib_path)
        for fn in ("oracle_router_logits", "oracle_route_from_logits", "oracle_capacity",
                   "oracle_assign_slots", "oracle_expert_ffn", "oracle_ffn_combine",
                   "oracle_expert_ffn_ex", "oracle_ffn_combine_ex", "oracle_load_stats", "oracle_backward",
                   "oracle_backward_sampled"):
            getattr(mutant, fn).argtypes = getattr(saved, fn).argtypes
            getattr(mutant, fn).restype = getattr(saved, fn).restype
        O._lib = mutant
        caught = []
        for check in P.ALL_CHECKS:
            try:
                check()
            except AssertionError:
                caught.append(check.__name__)
        assert caught, f"mutant {name} passed every pin"
    finally:
        O._lib = saved
