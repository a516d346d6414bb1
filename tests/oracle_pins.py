"""Checks that pin the CPU oracle to facts fixed outside it.

Each check raises AssertionError on a mismatch.  They are plain functions so
that the regular tests and the planted-mistake test (which swaps in a mutated
build of the oracle) run the very same checks.

Sources of truth used here, none of which is the oracle's own code:
  * the nanoMoE slides' worked examples (tests/golden/*.txt, with citations),
  * brute-force enumeration of expert subsets and of queue places,
  * numpy/scipy float64 library routines (matmul, softmax) and torch's
    float64 autograd (for the backward),
  * closed forms and invariants of the definition (gates sum to 1, sigma = 0
    leaves the scores unchanged, k = E with no capacity limit is the dense
    softmax mixture, E = 1 and k = 1 is a plain ReLU MLP).
"""
from __future__ import annotations

import itertools
import math

import numpy as np
from scipy.special import softmax as sp_softmax

import oracle
from tests.golden import load_m1, load_m2


# ---------------------------------------------------------------- helpers
def brute_topk(scores: np.ndarray, k: int):
    """The k-subset S with min over S >= max outside S; among several (ties),
    the one whose sorted index tuple is smallest.  Returned in (score desc,
    index asc) order.  Only comparisons, no arithmetic."""
    E = len(scores)
    best = None
    for S in itertools.combinations(range(E), k):
        inside = [scores[i] for i in S]
        outside = [scores[i] for i in range(E) if i not in S]
        if outside and min(inside) < max(outside):
            continue
        if best is None or S < best:
            best = S
    return sorted(best, key=lambda i: (-scores[i], i))


def brute_slots(topk: np.ndarray, E: int, C: int):
    """Queue place of (t, j) = number of assignments to the same expert that
    come earlier, where earlier means a lower choice rank j, or the same j and
    a lower token index.  O((N k)^2)."""
    N, k = topk.shape
    slot = np.full((N, k), -1, dtype=np.int64)
    for t in range(N):
        for j in range(k):
            e = topk[t, j]
            place = 0
            for t2 in range(N):
                for j2 in range(k):
                    if topk[t2, j2] == e and (j2 < j or (j2 == j and t2 < t)):
                        place += 1
            slot[t, j] = place if place < C else -1
    counts = np.array([np.sum((topk == e) & (slot >= 0)) for e in range(E)])
    return slot, counts


def np_expert(x, W_up, W_down, e):
    """numpy float64: W_down[e] @ max(0, W_up[e] @ x)."""
    return W_down[e] @ np.maximum(W_up[e] @ x, 0.0)


# ---------------------------------------------------------------- checks
def check_m1():
    """Slides 11-13: kept indices and 3-decimal gates of the 8 printed tokens."""
    rows = load_m1()
    logits = np.array([r[0] for r in rows], dtype=np.float32)
    idx, g = oracle.route_from_logits(logits, 2)
    for t, (lg, kept, gates) in enumerate(rows):
        assert tuple(sorted(idx[t].tolist())) == kept, (t, idx[t], kept)
        # descending order: the first choice has the larger logit
        assert lg[idx[t][0]] >= lg[idx[t][1]]
        by_index = {int(idx[t][j]): float(g[t][j]) for j in range(2)}
        for e, expect in zip(kept, gates):
            assert abs(by_index[e] - expect) <= 5e-4 + 1e-7, (t, e, by_index[e], expect)


def check_m2_slots():
    """Slides 15-23: queue places without a cut, and the cut at capacity 1."""
    m2 = load_m2()
    topk = np.array(m2["topk"], dtype=np.int32)
    slot, counts = oracle.assign_slots(topk, m2["E"], C=topk.shape[0])
    assert slot.tolist() == m2["rank_nocap"], slot.tolist()
    slot, counts = oracle.assign_slots(topk, m2["E"], C=m2["C"])
    assert slot.tolist() == m2["slot_cap1"], slot.tolist()
    assert counts.tolist() == m2["used"], counts.tolist()


def check_m2_combine(seed=3):
    """Slides 24-29 and 38-40: token 0 gets 0.6 a + 0.3 a', token 1 gets 0.3 b,
    tokens 2 and 3 get zero rows (their choices were all dropped)."""
    m2 = load_m2()
    rng = np.random.default_rng(seed)
    N, E, k, d, d_ff = 4, m2["E"], m2["k"], 5, 7
    x = rng.standard_normal((N, d)).astype(np.float32)
    W_up = rng.standard_normal((E, d_ff, d)).astype(np.float32)
    W_down = rng.standard_normal((E, d, d_ff)).astype(np.float32)
    topk = np.array(m2["topk"], dtype=np.int32)
    gates = np.array(m2["gates"], dtype=np.float32)
    slot = np.array(m2["slot_cap1"], dtype=np.int32)
    y = oracle.ffn_combine(x, W_up, W_down, topk, gates, slot)
    x64, u64, w64 = (a.astype(np.float64) for a in (x, W_up, W_down))
    for t, terms in enumerate(m2["combine"]):
        expect = np.zeros(d)
        for g, e, tok in terms:
            expect += np.float64(np.float32(g)) * np_expert(x64[tok], u64, w64, e)
        np.testing.assert_allclose(y[t], expect, rtol=1e-12, atol=1e-12)


def check_topk_bruteforce(seed=0, trials=300):
    """KeepTopK (the walkthrough's STEP 5) against subset enumeration, with
    random and deliberately tied scores; ties go to the lower index."""
    rng = np.random.default_rng(seed)
    for trial in range(trials):
        E = int(rng.integers(1, 9))
        k = int(rng.integers(1, E + 1))
        if trial % 2:
            s = rng.integers(-2, 3, size=E).astype(np.float32)  # many ties
        else:
            s = rng.standard_normal(E).astype(np.float32)
        idx, g = oracle.route_from_logits(s[None, :], k)
        assert idx[0].tolist() == brute_topk(s.tolist(), k), (s, k, idx[0])


def check_gates_invariants(seed=1):
    """STEP 6: kept gates sum to 1, masked experts get nothing (the kept set
    has exactly k distinct experts), k = 1 gives gate 1 exactly, and gate
    ratios follow exp(s_a - s_b)."""
    rng = np.random.default_rng(seed)
    for _ in range(50):
        E = int(rng.integers(2, 17))
        k = int(rng.integers(1, E + 1))
        s = (3 * rng.standard_normal((6, E))).astype(np.float32)
        idx, g = oracle.route_from_logits(s, k)
        for t in range(6):
            assert len(set(idx[t].tolist())) == k
            assert abs(float(np.sum(g[t].astype(np.float64))) - 1.0) < 1e-6
            assert np.all(g[t] > 0)
            if k == 1:
                assert g[t][0] == 1.0
            for a in range(k):
                for b in range(k):
                    r = float(g[t][a]) / float(g[t][b])
                    ref = math.exp(float(s[t, idx[t][a]]) - float(s[t, idx[t][b]]))
                    assert abs(r - ref) <= 1e-5 * ref, (r, ref)


def check_noise():
    """STEP 3-4: sigma = 0 leaves the scores as they are; a noise draw can
    reorder experts; the noisy score is the fp32 sum of s_raw and the fp32
    product sigma * eps (two separate roundings)."""
    rng = np.random.default_rng(7)
    s_raw = rng.standard_normal((16, 6)).astype(np.float32)
    eps = rng.standard_normal((16, 6)).astype(np.float32)
    i0, g0, s0 = oracle.route_from_logits(s_raw, 2, eps, 0.0, return_scores=True)
    i1, g1 = oracle.route_from_logits(s_raw, 2)
    assert np.array_equal(s0.view(np.uint32), s_raw.view(np.uint32))
    assert np.array_equal(i0, i1) and np.array_equal(g0.view(np.uint32), g1.view(np.uint32))
    # reorder: s_raw favours expert 0, the noise favours expert 1
    i2, _ = oracle.route_from_logits(np.array([[1.0, 0.0]], np.float32), 1,
                                     np.array([[0.0, 2.0]], np.float32), 1.0)
    assert i2[0, 0] == 1
    i3, _ = oracle.route_from_logits(np.array([[1.0, 0.0]], np.float32), 1,
                                     np.array([[0.0, 2.0]], np.float32), 0.25)
    assert i3[0, 0] == 0
    # two roundings: sigma = 1 + 2^-23, eps = 2^-24 - 2^-48.  The exact product
    # is 2^-24 (1 + 2^-24 - 2^-47), which rounds to 2^-24; 1 + 2^-24 is then a
    # tie and rounds to 1.  A fused multiply-add would round 1 + product up
    # to 1 + 2^-23.
    sr = np.array([[1.0, 0.0]], np.float32)
    ep = np.array([[2.0 ** -24 - 2.0 ** -48, 0.0]], np.float32)
    sig = np.float32(1.0 + 2.0 ** -23)
    assert float(ep[0, 0]) == 2.0 ** -24 - 2.0 ** -48   # exactly representable
    _, _, s4 = oracle.route_from_logits(sr, 1, ep, float(sig), return_scores=True)
    assert s4[0, 0] == np.float32(1.0)
    sigma = np.float32(0.75)
    _, _, s5 = oracle.route_from_logits(s_raw, 2, eps, float(sigma), return_scores=True)
    assert np.array_equal(s5, (s_raw + (sigma * eps).astype(np.float32)).astype(np.float32))


def check_capacity():
    """C = ceil(cf * N * k / E), at most N; cf = inf gives N."""
    assert oracle.capacity(8192, 8, 2, 1.25) == 2560
    assert oracle.capacity(16384, 8, 2, 1.25) == 5120
    assert oracle.capacity(32768, 64, 6, 1.0) == 3072
    assert oracle.capacity(64, 8, 2, math.inf) == 64
    assert oracle.capacity(10, 3, 2, 1.0) == 7
    assert oracle.capacity(4, 3, 2, 100.0) == 4
    assert oracle.capacity(4, 3, 2, 0.0) == -1
    assert oracle.capacity(4, 3, 2, float("nan")) == -1
    assert oracle.capacity(4, 3, 4, 1.0) == -1


def check_slots_bruteforce(seed=2, trials=60):
    """Queue places and drops against the counting definition, plus the
    invariants: per-expert load <= C, kept + dropped = N k, no drops when
    C = N, and a later choice rank is never kept while an earlier one to the
    same expert was dropped."""
    rng = np.random.default_rng(seed)
    for _ in range(trials):
        N = int(rng.integers(1, 13))
        E = int(rng.integers(1, 6))
        k = int(rng.integers(1, E + 1))
        topk = np.stack([rng.permutation(E)[:k] for _ in range(N)]).astype(np.int32)
        C = int(rng.integers(0, N + 1))
        slot, counts = oracle.assign_slots(topk, E, C)
        bs, bc = brute_slots(topk, E, C)
        assert np.array_equal(slot, bs) and np.array_equal(counts, bc)
        assert np.all(counts <= C)
        assert counts.sum() + np.sum(slot < 0) == N * k
        for e in range(E):
            kept_j = [j for t in range(N) for j in range(k) if topk[t, j] == e and slot[t, j] >= 0]
            drop_j = [j for t in range(N) for j in range(k) if topk[t, j] == e and slot[t, j] < 0]
            if kept_j and drop_j:
                assert max(kept_j) <= min(drop_j)
        slot_n, _ = oracle.assign_slots(topk, E, N)
        assert np.all(slot_n >= 0)


def check_logits_vs_numpy(seed=4):
    """STEP 2: s_raw = W_g x, against numpy's float64 matmul rounded to fp32
    (within one fp32 ulp, since numpy sums in another order), plus the fp32
    bias; bf16 inputs are read at their exact values."""
    from sparse_mixture_experts_noisy_b200.synth import f32_to_bf16_bits, bf16_bits_to_f32
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((9, 37)).astype(np.float32)
    W_g = rng.standard_normal((5, 37)).astype(np.float32)
    b_g = rng.standard_normal(5).astype(np.float32)
    for xin, xval in ((x, x), (f32_to_bf16_bits(x), bf16_bits_to_f32(f32_to_bf16_bits(x)))):
        ref = (xval.astype(np.float64) @ W_g.astype(np.float64).T).astype(np.float32)
        got = oracle.router_logits(xin, W_g)
        assert np.max(np.abs(got.view(np.int32) - ref.view(np.int32))) <= 1
        got_b = oracle.router_logits(xin, W_g, b_g)
        assert np.max(np.abs(got_b.view(np.int32) - (ref + b_g).view(np.int32))) <= 1
    one = np.array([[0x3F80, 0xC000, 0x3E80]], dtype=np.uint16)  # 1.0, -2.0, 0.25
    eye = np.eye(3, dtype=np.float32)
    assert oracle.router_logits(one, eye).tolist() == [[1.0, -2.0, 0.25]]


def check_ffn_vs_numpy(seed=5):
    """STEP 8-10 against numpy float64 matmuls, fp32 and bf16 storage."""
    from sparse_mixture_experts_noisy_b200.synth import f32_to_bf16_bits, bf16_bits_to_f32
    rng = np.random.default_rng(seed)
    E, d, d_ff = 3, 6, 11
    x = rng.standard_normal((4, d)).astype(np.float32)
    W_up = rng.standard_normal((E, d_ff, d)).astype(np.float32)
    W_down = rng.standard_normal((E, d, d_ff)).astype(np.float32)
    for conv in (lambda a: a, f32_to_bf16_bits):
        xs, us, ws = conv(x), conv(W_up), conv(W_down)
        val = (lambda a: a.astype(np.float64)) if xs.dtype == np.float32 else \
              (lambda a: bf16_bits_to_f32(a).astype(np.float64))
        for t in range(4):
            for e in range(E):
                h, o = oracle.expert_ffn(xs, us, ws, t, e)
                np.testing.assert_allclose(h, np.maximum(val(us)[e] @ val(xs)[t], 0), rtol=1e-12, atol=1e-12)
                np.testing.assert_allclose(o, np_expert(val(xs)[t], val(us), val(ws), e), rtol=1e-12, atol=1e-12)


def check_dense_mixture(seed=6):
    """With k = E and no capacity limit, nothing is masked or dropped and the
    layer is the dense softmax-gated mixture sum_e softmax(s)_e E_e(x)."""
    rng = np.random.default_rng(seed)
    N, d, E, d_ff = 7, 5, 4, 6
    x = rng.standard_normal((N, d)).astype(np.float32)
    W_g = rng.standard_normal((E, d)).astype(np.float32)
    W_up = rng.standard_normal((E, d_ff, d)).astype(np.float32)
    W_down = rng.standard_normal((E, d, d_ff)).astype(np.float32)
    out = oracle.forward(x, W_g, None, None, 0.0, E, math.inf, W_up, W_down)
    p = sp_softmax(out["s_raw"].astype(np.float64), axis=1)
    x64, u64, w64 = (a.astype(np.float64) for a in (x, W_up, W_down))
    for t in range(N):
        ref = sum(p[t, e] * np_expert(x64[t], u64, w64, e) for e in range(E))
        np.testing.assert_allclose(out["y"][t], ref, rtol=1e-6, atol=1e-6)


def check_single_expert_mlp(seed=8):
    """E = 1, k = 1: gate 1, nothing dropped with cf = 1, y = W_down relu(W_up x)."""
    rng = np.random.default_rng(seed)
    N, d, d_ff = 5, 4, 9
    x = rng.standard_normal((N, d)).astype(np.float32)
    W_g = rng.standard_normal((1, d)).astype(np.float32)
    W_up = rng.standard_normal((1, d_ff, d)).astype(np.float32)
    W_down = rng.standard_normal((1, d, d_ff)).astype(np.float32)
    out = oracle.forward(x, W_g, None, None, 0.0, 1, 1.0, W_up, W_down)
    assert np.all(out["gates"] == 1.0) and np.all(out["slot"][:, 0] == np.arange(N))
    ref = np.maximum(x.astype(np.float64) @ W_up[0].T.astype(np.float64), 0) @ W_down[0].T.astype(np.float64)
    np.testing.assert_allclose(out["y"], ref, rtol=1e-12, atol=1e-12)


def check_all_dropped_is_zero(seed=9):
    """A token whose every choice overflowed gets a zero row, not a
    renormalised one (slides 38-40, tokens 2 and 3)."""
    rng = np.random.default_rng(seed)
    N, d, E, d_ff, k = 6, 3, 2, 4, 1
    x = rng.standard_normal((N, d)).astype(np.float32)
    W_g = np.zeros((E, d), np.float32)
    b_g = np.array([1.0, 0.0], np.float32)      # every token picks expert 0
    W_up = rng.standard_normal((E, d_ff, d)).astype(np.float32)
    W_down = rng.standard_normal((E, d, d_ff)).astype(np.float32)
    out = oracle.forward(x, W_g, b_g, None, 0.0, k, 1.0, W_up, W_down)   # C = 3
    assert out["C"] == 3
    assert out["slot"][:, 0].tolist() == [0, 1, 2, -1, -1, -1]
    assert np.all(out["y"][3:] == 0.0)
    ref0 = np_expert(x[0].astype(np.float64), W_up.astype(np.float64), W_down.astype(np.float64), 0)
    np.testing.assert_allclose(out["y"][0], ref0, rtol=1e-12, atol=1e-12)


def check_gelu_expert_variant(seed=12):
    """nanoMoE slide 32 variant: GELU is x * Phi(x) with Phi the normal CDF
    (scipy.stats.norm.cdf, a library routine), at printed-in-every-table points
    and on random inputs; the biases are added after each projection."""
    from scipy.stats import norm
    z = np.array([0.0, 1.0, -1.0, 2.5, -3.0, 0.3], dtype=np.float32)
    x = np.ones((1, 1), dtype=np.float32)
    W_up = z.reshape(1, -1, 1)
    W_down = np.ones((1, 1, z.size), dtype=np.float32)
    h, o = oracle.expert_ffn_ex(x, W_up, W_down, 0, 0, act=oracle.ACT_GELU)
    ref = z.astype(np.float64) * norm.cdf(z.astype(np.float64))
    np.testing.assert_allclose(h, ref, rtol=1e-13, atol=1e-15)
    assert h[0] == 0.0 and abs(h[1] - 0.8413447460685429) < 1e-14 and abs(h[2] + 0.15865525393145707) < 1e-14
    rng = np.random.default_rng(seed)
    E, d, d_ff = 2, 5, 7
    x = rng.standard_normal((3, d)).astype(np.float32)
    W_up = rng.standard_normal((E, d_ff, d)).astype(np.float32)
    W_down = rng.standard_normal((E, d, d_ff)).astype(np.float32)
    b_up = rng.standard_normal((E, d_ff)).astype(np.float32)
    b_down = rng.standard_normal((E, d)).astype(np.float32)
    x64, u64, w64 = (a.astype(np.float64) for a in (x, W_up, W_down))
    for act in (oracle.ACT_RELU, oracle.ACT_GELU):
        for t in range(3):
            for e in range(E):
                h, o = oracle.expert_ffn_ex(x, W_up, W_down, t, e, act=act, b_up=b_up, b_down=b_down)
                zz = u64[e] @ x64[t] + b_up[e].astype(np.float64)
                hh = np.maximum(zz, 0) if act == oracle.ACT_RELU else zz * norm.cdf(zz)
                np.testing.assert_allclose(h, hh, rtol=1e-12, atol=1e-12)
                np.testing.assert_allclose(o, w64[e] @ hh + b_down[e].astype(np.float64), rtol=1e-12, atol=1e-12)
    # the plain layer is the variant with ReLU and no biases
    h0, o0 = oracle.expert_ffn(x, W_up, W_down, 1, 1)
    h1, o1 = oracle.expert_ffn_ex(x, W_up, W_down, 1, 1, act=oracle.ACT_RELU)
    assert np.array_equal(h0, h1) and np.array_equal(o0, o1)


def check_gelu_bias_layer(seed=13):
    """E = 1, k = 1 with GELU and biases is the dense nanoMoE MLP."""
    from scipy.stats import norm
    rng = np.random.default_rng(seed)
    N, d, d_ff = 6, 4, 10
    x = rng.standard_normal((N, d)).astype(np.float32)
    W_g = rng.standard_normal((1, d)).astype(np.float32)
    W_up = rng.standard_normal((1, d_ff, d)).astype(np.float32)
    W_down = rng.standard_normal((1, d, d_ff)).astype(np.float32)
    b_up = rng.standard_normal((1, d_ff)).astype(np.float32)
    b_down = rng.standard_normal((1, d)).astype(np.float32)
    out = oracle.forward(x, W_g, None, None, 0.0, 1, 1.0, W_up, W_down, act=oracle.ACT_GELU,
                         b_up=b_up, b_down=b_down)
    z = x.astype(np.float64) @ W_up[0].T.astype(np.float64) + b_up[0].astype(np.float64)
    ref = (z * norm.cdf(z)) @ W_down[0].T.astype(np.float64) + b_down[0].astype(np.float64)
    np.testing.assert_allclose(out["y"], ref, rtol=1e-12, atol=1e-12)


def check_load_stats_m2():
    """Slide 14's used_capacity on the capacity example (slides 15-23): used =
    1, 1, 1 at capacity 1; the load before the cut is one more than each
    expert's last queue place in the uncut ranking (slides 18-19); the gate
    mass is the sum of slide 24's picked probabilities per expert."""
    m2 = load_m2()
    topk = np.array(m2["topk"], dtype=np.int32)
    gates = np.array(m2["gates"], dtype=np.float32)
    load, used, imp = oracle.load_stats(topk, m2["E"], m2["C"], gates)
    assert used.tolist() == m2["used"], used.tolist()
    rank = np.array(m2["rank_nocap"])
    expect_load = [int(rank[topk == e].max()) + 1 for e in range(m2["E"])]
    assert load.tolist() == expect_load, (load.tolist(), expect_load)
    g64 = np.array(m2["gates"], dtype=np.float32).astype(np.float64)
    for e in range(m2["E"]):
        mass = float(g64[topk == e].sum())
        assert abs(imp[e] - mass) <= (topk == e).sum() * 2.0 ** -33, (e, imp[e], mass)


def check_load_stats_random(seed=14):
    """On random routings: load is numpy's bincount of the choices; used is
    the slot pass's per-expert count and min(load, C); the gate mass is within
    one 2^-33 rounding per choice of numpy's float64 weighted bincount, and
    exact when every gate is a multiple of 2^-32."""
    rng = np.random.default_rng(seed)
    for N, E, k, cf in ((500, 8, 2, 0.7), (257, 13, 3, 1.0), (64, 64, 6, math.inf)):
        topk = np.stack([rng.permutation(E)[:k] for _ in range(N)]).astype(np.int32)
        gates = rng.random((N, k)).astype(np.float32)
        C = oracle.capacity(N, E, k, cf)
        load, used, imp = oracle.load_stats(topk, E, C, gates)
        assert np.array_equal(load, np.bincount(topk.ravel(), minlength=E))
        _, counts = oracle.assign_slots(topk, E, C)
        assert np.array_equal(used, counts)
        assert np.array_equal(used, np.minimum(load, C))
        ref = np.bincount(topk.ravel(), weights=gates.ravel().astype(np.float64), minlength=E)
        assert np.all(np.abs(imp - ref) <= load * 2.0 ** -33 + 1e-300)
        dyadic = (np.floor(gates.astype(np.float64) * 64.0) / 64.0).astype(np.float32)
        _, _, imp2 = oracle.load_stats(topk, E, C, dyadic)
        ref2 = np.bincount(topk.ravel(), weights=dyadic.ravel().astype(np.float64), minlength=E)
        assert np.array_equal(imp2, ref2)
    # the rounding of each gate to units of 2^-32 is to nearest, ties to even:
    # 0.75 -> 1, 0.5 -> 0, 1.5 -> 2, 2.5 -> 2 units
    u = 2.0 ** -32
    topk = np.zeros((4, 1), dtype=np.int32)
    gates = np.array([[0.75 * u], [0.5 * u], [1.5 * u], [2.5 * u]], dtype=np.float32)
    _, _, imp = oracle.load_stats(topk, 1, 4, gates)
    assert imp[0] == 5 * u, imp[0] / u


def _autograd_grads(x64, Wg64, bg64, Wu64, Wd64, eps64, sigma, s32, topk, slot, dy):
    """torch float64 autograd of L = sum(dy * y) with the routing held fixed;
    the scores take the oracle's fp32 values s32 with an identity gradient."""
    import torch
    T = lambda a: torch.tensor(a, dtype=torch.float64, requires_grad=True)  # noqa: E731
    X, G, B, U, D = T(x64), T(Wg64), T(bg64), T(Wu64), T(Wd64)
    S = X @ G.T + B + sigma * torch.tensor(eps64, dtype=torch.float64)
    S = S + (torch.tensor(s32.astype(np.float64)) - S).detach()
    g = torch.softmax(S.gather(1, torch.tensor(topk, dtype=torch.int64)), dim=1)
    N, k = topk.shape
    rows = []
    for t in range(N):
        acc = torch.zeros(x64.shape[1], dtype=torch.float64)
        for j in range(k):
            if slot[t, j] >= 0:
                e = int(topk[t, j])
                acc = acc + g[t, j] * (D[e] @ torch.relu(U[e] @ X[t]))
        rows.append(acc)
    L = (torch.stack(rows) * torch.tensor(dy)).sum()
    L.backward()
    return dict(dx=X.grad.numpy(), dW_g=G.grad.numpy(), db_g=B.grad.numpy(), dW_up=U.grad.numpy(),
                dW_down=D.grad.numpy())


def check_backward_vs_autograd(seed=15):
    """The backward (STEP 6: the masked softmax stays differentiable; STEP 11:
    g_i E_i(x) carries the gradient to the router) against torch's float64
    autograd of the same forward with the routing fixed: fp32 and bf16
    storage, noise, bias, capacity drops (a dropped choice's score still
    enters the softmax), and k = 1 (the router gets no gradient)."""
    from sparse_mixture_experts_noisy_b200.synth import bf16_bits_to_f32, f32_to_bf16_bits
    rng = np.random.default_rng(seed)
    for N, d, E, d_ff, k, cf, sigma, bf16 in ((7, 5, 4, 6, 2, 0.6, 0.7, False), (9, 8, 6, 5, 3, 0.5, 0.0, True),
                                              (5, 4, 3, 4, 1, 1.0, 0.3, False)):
        x = rng.standard_normal((N, d)).astype(np.float32)
        Wg = rng.standard_normal((E, d)).astype(np.float32)
        bg = rng.standard_normal(E).astype(np.float32)
        Wu = rng.standard_normal((E, d_ff, d)).astype(np.float32)
        Wd = rng.standard_normal((E, d, d_ff)).astype(np.float32)
        eps = rng.standard_normal((N, E)).astype(np.float32)
        if bf16:
            x, Wu, Wd = f32_to_bf16_bits(x), f32_to_bf16_bits(Wu), f32_to_bf16_bits(Wd)
            x64, Wu64, Wd64 = (bf16_bits_to_f32(a).astype(np.float64) for a in (x, Wu, Wd))
        else:
            x64, Wu64, Wd64 = (a.astype(np.float64) for a in (x, Wu, Wd))
        s_raw = oracle.router_logits(x, Wg, bg)
        topk, _, s = oracle.route_from_logits(s_raw, k, eps if sigma else None, sigma, return_scores=True)
        slot, _ = oracle.assign_slots(topk, E, oracle.capacity(N, E, k, cf))
        assert (slot < 0).any() or cf >= 1.0
        dy = rng.standard_normal((N, d))
        got = oracle.backward(x, Wg, Wu, Wd, s, topk, slot, dy)
        ref = _autograd_grads(x64, Wg.astype(np.float64), bg.astype(np.float64), Wu64, Wd64,
                              eps.astype(np.float64), sigma, s, topk, slot, dy)
        for name in ref:
            scale = max(1.0, float(np.max(np.abs(ref[name]))))
            assert np.max(np.abs(got[name] - ref[name])) <= 1e-12 * scale, (name, N, d, E, k)
        if k == 1:
            assert np.all(got["dW_g"] == 0.0) and np.all(got["db_g"] == 0.0)


def _small_routed_case(rng, N, d, E, d_ff, k, cf, sigma, bf16):
    from sparse_mixture_experts_noisy_b200.synth import f32_to_bf16_bits
    x = rng.standard_normal((N, d)).astype(np.float32)
    Wg = rng.standard_normal((E, d)).astype(np.float32)
    bg = rng.standard_normal(E).astype(np.float32)
    Wu = rng.standard_normal((E, d_ff, d)).astype(np.float32)
    Wd = rng.standard_normal((E, d, d_ff)).astype(np.float32)
    eps = rng.standard_normal((N, E)).astype(np.float32)
    if bf16:
        x, Wu, Wd = f32_to_bf16_bits(x), f32_to_bf16_bits(Wu), f32_to_bf16_bits(Wd)
    s_raw = oracle.router_logits(x, Wg, bg)
    topk, _, s = oracle.route_from_logits(s_raw, k, eps if sigma else None, sigma, return_scores=True)
    slot, _ = oracle.assign_slots(topk, E, oracle.capacity(N, E, k, cf))
    dy = rng.standard_normal((N, d))
    return x, Wg, Wu, Wd, s, topk, slot, dy


def _z(x, Wu, topk, slot):
    """z of every kept pair in float64 numpy: [N, k, d_ff] (0 for dropped)."""
    from sparse_mixture_experts_noisy_b200.synth import bf16_bits_to_f32
    f = (lambda a: bf16_bits_to_f32(a).astype(np.float64)) if x.dtype == np.uint16 else (lambda a: a.astype(np.float64))
    x64, Wu64 = f(x), f(Wu)
    N, k = topk.shape
    z = np.zeros((N, k, Wu.shape[1]))
    for t in range(N):
        for j in range(k):
            if slot[t, j] >= 0:
                z[t, j] = Wu64[topk[t, j]] @ x64[t]
    return z, x64


def check_backward_sampled_matches_full(seed=21):
    """The sampled backward gives exactly the full backward's numbers at the
    listed tokens, dW_up rows and dW_down columns, and all of dW_g and db_g,
    with the ReLU decisions taken by the oracle or replayed from a mask."""
    rng = np.random.default_rng(seed)
    for N, d, E, d_ff, k, cf, sigma, bf16 in ((11, 6, 4, 7, 2, 0.6, 0.5, True), (8, 5, 3, 4, 3, 0.7, 0.0, False)):
        x, Wg, Wu, Wd, s, topk, slot, dy = _small_routed_case(rng, N, d, E, d_ff, k, cf, sigma, bf16)
        z, _ = _z(x, Wu, topk, slot)
        for mask in (None, (z > 0.1).astype(np.uint8)):
            full = oracle.backward(x, Wg, Wu, Wd, s, topk, slot, dy, relu_mask=mask)
            tokens = np.array([0, 3, N - 1])
            ef = [(0, 0), (E - 1, d_ff - 1), (1, 2)]
            got = oracle.backward_sampled(x, Wg, Wu, Wd, s, topk, slot, dy, tokens, ef, relu_mask=mask,
                                          nthreads=3)
            assert np.array_equal(got["dx_rows"], full["dx"][tokens])
            assert np.array_equal(got["dW_g"], full["dW_g"]) and np.array_equal(got["db_g"], full["db_g"])
            for q, (e, f) in enumerate(ef):
                assert np.array_equal(got["dW_up_rows"][q], full["dW_up"][e, f, :])
                assert np.array_equal(got["dW_down_cols"][q], full["dW_down"][e, :, f])


def check_backward_relu_mask_replay(seed=23):
    """A replayed ReLU mask equal to the oracle's own decisions changes
    nothing; turning one decision off for a kept pair (t, j) at unit f takes
    exactly dz_f x_t out of dW_up[e][f] and d_o z_f out of dW_down[e][:, f],
    and changes dx only in row t (the decision acts on both h and dz)."""
    rng = np.random.default_rng(seed)
    N, d, E, d_ff, k = 9, 6, 3, 8, 2
    x, Wg, Wu, Wd, s, topk, slot, dy = _small_routed_case(rng, N, d, E, d_ff, k, 1.0, 0.0, False)
    z, x64 = _z(x, Wu, topk, slot)
    own = (z > 0).astype(np.uint8)
    base = oracle.backward(x, Wg, Wu, Wd, s, topk, slot, dy)
    same = oracle.backward(x, Wg, Wu, Wd, s, topk, slot, dy, relu_mask=own)
    for name in base:
        assert np.array_equal(base[name], same[name]), name
    t, j = 2, 0
    assert slot[t, j] >= 0
    f = int(np.argmax(z[t, j]))
    assert z[t, j, f] > 0
    off = own.copy()
    off[t, j, f] = 0
    got = oracle.backward(x, Wg, Wu, Wd, s, topk, slot, dy, relu_mask=off)
    e = int(topk[t, j])
    g = np.exp(s[t, topk[t]].astype(np.float64) - s[t, topk[t, 0]])
    g = g / g.sum()
    d_o = g[j] * dy[t]
    Wd64 = Wd.astype(np.float64)
    dz_f = float(Wd64[e][:, f] @ d_o)
    du = base["dW_up"] - got["dW_up"]
    dd = base["dW_down"] - got["dW_down"]
    mask_up = np.zeros_like(du, dtype=bool)
    mask_up[e, f, :] = True
    mask_dn = np.zeros_like(dd, dtype=bool)
    mask_dn[e, :, f] = True
    assert np.all(du[~mask_up] == 0.0) and np.all(dd[~mask_dn] == 0.0)
    np.testing.assert_allclose(du[e, f, :], dz_f * x64[t], rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(dd[e, :, f], d_o * z[t, j, f], rtol=1e-9, atol=1e-12)
    ddx = base["dx"] - got["dx"]
    assert np.all(ddx[np.arange(N) != t] == 0.0) and np.any(ddx[t] != 0.0)


ALL_CHECKS = [check_m1, check_m2_slots, check_m2_combine, check_topk_bruteforce,
              check_gates_invariants, check_noise, check_capacity, check_slots_bruteforce,
              check_logits_vs_numpy, check_ffn_vs_numpy, check_dense_mixture,
              check_single_expert_mlp, check_all_dropped_is_zero, check_gelu_expert_variant,
              check_gelu_bias_layer, check_load_stats_m2, check_load_stats_random, check_backward_vs_autograd,
              check_backward_sampled_matches_full, check_backward_relu_mask_replay]
