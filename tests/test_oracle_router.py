"""Pins for the oracle's routing: router logits, top-k order and weights.

Routing is fused into the MoE kernel (legiblepapers summary, FAQ Q5); the
pages fix no formula, so the library reads it as: logits = x Wr^T (+ bias) in
fp32 in one fixed order, experts ranked by logit with ties to the lower
index, softmax probabilities over all experts, optional renormalisation over
the k selected.
"""
import itertools
import math

import numpy as np
import pytest

from any_precision_weight_pw_b200 import synth


def test_logits_exact_on_small_integers(oracle):
    rng = np.random.default_rng(0)
    T, H, E = 5, 96, 7
    x = rng.integers(-4, 5, size=(T, H)).astype(np.float32)
    Wr = rng.integers(-4, 5, size=(E, H)).astype(np.float32)
    bias = rng.integers(-3, 4, size=E).astype(np.float32)
    got = oracle.router_logits(synth.to_bf16_bits(x), Wr, bias)
    want = (x.astype(np.int64) @ Wr.astype(np.int64).T + bias.astype(np.int64)).astype(np.float32)
    np.testing.assert_array_equal(got, want)


def test_logits_follow_the_lane_butterfly_order(oracle):
    """x = 1 at columns 0, 8, 24; Wr = 2^24 at 0 and 1 at 8, 24.  Lane sums are
    s0 = 2^24, s8 = s24 = 1.  The butterfly adds (s0 + s16) + (s8 + s24) =
    2^24 + 2 exactly, while a left-to-right sum would lose both ones."""
    H = 32
    x = np.zeros((1, H), np.float32)
    x[0, [0, 8, 24]] = 1.0
    Wr = np.zeros((1, H), np.float32)
    Wr[0, 0] = 2.0 ** 24
    Wr[0, [8, 24]] = 1.0
    got = oracle.router_logits(synth.to_bf16_bits(x), Wr)
    assert got[0, 0] == np.float32(2.0 ** 24 + 2)
    # bias is added after the butterfly, in fp32
    got = oracle.router_logits(synth.to_bf16_bits(x), Wr, np.array([1.0], np.float32))
    assert got[0, 0] == np.float32(2.0 ** 24 + 2) + np.float32(1.0)
    # within a lane the terms fuse in ascending i: s0 = fma(1, 1, fma(1, 2^24, 0))
    H = 64
    x = np.zeros((1, H), np.float32)
    x[0, [0, 32]] = 1.0
    Wr = np.zeros((1, H), np.float32)
    Wr[0, 0], Wr[0, 32] = 2.0 ** 24, 1.0
    assert oracle.router_logits(synth.to_bf16_bits(x), Wr)[0, 0] == np.float32(2.0 ** 24)


def test_logits_within_fp32_bound_on_random_inputs(oracle):
    rng = np.random.default_rng(1)
    T, H, E = 4, 2048, 60
    x = synth.to_bf16_bits(rng.normal(size=(T, H)).astype(np.float32))
    Wr = rng.normal(0, 0.02, size=(E, H)).astype(np.float32)
    got = oracle.router_logits(x, Wr).astype(np.float64)
    xf = synth.bf16_bits_to_float(x).astype(np.float64)
    exact = xf @ Wr.astype(np.float64).T
    bound = (H / 32 + 6) * 2.0 ** -24 * (np.abs(xf) @ np.abs(Wr.astype(np.float64)).T)
    assert np.all(np.abs(got - exact) <= bound)


def _brute_topk(l, k):
    ranked = sorted(range(len(l)), key=lambda e: (-float(l[e]), e))
    return ranked[:k]


def test_topk_brute_force_with_ties(oracle):
    rng = np.random.default_rng(2)
    for E in range(1, 9):
        for k in range(1, min(E, 4) + 1):
            logits = rng.integers(-2, 3, size=(64, E)).astype(np.float32)  # many ties
            idx, _ = oracle.topk_softmax(logits, k, renorm=True)
            for t in range(64):
                assert list(idx[t]) == _brute_topk(logits[t], k)
                sel = set(idx[t])
                for a in idx[t]:
                    for b in range(E):
                        if b not in sel:
                            assert logits[t, a] >= logits[t, b]
                            if logits[t, a] == logits[t, b]:
                                assert a < b


def test_topk_exhaustive_tiny(oracle):
    """Every logit vector over {0,1,2}^4 with k = 2."""
    vals = np.array(list(itertools.product([0.0, 1.0, 2.0], repeat=4)), np.float32)
    idx, _ = oracle.topk_softmax(vals, 2, renorm=False)
    for t in range(len(vals)):
        assert list(idx[t]) == _brute_topk(vals[t], 2)


def test_routing_weights_closed_forms(oracle):
    # E = 2, k = 1, no renorm: the weight is the logistic function of the gap
    for a, b in [(0.0, 0.0), (1.0, 0.0), (-3.5, 2.25), (10.0, -10.0)]:
        idx, w = oracle.topk_softmax(np.array([[a, b]], np.float32), 1, renorm=False)
        hi = max(a, b)
        lo = min(a, b)
        assert w[0, 0] == pytest.approx(1.0 / (1.0 + math.exp(lo - hi)), rel=1e-14)
        assert idx[0, 0] == (0 if a >= b else 1)
    # k = E with renorm: the full softmax, summing to one; equal logits -> 1/E
    rng = np.random.default_rng(4)
    l = rng.normal(size=(3, 6)).astype(np.float32)
    idx, w = oracle.topk_softmax(l, 6, renorm=True)
    np.testing.assert_allclose(w.sum(axis=1), 1.0, rtol=1e-14)
    _, w_eq = oracle.topk_softmax(np.zeros((1, 5), np.float32), 3, renorm=False)
    np.testing.assert_allclose(w_eq, 0.2, rtol=1e-15)
    _, w_eq = oracle.topk_softmax(np.zeros((1, 5), np.float32), 3, renorm=True)
    np.testing.assert_allclose(w_eq, 1.0 / 3.0, rtol=1e-15)
    # k = 1 with renorm: weight exactly one
    _, w1 = oracle.topk_softmax(l, 1, renorm=True)
    assert np.all(w1 == 1.0)
    # shifting every logit by a constant changes nothing
    _, wa = oracle.topk_softmax(l, 2, renorm=False)
    _, wb = oracle.topk_softmax(l + np.float32(4.0), 2, renorm=False)
    np.testing.assert_allclose(wa, wb, rtol=1e-6)
    # renorm divides by the selected mass
    _, wr = oracle.topk_softmax(l, 2, renorm=True)
    np.testing.assert_allclose(wr, wa / wa.sum(axis=1, keepdims=True), rtol=1e-14)


# ---- routing statistics (the planner's online routing mass) ---------------

def test_routing_stats_hand_example(oracle):
    """The hand example's routing: t0 -> (0, 1) with weights (s, 1-s), t1 ->
    (1, 0) with (s, 1-s), t2 -> (0, 1) with (1/2, 1/2), s the logistic of 1.
    Each expert is used three times with weight mass s + (1-s) + 1/2 = 3/2;
    a second call adds the same again."""
    s = 1.0 / (1.0 + math.exp(-1.0))
    idx = np.array([[0, 1], [1, 0], [0, 1]], np.int32)
    w = np.array([[s, 1 - s], [s, 1 - s], [0.5, 0.5]])
    counts, mass = oracle.routing_stats(idx, w, 2)
    assert counts.tolist() == [3, 3]
    np.testing.assert_allclose(mass, [1.5, 1.5], rtol=1e-15)
    counts, mass = oracle.routing_stats(idx, w, 2, counts, mass)
    assert counts.tolist() == [6, 6]
    np.testing.assert_allclose(mass, [3.0, 3.0], rtol=1e-15)


def test_routing_stats_totals_and_unused_experts(oracle):
    """Totals: T*k assignments; with renormalised weights the mass sums to T.
    An expert that is never selected keeps zero count and mass."""
    rng = np.random.default_rng(9)
    l = rng.normal(size=(50, 8)).astype(np.float32)
    l[:, 5] = -100.0                      # expert 5 never wins a slot
    idx, w = oracle.topk_softmax(l, 3, renorm=True)
    counts, mass = oracle.routing_stats(idx, w, 8)
    assert int(counts.sum()) == 150 and counts[5] == 0 and mass[5] == 0.0
    assert mass.sum() == pytest.approx(50.0, rel=1e-13)


def test_routing_stats_k_equals_e_is_the_softmax_column_sum(oracle):
    """k = E without renormalisation: every expert is in every token's list
    with its full softmax probability, so mass[e] = sum_t softmax(l_t)[e],
    written here directly with numpy in float64."""
    rng = np.random.default_rng(10)
    l = rng.normal(size=(40, 6)).astype(np.float32)
    idx, w = oracle.topk_softmax(l, 6, renorm=False)
    counts, mass = oracle.routing_stats(idx, w, 6)
    z = np.exp(l.astype(np.float64) - l.max(axis=1, keepdims=True))
    p = z / z.sum(axis=1, keepdims=True)
    assert counts.tolist() == [40] * 6
    np.testing.assert_allclose(mass, p.sum(axis=0), rtol=1e-13)
