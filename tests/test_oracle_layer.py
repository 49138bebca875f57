"""Pins for the oracle's whole layer: SwiGLU experts, weighted combine and the
shared expert.

Fused expert activation and output accumulation: legiblepapers summary, FAQ
Q5.  SwiGLU experts, top-k routing and the ungated shared expert follow the
Qwen1.5-MoE / Mixtral layer shapes the pages evaluate (FAQ Q6).
"""
import math
from fractions import Fraction as Fr

import numpy as np
import pytest

from any_precision_weight_pw_b200 import synth


def _f16_bits(vals):
    return np.asarray(vals, dtype=np.float16).view(np.uint16)


def _hand_layer(oracle):
    """Two experts, H = 32, F = 4, k = 2, renorm, n_max = 3; expert 0 at 3 bits,
    expert 1 at 2 bits (reads code >> 1).  Codes: gate (o+i+e) mod 8,
    up (3o+i) mod 8, down (o+2f) mod 8.  LUT_3 gate/up: (2v-7)/8 + o/16,
    LUT_3 down: (2v-7)/8, LUT_2 (all): (2v-3)/4.  All exact in fp16."""
    H, F = 32, 4
    blocks = []
    for e, b in ((0, 3), (1, 2)):
        for proj in range(3):
            rows, cols = (F, H) if proj < 2 else (H, F)
            if proj == 0:
                codes = [[(o + i + e) % 8 for i in range(cols)] for o in range(rows)]
            elif proj == 1:
                codes = [[(3 * o + i) % 8 for i in range(cols)] for o in range(rows)]
            else:
                codes = [[(o + 2 * f) % 8 for f in range(cols)] for o in range(rows)]
            planes = oracle.pack_planes(np.array(codes, np.uint8), 3)
            if b == 3:
                lut = [[(2 * v - 7) / 8 + (o / 16 if proj < 2 else 0.0) for v in range(8)]
                       for o in range(rows)]
            else:
                lut = [[(2 * v - 3) / 4 for v in range(4)] for _ in range(rows)]
            blocks.append((planes, _f16_bits(lut), rows, cols, b))
    layer = oracle.Layer(H, F, 2, 2, 0, 3, 1, blocks)
    Wr = np.zeros((2, H), np.float32)
    Wr[0, 0] = Wr[1, 1] = 0.5
    x = np.zeros((3, H), np.float32)
    x[0, 0], x[0, 2] = 2, 1
    x[1, 1], x[1, 2] = 2, 1
    x[2, :3] = 1
    return layer, Wr, synth.to_bf16_bits(x)


def test_hand_example_routing_and_outputs(oracle):
    layer, Wr, x = _hand_layer(oracle)
    out, idx, w = layer.forward(x, Wr)
    # logits (1, 0), (0, 1), (0.5, 0.5): the tie goes to expert 0
    assert idx.tolist() == [[0, 1], [1, 0], [0, 1]]
    s = 1.0 / (1.0 + math.exp(-1.0))
    np.testing.assert_allclose(w, [[s, 1 - s], [s, 1 - s], [0.5, 0.5]], rtol=1e-15)
    # hand-derived in float64 (7 significant digits)
    want = [[-0.9035184, -0.9142537, 0.3580196, 0.3472844],
            [-0.6708742, -0.6615392, 0.5634112, 0.5727461],
            [-0.9166429, -0.9241294, 0.4995289, 0.4920425]]
    np.testing.assert_allclose(out[:, :4], want, atol=6e-8)


def test_hand_example_intermediates(oracle):
    """Token 0 through expert 0: g and u are the exact rationals below, so the
    activation h = silu(g) u follows in closed form."""
    layer, _, x = _hand_layer(oracle)
    xf = synth.bf16_bits_to_float(x[0]).astype(np.float64)
    y, h = layer.expert_ffn(0, xf)
    g = [Fr(-17, 8), Fr(-19, 16), Fr(-1, 4), Fr(11, 16)]
    u = [Fr(-17, 8), Fr(5, 16), Fr(3, 4), Fr(-13, 16)]
    want_h = [float(a) / (1.0 + math.exp(-float(a))) * float(c) for a, c in zip(g, u)]
    np.testing.assert_allclose(h, want_h, rtol=1e-15)
    # down row o has codes (o + 2f) mod 8 with LUT (2v-7)/8
    want_y = [sum((2 * ((o + 2 * f) % 8) - 7) / 8 * want_h[f] for f in range(4))
              for o in range(32)]
    np.testing.assert_allclose(y, want_y, rtol=1e-13, atol=1e-15)


def _random_blocks(oracle, rng, H, F, E, S, bits_pool, n_max=8):
    blocks = []
    for e in range(E + (1 if S else 0)):
        Fe = S if e == E else F
        for proj in range(3):
            rows, cols = (Fe, H) if proj < 2 else (H, Fe)
            b = int(rng.choice(bits_pool))
            planes = synth.random_planes(rng, n_max, rows, cols)
            blocks.append((planes, synth.random_lut(rng, rows, b), rows, cols, b))
    return blocks


def test_shared_expert_is_added_with_weight_one(oracle):
    rng = np.random.default_rng(5)
    H, F, E, k = 64, 48, 4, 2
    blocks = _random_blocks(oracle, rng, H, F, E, 0, (3, 5))
    # the shared expert re-uses expert 2's blocks
    with_shared = oracle.Layer(H, F, E, k, F, 8, 1, blocks + blocks[6:9])
    without = oracle.Layer(H, F, E, k, 0, 8, 1, blocks)
    Wr = rng.normal(0, 0.05, size=(E, H)).astype(np.float32)
    x = synth.to_bf16_bits(rng.normal(size=(3, H)).astype(np.float32))
    a, ia, wa = with_shared.forward(x, Wr)
    b, ib, wb = without.forward(x, Wr)
    np.testing.assert_array_equal(ia, ib)
    for t in range(3):
        y2, _ = without.expert_ffn(2, synth.bf16_bits_to_float(x[t]).astype(np.float64))
        np.testing.assert_allclose(a[t] - b[t], y2, rtol=1e-12, atol=1e-14)


def test_combine_is_the_weighted_sum_of_experts(oracle):
    rng = np.random.default_rng(6)
    H, F, E, k = 32, 40, 5, 3
    blocks = _random_blocks(oracle, rng, H, F, E, 0, (2, 4, 6))
    for renorm in (0, 1):
        layer = oracle.Layer(H, F, E, k, 0, 8, renorm, blocks)
        Wr = rng.normal(0, 0.1, size=(E, H)).astype(np.float32)
        x = synth.to_bf16_bits(rng.normal(size=(4, H)).astype(np.float32))
        out, idx, w = layer.forward(x, Wr)
        if renorm:
            np.testing.assert_allclose(w.sum(axis=1), 1.0, rtol=1e-14)
        for t in range(4):
            xt = synth.bf16_bits_to_float(x[t]).astype(np.float64)
            want = sum(w[t, j] * layer.expert_ffn(int(idx[t, j]), xt)[0] for j in range(k))
            np.testing.assert_allclose(out[t], want, rtol=1e-12, atol=1e-15)


def test_swiglu_limits(oracle):
    """silu(0) = 0 zeroes the expert; a large positive gate passes u through
    (silu(g) = g to double precision for g >= 40)."""
    H, F = 32, 3
    ones = np.ones((F, H), np.uint8)

    def layer_with(gate_val, up_val, down_val):
        blocks = []
        for proj, val in enumerate((gate_val, up_val, down_val)):
            rows, cols = (F, H) if proj < 2 else (H, F)
            planes = oracle.pack_planes(np.zeros((rows, cols), np.uint8), 1)
            lut = _f16_bits([[val, 0.0]] * rows)  # every code is 0 -> LUT[o][0]
            blocks.append((planes, lut, rows, cols, 1))
        return oracle.Layer(H, F, 1, 1, 0, 1, 1, blocks)

    x = np.full(H, 1.0)
    y, h = layer_with(0.0, 0.5, 0.25).expert_ffn(0, x)
    assert np.all(h == 0.0) and np.all(y == 0.0)
    # g = 32 * 1.5 = 48 per row, u = 32 * 0.5 = 16, h = 48 * 16, y = 3 * 0.25 * h
    y, h = layer_with(1.5, 0.5, 0.25).expert_ffn(0, x)
    np.testing.assert_allclose(h, 48.0 * 16.0, rtol=1e-15)
    np.testing.assert_allclose(y, 3 * 0.25 * 48.0 * 16.0, rtol=1e-15)
    del ones


def test_dense_restatement_matches(oracle):
    """A second plain restatement: dense float64 torch-free numpy recompute of
    one expert from the unpacked codes and gathered LUT values."""
    rng = np.random.default_rng(8)
    H, F = 64, 96
    blocks = _random_blocks(oracle, rng, H, F, 1, 0, (3, 4, 6, 8))
    layer = oracle.Layer(H, F, 1, 1, 0, 8, 1, blocks)
    Ws = []
    for planes, lut, rows, cols, b in blocks:
        codes = oracle.unpack_codes(planes, cols, b).astype(np.int64)
        Ws.append(np.take_along_axis(lut.view(np.float16).astype(np.float64), codes, axis=1))
    x = rng.normal(size=H)
    g, u = Ws[0] @ x, Ws[1] @ x
    want = Ws[2] @ (g / (1 + np.exp(-g)) * u)
    y, _ = layer.expert_ffn(0, x)
    np.testing.assert_allclose(y, want, rtol=1e-10, atol=1e-14)


def test_bf16_round_helper():
    """The tests' bf16 rounding of oracle outputs: exact values stay, halfway
    cases go to the even significand, and it agrees with a float32 round
    trip through the bf16 bit pattern on random values."""
    import pw_testutil as tu
    assert tu.bf16_round(np.array([1.0, -3.0, 0.5]))[:].tolist() == [1.0, -3.0, 0.5]
    # 1 + 2^-8 is halfway between 1 and 1 + 2^-7: ties to even -> 1
    assert tu.bf16_round(np.array([1.0 + 2.0 ** -8]))[0] == 1.0
    # 1 + 3 * 2^-8 is halfway between 1 + 2^-7 and 1 + 2^-6: -> 1 + 2^-6
    assert tu.bf16_round(np.array([1.0 + 3 * 2.0 ** -8]))[0] == 1.0 + 2.0 ** -6
    rng = np.random.default_rng(1)
    v = rng.normal(size=1000).astype(np.float32)
    want = synth.bf16_bits_to_float(synth.to_bf16_bits(v)).astype(np.float64)
    np.testing.assert_array_equal(tu.bf16_round(v.astype(np.float64)), want)
