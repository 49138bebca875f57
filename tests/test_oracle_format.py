"""Pins for the oracle's bit-plane view and dequantised linear.

The bit-plane / LUT format is the Any-Precision view that the PagedWeight
summaries name (arxivlens abstract; legiblepapers FAQ Q5: the fused kernel
reads bit-planes and lookup tables directly, one bitwidth per linear-block).
"""
import json
import os

import numpy as np
import pytest

from any_precision_weight_pw_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_pack_matches_hand_derived_words(oracle):
    g = json.load(open(os.path.join(GOLDEN, "bitplane_words.json")))
    rows, cols, n_max = g["rows"], g["cols"], g["n_max"]
    codes = np.array([[(i + o) % 8 for i in range(cols)] for o in range(rows)], np.uint8)
    want = np.array([[[int(w, 16) for w in row] for row in plane] for plane in g["planes"]],
                    dtype=np.uint32)
    got = oracle.pack_planes(codes, n_max)
    assert got.shape == want.shape
    np.testing.assert_array_equal(got, want)
    np.testing.assert_array_equal(oracle.unpack_codes(want, cols, n_max), codes)


@pytest.mark.parametrize("n_max", [3, 5, 8])
def test_b_bit_view_is_top_bits(oracle, n_max):
    rng = np.random.default_rng(n_max)
    for rows, cols in [(3, 32), (5, 77), (2, 200)]:
        planes = synth.random_planes(rng, n_max, rows, cols)
        full = oracle.unpack_codes(planes, cols, n_max).astype(np.int64)
        assert full.max() < (1 << n_max)
        for b in range(1, n_max + 1):
            view = oracle.unpack_codes(planes, cols, b).astype(np.int64)
            np.testing.assert_array_equal(view, full >> (n_max - b))
            # the b-bit view depends on planes 0..b-1 only
            scrambled = planes.copy()
            scrambled[b:] = rng.integers(0, 2**32, size=scrambled[b:].shape, dtype=np.uint32)
            if cols % 32:
                scrambled[:, :, -1] &= np.uint32((1 << (cols % 32)) - 1)
            np.testing.assert_array_equal(oracle.unpack_codes(scrambled, cols, b), view)


def test_pack_unpack_round_trip(oracle):
    rng = np.random.default_rng(7)
    for n_max in (1, 4, 8):
        for rows, cols in [(1, 1), (4, 31), (3, 64), (2, 100)]:
            planes = synth.random_planes(rng, n_max, rows, cols)
            codes = oracle.unpack_codes(planes, cols, n_max)
            np.testing.assert_array_equal(oracle.pack_planes(codes, n_max), planes)
            codes2 = rng.integers(0, 1 << n_max, size=(rows, cols), dtype=np.uint8)
            np.testing.assert_array_equal(
                oracle.unpack_codes(oracle.pack_planes(codes2, n_max), cols, n_max), codes2)


def _identity_lut(rows, b):
    # LUT_b[o][v] = v, exact in fp16 for v < 2048
    return np.tile(np.arange(1 << b, dtype=np.float16), (rows, 1)).view(np.uint16)


@pytest.mark.parametrize("b", list(range(1, 9)))
def test_identity_lut_linear_is_integer_matmul(oracle, b):
    """With LUT_b[o][v] = v the dequantised linear is the integer matmul of the
    b-bit codes (exact: integer x, all partial sums < 2^53)."""
    rng = np.random.default_rng(100 + b)
    rows, cols = 9, 70
    codes = rng.integers(0, 256, size=(rows, cols), dtype=np.uint8)
    planes = oracle.pack_planes(codes, 8)
    x = rng.integers(-8, 9, size=(3, cols)).astype(np.float64)
    y = oracle.linear(planes, _identity_lut(rows, b), cols, b, x)
    want = (x.astype(np.int64) @ (codes.astype(np.int64) >> (8 - b)).T).astype(np.float64)
    np.testing.assert_array_equal(y, want)


def test_linear_gathers_row_lut(oracle):
    """A non-uniform LUT: one-hot inputs return the gathered table entry, and a
    general input equals a dense matmul with W[o][i] = LUT[o][code[o][i]]."""
    rng = np.random.default_rng(3)
    rows, cols, b = 6, 45, 4
    codes = rng.integers(0, 256, size=(rows, cols), dtype=np.uint8)
    planes = oracle.pack_planes(codes, 8)
    lut = synth.random_lut(rng, rows, b)
    lutf = lut.view(np.float16).astype(np.float64)
    c4 = codes >> 4
    for i in (0, 31, 32, 44):
        x = np.zeros(cols)
        x[i] = 1.0
        y = oracle.linear(planes, lut, cols, b, x)
        np.testing.assert_array_equal(y, lutf[np.arange(rows), c4[:, i]])
    W = np.take_along_axis(lutf, c4.astype(np.int64), axis=1)
    x = rng.normal(size=cols)
    np.testing.assert_allclose(oracle.linear(planes, lut, cols, b, x), W @ x, rtol=1e-12,
                               atol=1e-15)
