"""Helpers shared by the tests: oracle layers from synthetic layers, and the
output tolerance.

Tolerance (the reading of "max relative error 2e-3, bf16 out, fp32
accumulate"): for every output element,
    |y_gpu - y_ref| <= ulp_bf16(max(|y_ref|, |y_gpu|)) / 2 + 2e-3 * max|y_ref|,
where y_ref is the oracle's float64 result.  The first term is the rounding
of a correctly rounded bf16 output (the output format's own error); the
second is the 2e-3 budget for the path's arithmetic, taken relative to the
largest output because a per-element relative error is ill-conditioned at
outputs near zero.  output_errors also reports that arithmetic part on its
own (arith_excess) and how often the output differs from the correctly
rounded oracle value (rne_mismatch).
"""
import os

import numpy as np

REL_TOL = 2e-3


def bf16_half_ulp(v):
    a = np.maximum(np.abs(np.asarray(v, dtype=np.float64)), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(a)) - 8)


def bf16_round(v):
    """Round float64 values to the nearest bf16 (ties to even), as float64
    (normal range; the outputs here are far from under- and overflow)."""
    v = np.asarray(v, dtype=np.float64)
    a = np.maximum(np.abs(v), 2.0 ** -126)
    ulp = 2.0 ** (np.floor(np.log2(a)) - 7)
    return np.round(v / ulp) * ulp      # v / ulp is exact; np.round ties to even


def output_errors(y_gpu, y_ref):
    """norm_max_rel: max |y_gpu - y_ref| / max |y_ref|, the bf16 output
    rounding included (alone it can reach 2^-8 of scale when the largest
    output sits just above a power of two).  arith_excess: the largest error
    beyond the output's own half-ulp, / max |y_ref| -- a bound on the path's
    arithmetic error before the final rounding.  rne_mismatch: the fraction
    of outputs that differ from the correctly rounded oracle value."""
    y_gpu = np.asarray(y_gpu, dtype=np.float64)
    y_ref = np.asarray(y_ref, dtype=np.float64)
    scale = float(np.max(np.abs(y_ref))) if y_ref.size else 0.0
    err = np.abs(y_gpu - y_ref)
    half = bf16_half_ulp(np.maximum(np.abs(y_ref), np.abs(y_gpu)))
    bound = half + REL_TOL * scale
    return {
        "max_abs": float(err.max()) if err.size else 0.0,
        "norm_max_rel": float(err.max() / scale) if scale > 0 else 0.0,
        "arith_excess": float(max(0.0, (err - half).max()) / scale) if scale > 0 else 0.0,
        "rne_mismatch": float(np.mean(y_gpu != bf16_round(y_ref))) if y_ref.size else 0.0,
        "rel_l2": float(np.linalg.norm(err) / max(np.linalg.norm(y_ref), 1e-300)),
        "excess": float((err - bound).max()) if err.size else -1.0,
    }


# (test id, errors) of every comparison made in this session, for the
# summary the test session prints at the end (tests/conftest.py)
RECORDED = []


def assert_output_close(y_gpu, y_ref):
    e = output_errors(y_gpu, y_ref)
    test = os.environ.get("PYTEST_CURRENT_TEST", "").split(" ")[0]
    RECORDED.append((test, e))
    assert e["excess"] <= 0.0, e
    return e


def oracle_layer(oracle, layer, bits=None):
    wl = layer.wl
    bits = layer.bits if bits is None else bits
    blocks = []
    for blk in range(wl.n_blocks):
        rows, cols = layer.shape(blk)
        blocks.append((layer.planes(blk), layer.lut(blk, bits[blk]), rows, cols, bits[blk]))
    return oracle.Layer(wl.hidden, wl.ffn, wl.n_experts, wl.top_k, wl.shared_ffn, wl.n_max,
                        wl.renorm_topk, blocks)
