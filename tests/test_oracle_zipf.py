"""The Zipf-skewed prefill workload's router bias (an input recipe, not an
expected value): expert usage skewed like Zipf(1.2) over 8 experts, which is
what the prefill configuration asks of its router.

The bias of the expert of rank r is alpha * log(pmf_r).  alpha is found by
bisection so that the share of the workload's 4096 tokens whose first
choice is expert 0 equals Zipf's top probability, with first choices taken
by the oracle's own router (fp32 logits in its fixed order, bias added last,
ties to the lower index).  The stored synth.ZIPF_BIAS_SCALE must be that
alpha (to its 4 decimals), and give a top-1 share within 0.02 of Zipf.
"""
import numpy as np
import pytest

from any_precision_weight_pw_b200 import synth

T = 4096


@pytest.fixture(scope="module")
def base_logits(oracle):
    wl = synth.WORKLOADS["mixtral_8x7b_prefill"]
    layer = synth.Layer(wl, seed=0)
    x = synth.tokens(wl, T, seed=0)
    # logits without the bias; the oracle adds the bias last, in fp32
    return wl, x, layer, oracle.router_logits(x, layer.router_w, None)


def _top1_share(wl, logits_nb, alpha):
    bias = synth.zipf_bias(wl.n_experts, wl.zipf_s, alpha)
    lg = (logits_nb + bias[None, :]).astype(np.float32)
    return float(np.mean(np.argmax(lg, axis=1) == 0))


def test_zipf_pmf():
    p = synth.zipf_pmf(8, 1.2)
    assert abs(p.sum() - 1.0) < 1e-15
    assert abs(p[0] - 1.0 / sum(r ** -1.2 for r in range(1, 9))) < 1e-15
    assert np.all(np.diff(p) < 0)


def test_bias_addition_matches_oracle(oracle, base_logits):
    """Adding the bias to the oracle's unbiased logits in fp32 is what the
    oracle's router does with the bias."""
    wl, x, layer, lnb = base_logits
    with_bias = oracle.router_logits(x[:64], layer.router_w, layer.router_bias)
    np.testing.assert_array_equal(with_bias, (lnb[:64] + layer.router_bias[None, :]).astype(np.float32))


def test_stored_bias_scale_is_the_bisection(base_logits):
    wl, _, _, lnb = base_logits
    target = synth.zipf_pmf(wl.n_experts, wl.zipf_s)[0]
    lo, hi = 0.0, 4.0
    assert _top1_share(wl, lnb, lo) < target < _top1_share(wl, lnb, hi)
    for _ in range(30):
        mid = 0.5 * (lo + hi)
        if _top1_share(wl, lnb, mid) < target:
            lo = mid
        else:
            hi = mid
    assert abs(synth.ZIPF_BIAS_SCALE - lo) < 2e-3, lo
    share = _top1_share(wl, lnb, synth.ZIPF_BIAS_SCALE)
    assert abs(share - target) <= 0.02, (share, target)
