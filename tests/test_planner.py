"""The library's release planner (pw_plan_release, host code behind the C
ABI) against the oracle's greedy: identical widths, released bytes and
damage on hand-made and random instances, including layer-shaped ones
(Mixtral- and Qwen-shaped blocks with routing mass from the oracle's own
routing of a synthetic batch).  Runs without a GPU: the planner is host
code, so only the library has to load."""
import numpy as np
import pytest

from any_precision_weight_pw_b200 import synth


@pytest.fixture(scope="module")
def pwlib():
    from any_precision_weight_pw_b200 import binding, build
    build.build()
    return binding


def _random_blocks(rng, n):
    blocks = []
    for _ in range(n):
        bits = int(rng.integers(1, 9))
        lo = int(rng.integers(1, bits + 1))
        sens = [0.0] + [float(rng.random() * 2) for _ in range(8)]
        if rng.random() < 0.2:                        # equal ratios: ties by index
            sens = [0.0] + [1.0] * 8
        blocks.append(dict(bits=bits, min_bits=lo, plane_bytes=int(rng.integers(0, 4)) * 4096,
                           rows=int(rng.choice([0, 128, 1408])), mass=float(rng.random()),
                           resid=float(rng.random()) if rng.random() < 0.5 else 0.0, sens=sens))
    return blocks


def test_matches_oracle_greedy_random(pwlib, oracle):
    rng = np.random.default_rng(12)
    for trial in range(200):
        blocks = _random_blocks(rng, int(rng.integers(0, 40)))
        total = sum(b["plane_bytes"] + b["rows"] * (1 << (k - 1)) * 2
                    for b in blocks for k in range(b["min_bits"] + 1, b["bits"] + 1))
        target = int(rng.integers(-5, total + 3))
        got = pwlib.plan_release(blocks, target)
        want = oracle.plan_greedy(blocks, target)
        assert got == want, trial


def test_hand_instance_and_gap(pwlib, oracle):
    sens0 = [0.0] * 9
    sens0[4], sens0[3] = 2.0, 8.0
    sens1 = [0.0] * 9
    sens1[3], sens1[2] = 1.0, 4.0
    blocks = [dict(bits=4, min_bits=2, plane_bytes=1000, rows=10, mass=0.5, resid=0.0, sens=sens0),
              dict(bits=3, min_bits=1, plane_bytes=2000, rows=10, mass=1.0, resid=1.0, sens=sens1)]
    got = pwlib.plan_release(blocks, 2000)
    assert got == {"bits": [3, 2], "released": 3240, "damage": 3.0, "reached": True}
    assert oracle.plan_exact(blocks, 2000)["damage"] == 2.0    # the greedy gap


def test_rejects_bad_blocks(pwlib):
    bad = dict(bits=3, min_bits=4, plane_bytes=1, rows=1, mass=1.0, resid=0.0, sens=[0.0] * 9)
    with pytest.raises(pwlib.PwError):
        pwlib.plan_release([bad], 10)


@pytest.mark.parametrize("name", ["mixtral_8x7b", "qwen15_moe_a27b"])
def test_layer_shaped_plan(pwlib, oracle, name):
    """A layer's blocks with routing mass from the oracle's routing of one
    synthetic batch, synthetic sensitivities growing as the width falls,
    and a target of a quarter of the active plane bytes."""
    wl = synth.WORKLOADS[name]
    layer = synth.Layer(wl, seed=0)
    x = synth.tokens(wl, 32, seed=0)
    idx, w = oracle.topk_softmax(oracle.router_logits(x, layer.router_w, None), wl.top_k,
                                 bool(wl.renorm_topk))
    _, mass = oracle.routing_stats(idx, w, wl.n_experts)
    rng = np.random.default_rng(3)
    blocks = []
    for blk in range(wl.n_blocks):
        rows, cols = layer.shape(blk)
        e = blk // 3
        m = float(mass[e]) if e < wl.n_experts else 32.0
        base = float(rng.random() + 0.5)
        sens = [0.0] + [base * 2.0 ** (8 - b) for b in range(1, 9)]
        pb = pwlib.plane_bytes(rows, cols)
        blocks.append(dict(bits=layer.bits[blk], min_bits=2, plane_bytes=pb, rows=rows, mass=m,
                           resid=0.0, sens=sens))
    target = sum(b["bits"] * b["plane_bytes"] for b in blocks) // 4
    got = pwlib.plan_release(blocks, target)
    assert got == oracle.plan_greedy(blocks, target)
    assert got["reached"] and got["released"] >= target
    # unused experts (mass 0) are drained first: zero damage per byte
    unused = [i for i in range(wl.n_experts) if mass[i] == 0.0]
    if unused:
        assert all(got["bits"][3 * e + p] < layer.bits[3 * e + p] or layer.bits[3 * e + p] == 2
                   for e in unused[:1] for p in range(3))
