"""Pins for the oracle's planner: the greedy least-damage-per-released-byte
selection of weight quantisation actions (legiblepapers summary, "Summary &
Methodology Analysis" and FAQ Q8) and the brute-force optimum it is measured
against.  The pages give no damage formula; the reading (damage = offline
sensitivity of the step x routing mass x (1 + prompt residual), bytes = the
plane page plus the LUT half that the step releases) is stated in
oracle/pw_oracle.cpp.
"""
import numpy as np
import pytest


def _blk(bits, min_bits, plane_bytes, rows, mass, resid, sens):
    s = [0.0] * 9
    for b, v in sens.items():
        s[b] = v
    return dict(bits=bits, min_bits=min_bits, plane_bytes=plane_bytes, rows=rows, mass=mass,
                resid=resid, sens=s)


def _hand_instance():
    # block 0: steps 4->3 (1000 + 10*8*2 = 1160 bytes, damage 2*0.5 = 1) and
    #          3->2 (1000 + 10*4*2 = 1080 bytes, damage 8*0.5 = 4)
    # block 1: steps 3->2 (2000 + 10*4*2 = 2080 bytes, damage 1*1*(1+1) = 2)
    #          and 2->1 (2000 + 10*2*2 = 2040 bytes, damage 4*2 = 8)
    return [_blk(4, 2, 1000, 10, 0.5, 0.0, {4: 2.0, 3: 8.0}),
            _blk(3, 1, 2000, 10, 1.0, 1.0, {3: 1.0, 2: 4.0})]


def test_hand_instance(oracle):
    blocks = _hand_instance()
    # target 1000: the cheapest step per byte (block 0, 1/1160) suffices
    g = oracle.plan_greedy(blocks, 1000)
    assert g == {"bits": [3, 3], "released": 1160, "damage": 1.0, "reached": True}
    assert oracle.plan_exact(blocks, 1000) == g
    # target 2000: greedy takes block 0 (1/1160) then block 1 (2/2080):
    # 3240 bytes for damage 3; the optimum is block 1's step alone (2080
    # bytes, damage 2) -- the greedy gap
    g = oracle.plan_greedy(blocks, 2000)
    assert g == {"bits": [3, 2], "released": 3240, "damage": 3.0, "reached": True}
    e = oracle.plan_exact(blocks, 2000)
    assert e == {"bits": [4, 2], "released": 2080, "damage": 2.0, "reached": True}
    # nothing to do, and an unreachable target (everything at its floor)
    assert oracle.plan_greedy(blocks, 0)["bits"] == [4, 3]
    g = oracle.plan_greedy(blocks, 10 ** 9)
    assert g["bits"] == [2, 1] and not g["reached"]
    assert g["released"] == 1160 + 1080 + 2080 + 2040
    assert not oracle.plan_exact(blocks, 10 ** 9)["reached"]


def _convex_instance(rng, n):
    """Equal step bytes everywhere (no LUT rows, one plane size) and damage
    non-decreasing as a block goes lower: the cheapest steps overall always
    form a prefix of each block's steps, so greedy is optimal for targets
    that are whole multiples of the step size."""
    blocks = []
    for _ in range(n):
        bits = int(rng.integers(2, 6))
        lo = int(rng.integers(1, bits))
        inc = np.sort(rng.random(bits - lo))          # damage of steps bits, bits-1, ...
        sens = {bits - j: float(inc[j]) for j in range(bits - lo)}
        blocks.append(_blk(bits, lo, 4096, 0, float(rng.random() + 0.1), 0.0, sens))
    return blocks


def test_greedy_is_optimal_where_the_exchange_argument_holds(oracle):
    rng = np.random.default_rng(5)
    for _ in range(40):
        blocks = _convex_instance(rng, int(rng.integers(1, 6)))
        steps = sum(b["bits"] - b["min_bits"] for b in blocks)
        m = int(rng.integers(0, steps + 1))
        g = oracle.plan_greedy(blocks, 4096 * m)
        e = oracle.plan_exact(blocks, 4096 * m)
        assert g["reached"] and e["reached"]
        assert g["released"] == 4096 * m
        assert g["damage"] == pytest.approx(e["damage"], rel=1e-12, abs=1e-15)


def test_greedy_never_beats_the_optimum(oracle):
    rng = np.random.default_rng(6)
    for _ in range(60):
        n = int(rng.integers(1, 5))
        blocks = []
        for _ in range(n):
            bits = int(rng.integers(2, 7))
            lo = int(rng.integers(1, bits + 1))
            sens = {b: float(rng.random() * 3) for b in range(lo + 1, bits + 1)}
            blocks.append(_blk(bits, lo, int(rng.integers(1, 5)) * 1024, int(rng.integers(0, 64)),
                               float(rng.random()), float(rng.random()), sens))
        total = sum(b["plane_bytes"] + b["rows"] * (1 << (k - 1)) * 2
                    for b in blocks for k in range(b["min_bits"] + 1, b["bits"] + 1))
        target = int(rng.integers(0, total + 2))
        g = oracle.plan_greedy(blocks, target)
        e = oracle.plan_exact(blocks, target)
        assert g["reached"] == e["reached"] == (target <= total)
        if e["reached"]:
            assert g["released"] >= target and e["released"] >= target
            assert g["damage"] >= e["damage"] - 1e-12
