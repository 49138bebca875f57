"""Seeded synthetic workloads shaped like the layers the PagedWeight pages
evaluate (Qwen1.5-MoE-A2.7B and Mixtral-8x7B, legiblepapers summary, FAQ Q6).

This module draws random numbers and nothing else: it holds none of the
layer's arithmetic, so the tests, the benchmark and the CPU oracle can all
take their inputs from it.  No model weights or datasets are used; every
tensor is drawn from the distributions stated per workload below.

Distributions (every workload):
  * activations x ~ N(0, 1), rounded to bf16 (round to nearest even);
  * router weights ~ N(0, 0.02) fp32, router bias zero unless stated;
  * codes uniform over [0, 2^n_max): every bit-plane word is 32 uniform bits
    (pad bits beyond ``cols`` cleared), which is the same distribution;
  * LUTs: per output row and per bitwidth b, 2^b draws of N(0, 0.02) rounded
    to fp16 and sorted ascending;
  * bitwidth per linear-block drawn uniformly from the workload's set.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional, Sequence, Tuple

import numpy as np

N_PROJ = 3  # gate, up, down
PROJ_NAMES = ("gate", "up", "down")


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    hidden: int
    ffn: int
    n_experts: int
    top_k: int
    shared_ffn: int
    n_max: int
    renorm_topk: int
    bit_choices: Tuple[int, ...]
    tokens: Tuple[int, ...]
    index: int  # mixed into every seed so workloads never share streams
    zipf_s: float = 0.0          # > 0: router bias skews expert usage (prefill)
    wide_experts: Tuple[int, ...] = ()  # experts forced to wide_bits (prefill)
    wide_bits: int = 8

    @property
    def n_blocks(self) -> int:
        return N_PROJ * (self.n_experts + (1 if self.shared_ffn > 0 else 0))


WORKLOADS: Dict[str, Workload] = {
    # Tiny MoE FFN layer: small enough for the oracle in a fraction of a second.
    "tiny_h256_f512_e8k2": Workload(
        "tiny_h256_f512_e8k2", 256, 512, 8, 2, 0, 8, 1, (3, 4), (16,), 0),
    # Qwen1.5-MoE-A2.7B-shaped layer: 60 routed experts (FFN 1408), top-4, one
    # ungated shared expert of FFN 5632; decode batches 1, 8, 32.
    "qwen15_moe_a27b": Workload(
        "qwen15_moe_a27b", 2048, 1408, 60, 4, 5632, 8, 0, (3, 4, 5, 6, 8), (1, 8, 32), 1),
    # Mixtral-8x7B-shaped layer: 8 experts (FFN 14336), top-2; decode 1, 16, 64.
    "mixtral_8x7b": Workload(
        "mixtral_8x7b", 4096, 14336, 8, 2, 0, 8, 1, (3, 4, 6), (1, 16, 64), 2),
    # Mixtral-8x7B-shaped layer at prefill scale: 4096 tokens, expert usage
    # skewed like Zipf(1.2) through the router bias, 4-bit everywhere except
    # experts 0 and 1 at 8-bit.
    "mixtral_8x7b_prefill": Workload(
        "mixtral_8x7b_prefill", 4096, 14336, 8, 2, 0, 8, 1, (4,), (4096,), 3,
        zipf_s=1.2, wide_experts=(0, 1), wide_bits=8),
    # Bitwidth-switch stress on the Qwen-shaped layer, decode batch 32.
    "qwen15_moe_a27b_switch": Workload(
        "qwen15_moe_a27b_switch", 2048, 1408, 60, 4, 5632, 8, 0, (3, 4, 5, 6, 8), (32,), 4),
}

# Router-bias scale alpha of the Zipf-skewed prefill workload: the bias of the
# expert of rank r is alpha * log(zipf_pmf[r]).  Chosen so that the share of
# the workload's 4096 tokens whose FIRST choice is expert 0 equals Zipf(1.2)'s
# top probability over 8 experts (0.4286) within 0.02; the value is the
# bisection of tests/test_oracle_zipf.py, which re-derives it with the
# oracle's router and checks it.
ZIPF_BIAS_SCALE = 0.8483


def zipf_pmf(n: int, s: float) -> np.ndarray:
    """Zipf(s) probabilities of ranks 1..n."""
    p = np.arange(1, n + 1, dtype=np.float64) ** (-s)
    return p / p.sum()


def _rng(wl: Workload, seed: int, *tags: int) -> np.random.Generator:
    return np.random.default_rng([int(seed), wl.index, *[int(t) for t in tags]])


def zipf_bias(n: int, s: float, alpha: float) -> np.ndarray:
    """Router bias alpha * log(Zipf(s) pmf) over expert rank (fp32)."""
    return (alpha * np.log(zipf_pmf(n, s))).astype(np.float32)


def block_shape(wl: Workload, block_id: int) -> Tuple[int, int]:
    """(rows, cols) of a linear-block; y = W x with W rows x cols."""
    expert, proj = divmod(block_id, N_PROJ)
    F = wl.shared_ffn if expert == wl.n_experts else wl.ffn
    return (F, wl.hidden) if proj < 2 else (wl.hidden, F)


def random_planes(rng: np.random.Generator, n_max: int, rows: int, cols: int) -> np.ndarray:
    """[n_max][rows][ceil(cols/32)] uint32 of uniform bits, pad bits cleared."""
    words = (cols + 31) // 32
    n = n_max * rows * words
    raw = rng.bit_generator.random_raw((n + 1) // 2).view(np.uint32)[:n]
    planes = raw.reshape(n_max, rows, words).copy()
    if cols % 32:
        planes[:, :, -1] &= np.uint32((1 << (cols % 32)) - 1)
    return planes


def random_lut(rng: np.random.Generator, rows: int, b: int) -> np.ndarray:
    """[rows][2^b] fp16 bit patterns, N(0, 0.02) sorted ascending per row."""
    v = rng.normal(0.0, 0.02, size=(rows, 1 << b)).astype(np.float16)
    v.sort(axis=1)
    return v.view(np.uint16)


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns, round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def bf16_bits_to_float(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


class Layer:
    """One synthetic MoE layer: planes per block (all n_max planes), the
    initial bitwidth per block, LUTs per (block, b) drawn on first use, and
    the router."""

    def __init__(self, wl: Workload, seed: int = 0, bits: Optional[Sequence[int]] = None):
        self.wl, self.seed = wl, seed
        rng = _rng(wl, seed, 1)
        if bits is None:
            bits = rng.choice(np.asarray(wl.bit_choices), size=wl.n_blocks)
            for e in wl.wide_experts:
                bits[N_PROJ * e:N_PROJ * (e + 1)] = wl.wide_bits
        self.bits = [int(b) for b in bits]
        assert len(self.bits) == wl.n_blocks
        self._planes: Dict[int, np.ndarray] = {}
        self._luts: Dict[Tuple[int, int], np.ndarray] = {}
        r = _rng(wl, seed, 2)
        self.router_w = r.normal(0.0, 0.02, size=(wl.n_experts, wl.hidden)).astype(np.float32)
        self.router_bias = None
        if wl.zipf_s > 0:
            self.router_bias = zipf_bias(wl.n_experts, wl.zipf_s, ZIPF_BIAS_SCALE)

    def shape(self, block_id: int) -> Tuple[int, int]:
        return block_shape(self.wl, block_id)

    def planes(self, block_id: int) -> np.ndarray:
        if block_id not in self._planes:
            rows, cols = self.shape(block_id)
            self._planes[block_id] = random_planes(
                _rng(self.wl, self.seed, 3, block_id), self.wl.n_max, rows, cols)
        return self._planes[block_id]

    def lut(self, block_id: int, b: int) -> np.ndarray:
        key = (block_id, b)
        if key not in self._luts:
            rows, _ = self.shape(block_id)
            self._luts[key] = random_lut(_rng(self.wl, self.seed, 4, block_id, b), rows, b)
        return self._luts[key]

    def drop(self, block_id: int) -> None:
        """Forget the host copies of one block (memory for large layers)."""
        self._planes.pop(block_id, None)
        for key in [k for k in self._luts if k[0] == block_id]:
            del self._luts[key]


def tokens(wl: Workload, T: int, seed: int = 0, batch: int = 0) -> np.ndarray:
    """[T][hidden] bf16 bit patterns of N(0, 1) activations."""
    rng = _rng(wl, seed, 5, T, batch)
    return to_bf16_bits(rng.normal(0.0, 1.0, size=(T, wl.hidden)).astype(np.float32))


def switch_schedule(wl: Workload, bits: Sequence[int], n_forwards: int, every: int = 10,
                    fraction: float = 0.25, lo: int = 3, hi: int = 8, seed: int = 0):
    """Bitwidth changes for the switch-stress workload.

    Before forward f (f = every, 2*every, ...) a fraction of the blocks, chosen
    without replacement, change bitwidth: direction up or down with equal
    probability (forced up at ``lo`` and down at ``hi``), then a new width
    uniform over the allowed side of [lo, hi].  Returns {f: [(block, new_b)]}.
    """
    rng = _rng(wl, seed, 6)
    cur = [int(b) for b in bits]
    out = {}
    nb = len(cur)
    m = int(round(fraction * nb))
    for f in range(every, n_forwards, every):
        chosen = rng.choice(nb, size=m, replace=False)
        changes = []
        for blk in sorted(int(c) for c in chosen):
            b = cur[blk]
            up = b <= lo or (b < hi and rng.random() < 0.5)
            nb_ = int(rng.integers(b + 1, hi + 1)) if up else int(rng.integers(lo, b))
            changes.append((blk, nb_))
            cur[blk] = nb_
        out[f] = changes
    return out
