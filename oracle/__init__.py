"""CPU oracle for the PagedWeight fused mixed-precision MoE layer.

TEST INFRASTRUCTURE ONLY: imported by tests/, by the smoke check and by the
benchmark's CPU-baseline leg, never by the product library.  It wraps the plain
C++ reference in ``pw_oracle.cpp`` (built into ``libpw_oracle.so`` next to this
file) with numpy-friendly functions.  It shares no code with the CUDA path.

Seeded inputs come from ``any_precision_weight_pw_b200.synth`` (random numbers
only, none of the method's arithmetic); expected values come from here.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pw_oracle.cpp")
_LIB = os.path.join(_HERE, "libpw_oracle.so")


def build(force: bool = False) -> str:
    """Compile the oracle with g++ (no fused multiply-add contraction beyond
    the explicit fmaf calls, so the router order is the one written)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp.%d" % os.getpid()
        subprocess.check_call([
            "g++", "-O2", "-std=c++17", "-fPIC", "-shared", "-pthread",
            "-ffp-contract=off", "-fno-fast-math", _SRC, "-o", tmp])
        os.replace(tmp, _LIB)
    return _LIB


class _Block(C.Structure):
    _fields_ = [("planes", C.c_void_p), ("lut", C.c_void_p),
                ("rows", C.c_int32), ("cols", C.c_int32), ("bits", C.c_int32)]


class _Layer(C.Structure):
    _fields_ = [("hidden", C.c_int32), ("ffn", C.c_int32), ("n_experts", C.c_int32),
                ("top_k", C.c_int32), ("shared_ffn", C.c_int32), ("n_max", C.c_int32),
                ("renorm_topk", C.c_int32), ("blocks", C.POINTER(_Block))]


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = C.CDLL(build())
        P = C.c_void_p
        i = C.c_int
        _lib.pwo_pack_planes.argtypes = [P, i, i, i, P]
        _lib.pwo_unpack_codes.argtypes = [P, i, i, i, i, P]
        _lib.pwo_linear.argtypes = [P, P, i, i, i, P, P, i]
        _lib.pwo_router_logits.argtypes = [P, i, i, P, P, i, P]
        _lib.pwo_topk_softmax.argtypes = [P, i, i, i, i, P, P]
        _lib.pwo_expert_ffn.argtypes = [C.POINTER(_Layer), i, P, P, P, i]
        _lib.pwo_moe_forward.argtypes = [C.POINTER(_Layer), P, i, P, P, P, P, P, i]
        _lib.pwo_routing_stats.argtypes = [P, P, i, i, i, P, P]
        _lib.pwo_plan_greedy.argtypes = [P, i, C.c_int64, P, P, P]
        _lib.pwo_plan_exact.argtypes = [P, i, C.c_int64, P, P, P]
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data


def _check(rc, what):
    if rc != 0:
        raise ValueError("oracle %s rejected its arguments" % what)


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)))


# ---- the bit-plane view ----------------------------------------------------

def pack_planes(codes: np.ndarray, n_max: int) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    rows, cols = codes.shape
    words = (cols + 31) // 32
    out = np.zeros((n_max, rows, words), dtype=np.uint32)
    _check(lib().pwo_pack_planes(_ptr(codes), rows, cols, n_max, _ptr(out)), "pack")
    return out


def unpack_codes(planes: np.ndarray, cols: int, b: int) -> np.ndarray:
    planes = np.ascontiguousarray(planes, dtype=np.uint32)
    n_max, rows, _ = planes.shape
    out = np.zeros((rows, cols), dtype=np.uint8)
    _check(lib().pwo_unpack_codes(_ptr(planes), rows, cols, n_max, b, _ptr(out)), "unpack")
    return out


def linear(planes: np.ndarray, lut: np.ndarray, cols: int, b: int, x: np.ndarray,
           threads: int = 1) -> np.ndarray:
    """y = W_b x for one block; x is [cols] or [T][cols] (rows of tokens)."""
    planes = np.ascontiguousarray(planes, dtype=np.uint32)
    lut = np.ascontiguousarray(lut, dtype=np.uint16)
    rows = planes.shape[1]
    assert lut.shape == (rows, 1 << b)
    x = np.asarray(x, dtype=np.float64)
    xs = x.reshape(-1, cols)
    ys = np.zeros((xs.shape[0], rows), dtype=np.float64)
    for t in range(xs.shape[0]):
        xt = np.ascontiguousarray(xs[t])
        yt = np.zeros(rows, dtype=np.float64)
        _check(lib().pwo_linear(_ptr(planes), _ptr(lut), rows, cols, b, _ptr(xt), _ptr(yt),
                                threads), "linear")
        ys[t] = yt
    return ys.reshape(x.shape[:-1] + (rows,))


def router_logits(x_bf16: np.ndarray, Wr: np.ndarray, bias=None) -> np.ndarray:
    x_bf16 = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    Wr = np.ascontiguousarray(Wr, dtype=np.float32)
    T, H = x_bf16.shape
    E = Wr.shape[0]
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
    out = np.zeros((T, E), dtype=np.float32)
    _check(lib().pwo_router_logits(_ptr(x_bf16), T, H, _ptr(Wr), _ptr(b), E, _ptr(out)),
           "router")
    return out


def topk_softmax(logits: np.ndarray, k: int, renorm: bool):
    logits = np.ascontiguousarray(logits, dtype=np.float32)
    T, E = logits.shape
    idx = np.zeros((T, k), dtype=np.int32)
    w = np.zeros((T, k), dtype=np.float64)
    _check(lib().pwo_topk_softmax(_ptr(logits), T, E, k, int(renorm), _ptr(idx), _ptr(w)),
           "topk")
    return idx, w


def routing_stats(idx: np.ndarray, w: np.ndarray, n_experts: int, counts=None, mass=None):
    """Per-expert assignment counts and routing-weight sums of a batch,
    added to (counts, mass) when given (accumulation over forwards)."""
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    w = np.ascontiguousarray(w, dtype=np.float64)
    T, k = idx.shape
    counts = np.zeros(n_experts, np.uint64) if counts is None else counts
    mass = np.zeros(n_experts, np.float64) if mass is None else mass
    assert counts.dtype == np.uint64 and mass.dtype == np.float64
    _check(lib().pwo_routing_stats(_ptr(idx), _ptr(w), T, k, n_experts, _ptr(counts),
                                   _ptr(mass)), "routing_stats")
    return counts, mass


class PlanBlock(C.Structure):
    """One block as the planner sees it (see pwo_plan_greedy)."""
    _fields_ = [("bits", C.c_int32), ("min_bits", C.c_int32), ("plane_bytes", C.c_int64),
                ("rows", C.c_int32), ("mass", C.c_double), ("resid", C.c_double),
                ("sens", C.c_double * 9)]


def _plan_array(blocks):
    arr = (PlanBlock * len(blocks))()
    for j, b in enumerate(blocks):
        arr[j].bits, arr[j].min_bits = int(b["bits"]), int(b["min_bits"])
        arr[j].plane_bytes, arr[j].rows = int(b["plane_bytes"]), int(b["rows"])
        arr[j].mass, arr[j].resid = float(b["mass"]), float(b.get("resid", 0.0))
        for k in range(9):
            arr[j].sens[k] = float(b["sens"][k]) if k < len(b["sens"]) else 0.0
    return arr


def _plan(fn, blocks, target):
    arr = _plan_array(blocks)
    n = len(blocks)
    bits = (C.c_int32 * max(n, 1))()
    rel = C.c_int64()
    dmg = C.c_double()
    rc = fn(arr, n, int(target), bits, C.byref(rel), C.byref(dmg))
    if rc == 1:
        raise ValueError("oracle planner rejected its arguments")
    return {"bits": list(bits)[:n], "released": rel.value, "damage": dmg.value,
            "reached": rc == 0}


def plan_greedy(blocks, target):
    """Greedy least-damage-per-byte release plan (dicts with bits, min_bits,
    plane_bytes, rows, mass, resid, sens[0..8])."""
    return _plan(lib().pwo_plan_greedy, blocks, target)


def plan_exact(blocks, target):
    """The brute-force optimum of the same problem (tiny instances)."""
    return _plan(lib().pwo_plan_exact, blocks, target)


class Layer:
    """Keeps the numpy buffers of one layer alive for the C structs."""

    def __init__(self, hidden, ffn, n_experts, top_k, shared_ffn, n_max, renorm_topk,
                 blocks):
        # blocks: list of (planes [n_max][rows][words] uint32, lut [rows][2^b] uint16,
        #                  rows, cols, bits)
        self._keep = []
        self.block_list = []
        arr = (_Block * len(blocks))()
        for j, (pl, lt, rows, cols, bits) in enumerate(blocks):
            pl = np.ascontiguousarray(pl, dtype=np.uint32)
            lt = np.ascontiguousarray(lt, dtype=np.uint16)
            assert lt.shape == (rows, 1 << bits), (lt.shape, rows, bits)
            assert pl.shape[1] == rows and pl.shape[2] == (cols + 31) // 32
            assert bits <= pl.shape[0] <= 8
            self._keep += [pl, lt]
            self.block_list.append((pl, lt, rows, cols, bits))
            arr[j] = _Block(pl.ctypes.data, lt.ctypes.data, rows, cols, bits)
        self._blocks = arr
        self.c = _Layer(hidden, ffn, n_experts, top_k, shared_ffn, n_max, renorm_topk,
                        C.cast(arr, C.POINTER(_Block)))
        self.hidden, self.n_experts, self.top_k = hidden, n_experts, top_k
        self.ffn, self.shared_ffn = ffn, shared_ffn

    def expert_ffn(self, e, x, threads=1):
        x = np.ascontiguousarray(x, dtype=np.float64)
        y = np.zeros(self.hidden, dtype=np.float64)
        F = self.shared_ffn if e == self.n_experts else self.ffn
        h = np.zeros(F, dtype=np.float64)
        _check(lib().pwo_expert_ffn(C.byref(self.c), e, _ptr(x), _ptr(y), _ptr(h), threads),
               "expert")
        return y, h

    def forward(self, x_bf16, Wr, bias=None, threads=1):
        x_bf16 = np.ascontiguousarray(x_bf16, dtype=np.uint16)
        T = x_bf16.shape[0]
        Wr = np.ascontiguousarray(Wr, dtype=np.float32)
        b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
        out = np.zeros((T, self.hidden), dtype=np.float64)
        idx = np.zeros((T, self.top_k), dtype=np.int32)
        w = np.zeros((T, self.top_k), dtype=np.float64)
        _check(lib().pwo_moe_forward(C.byref(self.c), _ptr(x_bf16), T, _ptr(Wr), _ptr(b),
                                     _ptr(out), _ptr(idx), _ptr(w), threads), "forward")
        return out, idx, w
