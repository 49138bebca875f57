#!/usr/bin/env python
"""Benchmark of the fused mixed-bitwidth MoE layer forward on B200.

Metric: MoE-layer decode tokens/s and achieved HBM GB/s (fraction of the
measured HBM copy bandwidth), on synthetic layers shaped like the models the
PagedWeight pages evaluate (legiblepapers summary, FAQ Q6).  Headline
workload: the Mixtral-8x7B-shaped layer (hidden 4096, 8 experts of FFN 14336,
top-2, bitwidths drawn from {3, 4, 6}) at a decode batch of 16 tokens.  One
step = one forward (router, top-k, bucketing, gate/up, SwiGLU, down,
weighted combine) over a fresh token batch already resident in HBM.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun (N > 1) every rank runs its own replica of the layer on its
own GPU (the layer does not shard: replicas only); value = all tokens / the
slowest rank's time.  --impl reference times the CPU oracle (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import tempfile
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE-layer decode tokens/s and achieved HBM GB/s (% of B200 roofline), 1 GPU"
HEADLINE = ("mixtral_8x7b", 16)
SWEEP = [("mixtral_8x7b", 1), ("mixtral_8x7b", 64), ("qwen15_moe_a27b", 1),
         ("qwen15_moe_a27b", 8), ("qwen15_moe_a27b", 32)]
N_BATCHES = 8  # distinct token batches cycled through the timed steps
FALLBACK_TFLOPS = 1590.0
FALLBACK_HBM_GBS = 6650.0


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


# ---------------------------------------------------------------- ranks
def max_over_ranks(x, world, device=None):
    """The largest of every rank's value (all ranks get it; timings are taken
    as the slowest rank's).  world == 1 returns x unchanged."""
    if world <= 1:
        return float(x)
    import torch
    t = torch.tensor([float(x)], device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(world, steps, T, ms):
    """Tokens per second of the whole job: every rank runs `steps` forwards of
    T tokens (its own replica) in the slowest rank's `ms`."""
    return world * steps * T / (ms / 1e3)


# ---------------------------------------------------------------- bytes
def block_bytes(layer, blk, bits=None):
    rows, cols = layer.shape(blk)
    b = layer.bits[blk] if bits is None else bits[blk]
    return b * rows * ((cols + 31) // 32) * 4 + rows * (1 << b) * 2


def algorithmic_bytes(layer, idx, bits=None):
    """Bytes the method must move for one forward: the active planes and LUTs
    of every expert with at least one routed token (plus the shared expert),
    the router weights, the activations in and the output out."""
    wl = layer.wl
    T = idx.shape[0]
    active = sorted(set(int(e) for e in np.unique(idx)))
    if wl.shared_ffn > 0:
        active.append(wl.n_experts)
    gu = sum(block_bytes(layer, 3 * e + p, bits) for e in active for p in (0, 1))
    down = sum(block_bytes(layer, 3 * e + 2, bits) for e in active)
    router = wl.n_experts * wl.hidden * 4
    act = 2 * T * wl.hidden * 2
    return {"gu": gu + T * wl.hidden * 2, "down": down, "total": gu + down + router + act}


def kernel_source_hash():
    """sha256 of the tensor-core kernel's code (tc.cu, dequant.cuh, pages.h,
    tc.h) with line comments and blank lines removed, so that only a change
    of the code itself retires the recorded DRAM traffic."""
    import hashlib
    import re
    code = []
    for f in ("tc.cu", "dequant.cuh", "pages.h", "tc.h"):
        for line in open(os.path.join(ROOT, "any_precision_weight_pw_b200", "csrc", f)):
            line = re.sub(r"//.*", "", line).rstrip()
            if line:
                code.append(line)
    return hashlib.sha256("\n".join(code).encode()).hexdigest()


# ---------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        # raw samples go to PW_BENCH_CLOCKS_DIR (default: the temp directory)
        self.path = os.path.join(os.environ.get("PW_BENCH_CLOCKS_DIR", tempfile.gettempdir()),
                                 "bench_clocks_%d.csv" % os.getpid())

    def __enter__(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.f.close()

    def summary(self, t_begin=None, t_end=None):
        """Samples taken between t_begin and t_end (host wall clock)."""
        import datetime
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                if t_begin is not None and not (t_begin - 0.15 <= ts <= t_end + 0.15):
                    continue
                rows.append((float(parts[1]), float(parts[2]), parts[5], parts[6], parts[7],
                             parts[8]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [r[0] for r in rows]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[2 + i] == "Active"})
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": max(r[1] for r in rows),
                "samples": len(rows), "reasons": reasons}


# ---------------------------------------------------------------- our arm
def page_move_stress(dev, n_forwards=1000, warmup=20):
    """Bitwidth-switch stress on the Qwen-shaped layer at 32 decode tokens:
    before every 10th forward a quarter of the linear-blocks change bitwidth
    (up or down within 3..8); each change is a page move on a side stream
    (plane pages of an upgrade and the new LUT, from pinned host copies).
    Reports steady-state tokens/s and the per-forward latency distribution
    from CUDA events on the forward stream, next to the same layer without
    switches.  No L2 flush: steady serving."""
    import torch
    from any_precision_weight_pw_b200 import binding, synth
    wl = synth.WORKLOADS["qwen15_moe_a27b_switch"]
    T = wl.tokens[0]
    layer = synth.Layer(wl, seed=0)
    d = binding.upload_synth_layer(layer, max_tokens=T, host_copies=True)
    wr = torch.from_numpy(layer.router_w).to(dev)
    xs = [torch.from_numpy(synth.tokens(wl, T, seed=0, batch=b).view(np.int16)).to(dev)
          for b in range(N_BATCHES)]
    ys = [torch.empty_like(x) for x in xs]
    stream = torch.cuda.current_stream()
    side = torch.cuda.Stream()
    total = warmup + n_forwards
    sched = synth.switch_schedule(wl, layer.bits, total, every=10)
    pb = [binding.plane_bytes(*layer.shape(blk)) for blk in range(wl.n_blocks)]
    # routing of each batch (untimed), for the bytes each forward must move
    routing = []
    for x, y in zip(xs, ys):
        d.forward(x, wr, None, y)
        routing.append(d.routing(T)[0].cpu().numpy())

    def run(with_switches, track=False):
        # track: also read back, after every forward, the widths it used, to
        # count how many forwards each switch takes to apply (an extra host
        # call per forward, so only in an untimed pass)
        bits = list(layer.bits) if with_switches else None
        moved = 0
        lags = []        # forwards from a switch's request until all of it applies
        waiting = []     # (forward of the request, widths after it)
        widths = []      # widths of every forward (tracked pass)
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(total)]
        for f in range(total):
            if with_switches and f in sched:
                for blk, nb in sched[f]:
                    d.set_block_bits(blk, nb, side)
                    rows = layer.shape(blk)[0]
                    if f >= warmup:
                        moved += max(nb - bits[blk], 0) * pb[blk] + rows * (1 << nb) * 2
                    bits[blk] = nb
                if track:
                    waiting.append((f, list(bits)))
            evs[f][0].record(stream)
            d.forward(xs[f % N_BATCHES], wr, None, ys[f % N_BATCHES])
            evs[f][1].record(stream)
            if track:
                used = d.forward_bits()
                widths.append(used)
                while waiting and used == waiting[0][1]:
                    lags.append(f - waiting.pop(0)[0])
        torch.cuda.synchronize()
        d.check_device_error()
        lat = np.array([a.elapsed_time(b) for a, b in evs[warmup:]])
        span = evs[warmup][0].elapsed_time(evs[-1][1])
        return lat, span, moved, lags, widths

    base_lat, base_span, _, _, _ = run(False)
    lat, span, moved, _, _ = run(True)
    # widths back to the starting table, then the untimed pass that counts lags
    for blk in range(wl.n_blocks):
        d.set_block_bits(blk, layer.bits[blk], side)
    for _ in range(10):
        d.forward(xs[0], wr, None, ys[0])
        torch.cuda.synchronize()
    _, _, _, lags, widths = run(True, track=True)
    n_switch = sum(1 for f in sched if f >= warmup)
    # achieved GB/s of both runs: the switches change the widths (and so the
    # bytes) of later forwards; the switch run's widths are those the
    # tracked pass used, forward by forward
    base_bytes = sum(algorithmic_bytes(layer, routing[f % N_BATCHES])["total"]
                     for f in range(warmup, total))
    sw_bytes = sum(algorithmic_bytes(layer, routing[f % N_BATCHES], widths[f])["total"]
                   for f in range(warmup, total))
    out = {"workload": "qwen15_moe_a27b decode T=%d, 25%% of blocks switch every 10 forwards" % T,
           "forwards": n_forwards, "tokens_per_s": round(n_forwards * T / (span / 1e3), 1),
           "ms_per_forward_mean": round(float(lat.mean()), 4),
           "ms_per_forward_p50": round(float(np.percentile(lat, 50)), 4),
           "ms_per_forward_p99": round(float(np.percentile(lat, 99)), 4),
           "ms_per_forward_max": round(float(lat.max()), 4),
           "page_bytes_per_switch": int(moved / max(n_switch, 1)),
           "blocks_per_switch": len(next(iter(sched.values()))),
           "forwards_until_applied": {"mean": round(float(np.mean(lags)), 2) if lags else None,
                                      "max": int(max(lags)) if lags else None,
                                      "max_lag": 8},
           "gbs": round(sw_bytes / (span / 1e3) / 1e9, 1),
           "avg_bits": round(float(np.mean([np.mean(w) for w in widths[warmup:]])), 3),
           "no_switch": {"tokens_per_s": round(n_forwards * T / (base_span / 1e3), 1),
                         "ms_per_forward_p99": round(float(np.percentile(base_lat, 99)), 4),
                         "gbs": round(base_bytes / (base_span / 1e3) / 1e9, 1),
                         "avg_bits": round(float(np.mean(layer.bits)), 3)}}
    d.close()
    return out


def time_flushed(d, xs, ys, wr, bias, flush, n=20, warmup=3):
    """Median ms of single forwards, each after an L2 flush (CUDA events on
    the forward stream)."""
    import torch
    stream = torch.cuda.current_stream()
    times = []
    for i in range(warmup + n):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        d.forward(xs[i % len(xs)], wr, bias, ys[i % len(ys)])
        b.record(stream)
        torch.cuda.synchronize()
        if i >= warmup:
            times.append(a.elapsed_time(b))
    d.check_device_error()
    return float(np.median(times))


def uniform_vs_mixed(dev, hbm_peak):
    """Mixed per-block bitwidths against uniform ones, at kernel level: the
    same layer shape and token batches with every block at one width b (for
    each b of the workload's set), then with the workload's mixed table.
    The pages report at most 4.1% throughput loss of the mixed system
    against uniform quantisation (legiblepapers FAQ Q7; hardware unstated);
    here the comparable figure is the achieved GB/s of the mixed table
    against the uniform widths' (same bytes-per-second machinery, different
    bytes per forward)."""
    import torch
    from any_precision_weight_pw_b200 import binding, synth
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    out = []
    for name, T in (("mixtral_8x7b", 16), ("qwen15_moe_a27b", 32)):
        wl = synth.WORKLOADS[name]
        mixed = synth.Layer(wl, seed=0)
        rows = []
        for tag, bits in [("uniform %d" % b, [b] * wl.n_blocks) for b in wl.bit_choices
                          if b in (3, 4, 6)] + [("mixed", None)]:
            layer = mixed if bits is None else synth.Layer(wl, seed=0, bits=bits)
            d = binding.upload_synth_layer(layer, max_tokens=T)
            wr = torch.from_numpy(layer.router_w).to(dev)
            xs_np = [synth.tokens(wl, T, seed=0, batch=b) for b in range(N_BATCHES)]
            xs = [torch.from_numpy(x.view(np.int16)).to(dev) for x in xs_np]
            ys = [torch.empty_like(x) for x in xs]
            mb = []
            for x, y in zip(xs, ys):
                d.forward(x, wr, None, y)
                idx, _ = d.routing(T)
                mb.append(algorithmic_bytes(layer, idx.cpu().numpy())["total"])
            ms = time_flushed(d, xs, ys, wr, None, flush)
            gbs = float(np.mean(mb)) / (ms / 1e3) / 1e9
            rows.append({"bits": tag, "avg_bits": round(float(np.mean(layer.bits)), 3),
                         "ms": round(ms, 4), "tokens_per_s": round(T / (ms / 1e3), 1),
                         "gbs": round(gbs, 1), "frac_of_measured_hbm": round(gbs / hbm_peak, 4)})
            d.close()
            del xs, ys
        uni = [r["gbs"] for r in rows if r["bits"] != "mixed"]
        mix = [r["gbs"] for r in rows if r["bits"] == "mixed"][0]
        out.append({"workload": "%s decode T=%d" % (name, T), "runs": rows,
                    "mixed_gbs_vs_uniform_mean": round(mix / float(np.mean(uni)), 4)})
    del flush
    return out


def small_batch_paths(dev, hbm_peak):
    """The two decode paths head to head at small batches: the tensor-core
    passes (the default) and the CUDA-core dequant-GEMV passes (opt-in,
    PW_GV_T), same layer and token batches, flushed L2, median of 20."""
    import torch
    from any_precision_weight_pw_b200 import binding, synth
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    out = []
    old = os.environ.get("PW_GV_T")
    os.environ["PW_GV_T"] = "4"
    try:
        for name in ("mixtral_8x7b", "qwen15_moe_a27b"):
            wl = synth.WORKLOADS[name]
            layer = synth.Layer(wl, seed=0)
            d = binding.upload_synth_layer(layer, max_tokens=4)
            wr = torch.from_numpy(layer.router_w).to(dev)
            for T in (1, 2, 4):
                xs = [torch.from_numpy(synth.tokens(wl, T, seed=0, batch=b).view(np.int16)).to(dev)
                      for b in range(N_BATCHES)]
                ys = [torch.empty_like(x) for x in xs]
                mb = []
                for x, y in zip(xs, ys):
                    d.forward(x, wr, None, y)
                    mb.append(algorithmic_bytes(layer, d.routing(T)[0].cpu().numpy())["total"])
                row = {"workload": "%s decode T=%d" % (name, T)}
                for tag, gv in (("tensor_core", "0"), ("cuda_core", "1")):
                    os.environ["PW_GV"] = gv
                    ms = time_flushed(d, xs, ys, wr, None, flush)
                    gbs = float(np.mean(mb)) / (ms / 1e3) / 1e9
                    row[tag] = {"ms": round(ms, 4), "gbs": round(gbs, 1),
                                "frac_of_measured_hbm": round(gbs / hbm_peak, 4)}
                os.environ.pop("PW_GV", None)
                out.append(row)
            d.close()
    finally:
        os.environ.pop("PW_GV", None)
        if old is None:
            os.environ.pop("PW_GV_T", None)
        else:
            os.environ["PW_GV_T"] = old
    del flush
    return out


def decode_only(dev, name, T, n=5):
    """A few forwards of one decode workload (an entry point for ncu
    captures); returns the mean ms of the last n forwards."""
    import torch
    from any_precision_weight_pw_b200 import binding, build, synth
    build.build()
    wl = synth.WORKLOADS[name]
    layer = synth.Layer(wl, seed=0)
    d = binding.upload_synth_layer(layer, max_tokens=max(T, 1))
    wr = torch.from_numpy(layer.router_w).to(dev)
    xs = [torch.from_numpy(synth.tokens(wl, T, seed=0, batch=b).view(np.int16)).to(dev)
          for b in range(4)]
    for i in range(3):
        d.forward(xs[i % 4], wr)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(n):
        d.forward(xs[i % 4], wr)
    e1.record()
    torch.cuda.synchronize()
    d.check_device_error()
    out = {"workload": "%s decode T=%d" % (name, T), "ms_per_forward": e0.elapsed_time(e1) / n,
           "launches_per_forward": d.launches(T)}
    d.close()
    return out


def paging_measure(dev, hbm_peak, T=16, n_fwd=200):
    """Residency paging on the Mixtral-shaped layer (decode batch 16): the
    layer switched to library-owned plane storage (only each block's
    resident planes on the device), then the planner frees 25% and then 50%
    of the resident plane bytes (damage = synthetic offline sensitivity x
    the routing mass the library counted over the warm-up forwards), the
    plan is applied as page moves and the resident planes are packed, and
    each table is reported as resident plane bytes, pool bytes after a
    trim, device free memory, and forward tokens/s (back to back, inputs
    larger than L2)."""
    import torch
    from any_precision_weight_pw_b200 import binding, synth
    wl = synth.WORKLOADS["mixtral_8x7b"]
    layer = synth.Layer(wl, seed=0)
    d = binding.upload_synth_layer(layer, max_tokens=T, host_copies=True)
    d.enable_paging()
    d._keep[0] = None                      # the caller's plane buffers are released
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    wr = torch.from_numpy(layer.router_w).to(dev)
    xs = [torch.from_numpy(synth.tokens(wl, T, seed=0, batch=b).view(np.int16)).to(dev)
          for b in range(N_BATCHES)]
    ys = [torch.empty_like(x) for x in xs]
    side = torch.cuda.Stream()
    rng = np.random.default_rng(0)
    base = rng.random(wl.n_blocks) + 0.5

    def timed():
        for i in range(10):
            d.forward(xs[i % N_BATCHES], wr, None, ys[i % N_BATCHES])
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for i in range(n_fwd):
            d.forward(xs[i % N_BATCHES], wr, None, ys[i % N_BATCHES])
        e1.record()
        torch.cuda.synchronize()
        d.check_device_error()
        return e0.elapsed_time(e1) / n_fwd

    rows_out = []
    d.routing_stats(reset=True)
    ms = timed()
    _, mass = d.routing_stats()
    bits = list(layer.bits)
    resident0 = None
    for frac in (0.0, 0.25, 0.5):
        if frac > 0:
            blocks = []
            for blk in range(wl.n_blocks):
                rows, cols = layer.shape(blk)
                sens = [0.0] + [float(base[blk]) * 2.0 ** (8 - b) for b in range(1, 9)]
                blocks.append(dict(bits=bits[blk], min_bits=2,
                                   plane_bytes=binding.plane_bytes(rows, cols), rows=rows,
                                   mass=float(mass[blk // 3]), resid=0.0, sens=sens))
            plan = binding.plan_release(blocks, int(resident0 * frac) - (resident0 - resident))
            d.set_switch_lag(0)
            for blk, b in enumerate(plan["bits"]):
                d.set_block_bits(blk, b, side)
            bits = plan["bits"]
            d.forward(xs[0], wr, None, ys[0])
            # pack the resident planes so the pool can hand the freed bytes back
            d.compact_pages()
            torch.cuda.synchronize()
            ms = timed()
        resident, reserved = d.resident_bytes(trim=True)
        if resident0 is None:
            resident0 = resident
        free_b, total_b = torch.cuda.mem_get_info(dev)
        rows_out.append({"released_target": frac, "resident_plane_bytes": int(resident),
                         "pool_reserved_bytes": int(reserved), "device_free_bytes": int(free_b),
                         "avg_bits": round(float(np.mean(bits)), 3),
                         "ms_per_forward": round(ms, 4),
                         "tokens_per_s": round(T / (ms / 1e3), 1)})
    d.close()
    return {"workload": "mixtral_8x7b decode T=%d, paged planes, planner releases 25%% / 50%%" % T,
            "steps": rows_out}


def prefill_measure(dev, steps=20, warmup=3):
    """The Mixtral-shaped layer at prefill scale (4096 tokens, Zipf-skewed
    routing): forward time with CUDA events, tokens/s and achieved TFLOP/s of
    the expert contractions (2 x 3 x H x F per routed slot) against the
    measured dense bf16 peak (fp16 runs at the same tensor rate)."""
    import torch
    from any_precision_weight_pw_b200 import binding, synth
    wl = synth.WORKLOADS["mixtral_8x7b_prefill"]
    T = wl.tokens[0]
    layer = synth.Layer(wl, seed=0)
    d = binding.upload_synth_layer(layer, max_tokens=T)
    wr = torch.from_numpy(layer.router_w).to(dev)
    bias = torch.from_numpy(layer.router_bias).to(dev)
    x = torch.from_numpy(synth.tokens(wl, T, seed=0).view(np.int16)).to(dev)
    y = torch.empty_like(x)
    for _ in range(warmup):
        d.forward(x, wr, bias, y)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        d.forward(x, wr, bias, y)
    e1.record()
    torch.cuda.synchronize()
    d.check_device_error()
    ms = e0.elapsed_time(e1) / steps
    idx, _ = d.routing(T)
    counts = np.bincount(idx.cpu().numpy().reshape(-1), minlength=wl.n_experts)
    flops = 2.0 * 3 * wl.hidden * wl.ffn * T * wl.top_k
    pk = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json"))) if os.path.exists(
        os.path.join(ROOT, "MEASURED_PEAKS.json")) else {}
    peak = float(pk.get("bf16_tflops", FALLBACK_TFLOPS))
    d.close()
    return {"workload": "mixtral_8x7b prefill T=%d (Zipf 1.2 usage, experts 0-1 at 8 bits, rest 4)" % T,
            "ms_per_forward": round(ms, 3), "tokens_per_s": round(T / (ms / 1e3), 1),
            "tflops": round(flops / (ms / 1e3) / 1e12, 2), "peak_tflops": peak,
            "frac_of_peak": round(flops / (ms / 1e3) / 1e12 / peak, 4),
            "tokens_per_expert": counts.tolist()}


def run_ours(args, rank, world, local_rank):
    import torch
    from any_precision_weight_pw_b200 import binding, build, synth

    if rank == 0:
        build.build()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    hbm_peak, peak_kind = peaks()

    def prepare_layer(name, seed):
        layer = synth.Layer(synth.WORKLOADS[name], seed=seed)
        d = binding.upload_synth_layer(layer, max_tokens=64)
        wr = torch.from_numpy(layer.router_w).to(dev)
        bias = None if layer.router_bias is None else torch.from_numpy(layer.router_bias).to(dev)
        return layer, d, wr, bias

    def prepare_batches(layer, d, wr, bias, T, seed):
        xs_np = [synth.tokens(layer.wl, T, seed=seed, batch=b) for b in range(N_BATCHES)]
        xs = [torch.from_numpy(x.view(np.int16)).to(dev) for x in xs_np]
        ys = [torch.empty_like(x) for x in xs]
        bts = []  # routing of every batch (untimed) for the byte accounting
        for x, y in zip(xs, ys):
            d.forward(x, wr, bias, y)
            idx, _ = d.routing(T)
            bts.append(algorithmic_bytes(layer, idx.cpu().numpy()))
        torch.cuda.synchronize()
        d.check_device_error()
        return xs, xs_np, ys, bts

    name, T = HEADLINE
    layer, d, wr, bias = prepare_layer(name, seed=rank)
    xs, xs_np, ys, bts = prepare_batches(layer, d, wr, bias, T, seed=rank)
    stream = torch.cuda.current_stream()
    for i in range(args.warmup):
        d.forward(xs[i % N_BATCHES], wr, bias, ys[i % N_BATCHES])
    torch.cuda.synchronize()
    d.profile(True)
    d.profile_read()
    with ClockSampler(local_rank) as clk:
        time.sleep(1.0)  # let nvidia-smi start sampling
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        t_begin = time.time()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(args.steps):
            d.forward(xs[i % N_BATCHES], wr, bias, ys[i % N_BATCHES])
        e1.record(stream)
        torch.cuda.synchronize()
        t_end = time.time()
        if world > 1:
            torch.distributed.barrier()
        ms = e0.elapsed_time(e1)
    y0 = ys[0].view(torch.int16).cpu().numpy().view(np.uint16)  # the output for batch 0
    per_launch, n_fwd = d.profile_read()
    d.profile(False)
    launches_per_forward = d.launches(T)
    d.check_device_error()
    ms_max = max_over_ranks(ms, world, dev)
    steps = args.steps
    bytes_total = sum(bts[i % N_BATCHES]["total"] for i in range(steps))
    bytes_gu = sum(bts[i % N_BATCHES]["gu"] for i in range(steps))
    bytes_down = sum(bts[i % N_BATCHES]["down"] for i in range(steps))
    tok_s = whole_job_rate(world, steps, T, ms_max)
    fwd_gbs = bytes_total / (ms / 1e3) / 1e9
    # dominant kernel: the tensor-core dequant-GEMM.  Launch slots 1 and 2 hold the
    # gather launch and the tensor-core launch(es) (one fused launch at decode),
    # so the duration includes the small gather kernel: achieved is a slight
    # underestimate of the tensor-core kernel alone.
    tc_ms = per_launch[1] + per_launch[2]
    tc_gbs = (bytes_gu + bytes_down) / (tc_ms / 1e3) / 1e9 if tc_ms > 0 else None
    traffic = None
    prof_path = os.path.join(ROOT, "profiles", "traffic_per_forward.json")
    if os.path.exists(prof_path):
        tr = json.load(open(prof_path))
        # counters count only while the kernel source is the one they were taken on
        if tr.get("workload") == "%s T=%d" % HEADLINE and tr.get("source_sha256") == kernel_source_hash():
            traffic = tr.get("dram_bytes_per_forward")

    # end to end: host activations in, host output out, through the C ABI
    xh = [torch.from_numpy(x.view(np.int16)).pin_memory() for x in xs_np]
    yh = torch.empty_like(xh[0]).pin_memory()
    for i in range(min(3, args.warmup)):
        d.forward_host(xh[i % N_BATCHES], wr, bias, yh)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    e2 = torch.cuda.Event(enable_timing=True)
    e3 = torch.cuda.Event(enable_timing=True)
    e2.record(stream)
    for i in range(args.steps):
        d.forward_host(xh[i % N_BATCHES], wr, bias, yh)
    e3.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e2.elapsed_time(e3)
    e2e_wall = time.perf_counter() - t0
    e2e_tok_s = whole_job_rate(world, args.steps, T,
                               max_over_ranks(max(e2e_ms, e2e_wall * 1e3), world, dev))

    # decode sweep (other batch sizes and the Qwen-shaped layer); L2 flushed
    # between timed forwards so small layers are not served from cache
    sweep = []
    page_move = None
    prefill = None
    uniform = None
    paging = None
    small = None
    if rank == 0 and not args.no_sweep:
        flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        cur = (name, layer, d, wr, bias)
        for (wname, wT) in SWEEP:
            if wname != cur[0]:
                cur[2].close()
                cur = (wname,) + prepare_layer(wname, seed=rank)
            _, lay, dd, wr2, b2 = cur
            xs2, _, ys2, bts2 = prepare_batches(lay, dd, wr2, b2, wT, seed=rank)
            med = time_flushed(dd, xs2, ys2, wr2, b2, flush)
            mb = float(np.mean([bb["total"] for bb in bts2]))
            sweep.append({"workload": wname, "tokens": wT, "ms_median": round(med, 4),
                          "tokens_per_s": round(wT / (med / 1e3), 1),
                          "gbs": round(mb / (med / 1e3) / 1e9, 1),
                          "frac_of_measured_hbm": round(mb / (med / 1e3) / 1e9 / hbm_peak, 4),
                          "bytes_alg": int(mb)})
            del xs2, ys2
        cur[2].close()
        del flush
        if not args.quick:
            page_move = page_move_stress(dev)
            prefill = prefill_measure(dev)
            uniform = uniform_vs_mixed(dev, hbm_peak)
            paging = paging_measure(dev, hbm_peak)
            small = small_batch_paths(dev, hbm_peak)
    else:
        d.close()

    cpu, accuracy = None, None
    if rank == 0 and world == 1 and not args.no_cpu:
        cpu, ref = cpu_baseline(layer, xs_np[0], T)
        # the same tokens' GPU outputs against the oracle's (bf16 output
        # rounding included in norm_max_rel; arith_excess is what lies beyond
        # each output's half-ulp)
        sys.path.insert(0, os.path.join(ROOT, "tests"))
        from pw_testutil import output_errors
        yg = (y0[:len(ref)].astype(np.uint32) << 16).view(np.float32)
        e = output_errors(yg, np.asarray(ref))
        accuracy = {"tokens": len(ref), "vs": "CPU oracle (float64)",
                    "norm_max_rel": round(e["norm_max_rel"], 6),
                    "arith_excess": round(e["arith_excess"], 6),
                    "rne_mismatch": round(e["rne_mismatch"], 4), "tolerance_ok": e["excess"] <= 0}
    if rank != 0:
        return None
    wl = layer.wl
    launches = launches_per_forward * args.steps
    out = {
        "metric": METRIC,
        "value": round(tok_s, 1),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_max / args.steps, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f16",
        "data": "synthetic",
        "config": {"workload": "%s decode T=%d" % (name, T), "hidden": wl.hidden, "ffn": wl.ffn,
                   "experts": wl.n_experts, "top_k": wl.top_k,
                   "bits": sorted(set(layer.bits)),
                   "l2": "inputs larger than L2 (active planes %.2f GB per forward, L2 126 MB)"
                         % (bytes_total / steps / 1e9),
                   "batches": N_BATCHES, "parallelism": "replicas" if world > 1 else "1 GPU"},
        "hbm_gbs": round(fwd_gbs, 1),
        "hbm_frac": round(fwd_gbs / hbm_peak, 4),
        # the same against the nominal ~8 TB/s of B200 HBM3e
        "hbm_frac_of_8tbs": round(fwd_gbs / 8000.0, 4),
        "hbm_peak": {"gbs": hbm_peak, "kind": peak_kind},
        "roofline": {"bound": "hbm", "kernel": "tc_kernel (gate/up and down items; one fused launch at decode)",
                     "achieved": round(tc_gbs, 1) if tc_gbs else None, "peak": hbm_peak,
                     "unit": "GB/s", "frac": round(tc_gbs / hbm_peak, 4) if tc_gbs else None,
                     "traffic": traffic,
                     "traffic_source": ("recorded: dram__bytes_read.sum + dram__bytes_write.sum "
                                        "of an ncu capture of this kernel source "
                                        "(profiles/traffic_per_forward.json)")
                                       if traffic else None,
                     "launch_ms_per_forward": [round(m / max(n_fwd, 1), 5) for m in per_launch]},
        "cpu_baseline": cpu,
        "accuracy": accuracy,
        "e2e": {"value": round(e2e_tok_s, 1), "unit": "tokens/s",
                "h2d_bytes_per_step": int(T * wl.hidden * 2),
                "d2h_bytes_per_step": int(T * wl.hidden * 2)},
        "clocks": clk.summary(t_begin, t_end),
        "gpu_launches": launches,
        "workspace_bytes": {"headline_max_tokens_64": int(binding.workspace_bytes(
                                dict(d.cfg, max_tokens=64))),
                            "mixtral_max_tokens_4096": int(binding.workspace_bytes(
                                dict(d.cfg, max_tokens=4096)))},
        "sweep": sweep,
        "page_move": page_move,
        "prefill": prefill,
        "uniform_vs_mixed": uniform,
        "paging": paging,
        "small_batch_paths": small,
    }
    return out


def cpu_baseline(layer, x_np, T, budget_s=12.0):
    """The oracle as it stands, on this host's cores, one token at a time
    until the time budget is spent (a bounded sample of the batch)."""
    import oracle
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from pw_testutil import oracle_layer
    threads = oracle.default_threads()
    L = oracle_layer(oracle, layer)
    done = 0
    outs = []
    t0 = time.perf_counter()
    while done < T and (time.perf_counter() - t0) < budget_s:
        o, _, _ = L.forward(x_np[done:done + 1], layer.router_w, layer.router_bias,
                            threads=threads)
        outs.append(o[0])
        done += 1
    dt = time.perf_counter() - t0
    # the same oracle on one thread, one token (the per-core figure)
    t1 = time.perf_counter()
    L.forward(x_np[0:1], layer.router_w, layer.router_bias, threads=1)
    one = 1.0 / (time.perf_counter() - t1)
    return ({"value": round(done / dt, 3), "unit": "tokens/s", "cores": threads, "kind": "oracle",
             "sample": "%d of the %d tokens of one batch, one token per oracle call, %.1f s"
                       % (done, T, dt),
             "one_thread_tokens_per_s": round(one, 4)}, outs)


def run_reference(args):
    """The oracle timed as the reference arm on the headline workload.  Each
    step is one bounded sample: one token's routing in full and, for every
    expert it selects, the first `frac` of each block's output rows through
    the oracle's own linear routine (frac sized so that warm-up plus timed
    steps take about two minutes; 1 when that allows whole tokens).  The
    value counts frac tokens per step."""
    from any_precision_weight_pw_b200 import synth
    import oracle
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from pw_testutil import oracle_layer
    name, T = HEADLINE
    layer = synth.Layer(synth.WORKLOADS[name], seed=0)
    wl = layer.wl
    x = synth.tokens(wl, T, seed=0, batch=0)
    threads = oracle.default_threads()
    # calibrate: one whole token through the oracle layer
    L = oracle_layer(oracle, layer)
    t0 = time.perf_counter()
    L.forward(x[0:1], layer.router_w, layer.router_bias, threads=threads)
    t_tok = time.perf_counter() - t0
    del L
    budget_s = 120.0
    frac = min(1.0, budget_s / max((args.steps + args.warmup) * t_tok, 1e-9))
    sliced = {}
    for blk in range(wl.n_blocks):
        rows, cols = layer.shape(blk)
        R = max(1, int(round(rows * frac)))
        b = layer.bits[blk]
        sliced[blk] = (np.ascontiguousarray(layer.planes(blk)[:, :R, :]),
                       np.ascontiguousarray(layer.lut(blk, b)[:R]), cols, b, R)

    def step(t):
        xt = x[t % T:t % T + 1]
        logits = oracle.router_logits(xt, layer.router_w, layer.router_bias)
        idx, _ = oracle.topk_softmax(logits, wl.top_k, bool(wl.renorm_topk))
        experts = [int(e) for e in idx[0]] + ([wl.n_experts] if wl.shared_ffn else [])
        xf = synth.bf16_bits_to_float(xt[0]).astype(np.float64)
        for e in experts:
            pg, lg, cg, bg, rg = sliced[3 * e]
            pu, lu, cu, bu, _ = sliced[3 * e + 1]
            pd, ld, cd, bd, _ = sliced[3 * e + 2]
            g = oracle.linear(pg, lg, cg, bg, xf, threads)
            u = oracle.linear(pu, lu, cu, bu, xf, threads)
            h = np.zeros(cd)
            h[:rg] = g / (1.0 + np.exp(-g)) * u
            oracle.linear(pd, ld, cd, bd, h, threads)

    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        step(i)
    dt = time.perf_counter() - t0
    value = frac * args.steps / dt
    sample = ("per step: one token's routing and %.4f of the output rows of every block it "
              "selects (%d steps)" % (frac, args.steps))
    return {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "tokens/s",
            "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(dt / args.steps * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "%s decode T=%d" % HEADLINE, "hidden": wl.hidden,
                       "ffn": wl.ffn, "experts": wl.n_experts, "top_k": wl.top_k},
            "cpu_baseline": {"value": round(value, 4), "unit": "tokens/s", "cores": threads,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 4), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-sweep", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--decode", nargs=2, metavar=("WORKLOAD", "T"),
                    help="only a few forwards of one decode workload (an entry point for ncu "
                         "captures; one JSON object)")
    ap.add_argument("--quick", action="store_true",
                    help="headline and decode sweep only (no page-move, prefill, uniform-width "
                         "and paging measurements)")
    ap.add_argument("--prefill", action="store_true",
                    help="only the prefill-scale measurement (one JSON object; for profiling)")
    args = ap.parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.decode:
        import torch
        print(json.dumps(decode_only(torch.device("cuda", local_rank), args.decode[0],
                                     int(args.decode[1]))), flush=True)
        return
    if args.prefill:
        import torch
        print(json.dumps(prefill_measure(torch.device("cuda", local_rank), steps=max(args.steps, 1),
                                         warmup=max(args.warmup, 1))), flush=True)
        return
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return
    if world > 1:
        import datetime
        import torch
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    out = run_ours(args, rank, world, local_rank)
    if rank == 0 and out is not None:
        print(json.dumps(out), flush=True)
    if world > 1:
        import torch
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
