"""The multi-rank host logic of bench.py (replicas: one process per GPU, no
data-path collective) on CPU with two gloo ranks: every rank gets the slowest
rank's time, the whole-job rate counts every rank's tokens, each rank builds
its own seeded replica, and the reference arm prints on rank 0 only."""
import json
import os
import socket
import subprocess
import sys

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        from any_precision_weight_pw_b200 import synth
        local_ms = [12.5, 17.25][rank]
        ms = bench.max_over_ranks(local_ms, world)
        rate = bench.whole_job_rate(world, 100, 16, ms)
        # replicas: rank r draws its own seeded layer and tokens
        x = synth.tokens(synth.WORKLOADS["tiny_h256_f512_e8k2"], 4, seed=rank)
        gathered = [None] * world
        dist.all_gather_object(gathered, x.tobytes().hex()[:64])
        out.put((rank, ms, rate, gathered))
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_and_replicas():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms, rate, gathered in res:
        assert ms == 17.25                          # the slowest rank's time
        assert rate == pytest.approx(2 * 100 * 16 / 17.25e-3)
        assert gathered[0] != gathered[1]           # independent replicas


def test_reference_arm_prints_on_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "1"], capture_output=True, text=True,
                       env=env, timeout=120)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_single_rank_helpers():
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.whole_job_rate(1, 10, 16, 2.0) == pytest.approx(80000.0)
