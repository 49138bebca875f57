"""GPU parity: the CUDA library (through its C ABI) against the CPU oracle on
the same seeded inputs.

Bit-exact: unpacked codes (identity LUT with one-hot inputs returns every
code), integer linear results, and the top-k expert indices and order.
Floating point: the output tolerance of tests/pw_testutil.py.
"""
import os

import numpy as np
import pytest

from any_precision_weight_pw_b200 import synth
from pw_testutil import assert_output_close, oracle_layer, output_errors

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def pw():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from any_precision_weight_pw_b200 import binding, build
    build.build()
    return binding


def _dev_planes(planes, cols, pw):
    """Row-major planes -> plane pages on the device (the library's layout)."""
    dev = torch.from_numpy(np.ascontiguousarray(planes).view(np.int32)).cuda()
    return pw.repack_planes(dev, cols)


def _dev_lut(lut):
    return torch.from_numpy(np.ascontiguousarray(lut).view(np.int16)).cuda()


def _dev_bf16(xbits):
    return torch.from_numpy(np.ascontiguousarray(xbits).view(np.int16)).cuda()


def _to_f32(y):
    """bf16 device tensor (int16 storage) -> float32 numpy."""
    return (y.view(torch.int16).cpu().numpy().view(np.uint16).astype(np.uint32) << 16).view(np.float32)


def _identity_lut(rows, b):
    return np.tile(np.arange(1 << b, dtype=np.float16), (rows, 1)).view(np.uint16)


# ---------------------------------------------------------------- page layout

def _paged_reference(planes, cols):
    """The paged layout written out from its definition: tile groups of 128
    rows x 8 words in (row tile, word tile) order, each holding the n planes'
    tiles of 1024 words one after the other; row r at 8r words within a tile,
    its two 4-word halves swapped when bit 2 of r is set."""
    n, rows, words = planes.shape
    n_rt, n_kt = -(-rows // 128), -(-words // 8)
    padded = np.zeros((n, n_rt * 128, n_kt * 8), np.uint32)
    padded[:, :rows, :words] = planes
    out = np.zeros((n_rt, n_kt, n, 128, 8), np.uint32)
    for rt in range(n_rt):
        for kt in range(n_kt):
            for k in range(n):
                tile = padded[k, rt * 128:(rt + 1) * 128, kt * 8:(kt + 1) * 8]
                for r in range(128):
                    row = tile[r]
                    out[rt, kt, k, r] = np.concatenate([row[4:], row[:4]]) if (r >> 2) & 1 else row
    return out.reshape(-1)


@pytest.mark.parametrize("rows,cols", [(128, 256), (200, 300), (5, 33), (300, 1408)])
def test_repack_matches_page_layout(pw, rows, cols):
    rng = np.random.default_rng(rows + cols)
    planes = synth.random_planes(rng, 3, rows, cols)
    got = _dev_planes(planes, cols, pw).cpu().numpy().view(np.uint32)
    assert got.size * 4 == 3 * pw.plane_bytes(rows, cols)
    np.testing.assert_array_equal(got, _paged_reference(planes, cols))


# ---------------------------------------------------------------- pw_linear

LINEAR_SHAPES = [
    (256, 256),   # tensor-core path, full tiles
    (200, 384),   # tensor-core path, partial row tile, ragged K stage
    (64, 40),     # CUDA-core path (ceil(40/32) = 2 words)
]


@pytest.mark.parametrize("rows,cols", LINEAR_SHAPES)
@pytest.mark.parametrize("b", [1, 2, 3, 4, 5, 6, 7, 8])
def test_linear_unpacks_codes_bit_exactly(pw, oracle, rows, cols, b):
    """Identity LUT and one-hot tokens: y[t][o] = code_b(o, t) for every column."""
    rng = np.random.default_rng(rows * 100 + cols + b)
    planes = synth.random_planes(rng, 8, rows, cols)
    want = oracle.unpack_codes(planes, cols, b).astype(np.float32).T  # [cols][rows]
    x = synth.to_bf16_bits(np.eye(cols, dtype=np.float32))
    y = pw.linear(_dev_planes(planes, cols, pw), _dev_lut(_identity_lut(rows, b)), b, _dev_bf16(x),
                  rows)
    np.testing.assert_array_equal(y.cpu().numpy(), want)


@pytest.mark.parametrize("rows,cols", LINEAR_SHAPES)
def test_linear_integer_exact(pw, oracle, rows, cols):
    rng = np.random.default_rng(7)
    planes = synth.random_planes(rng, 8, rows, cols)
    for b in (3, 4, 6, 8):
        x = rng.integers(-8, 9, size=(37, cols)).astype(np.float32)
        codes = oracle.unpack_codes(planes, cols, b).astype(np.int64)
        want = (x.astype(np.int64) @ codes.T).astype(np.float32)
        y = pw.linear(_dev_planes(planes, cols, pw), _dev_lut(_identity_lut(rows, b)), b,
                      _dev_bf16(synth.to_bf16_bits(x)), rows)
        np.testing.assert_array_equal(y.cpu().numpy(), want)


@pytest.mark.parametrize("rows,cols", LINEAR_SHAPES + [(1408, 2048), (512, 1408)])
def test_linear_random_matches_oracle(pw, oracle, rows, cols):
    rng = np.random.default_rng(11)
    planes = synth.random_planes(rng, 8, rows, cols)
    for b in (3, 5, 8):
        lut = synth.random_lut(rng, rows, b)
        x = synth.to_bf16_bits(rng.normal(size=(5, cols)).astype(np.float32))
        ref = oracle.linear(planes, lut, cols, b, synth.bf16_bits_to_float(x).astype(np.float64),
                            threads=8)
        y = pw.linear(_dev_planes(planes, cols, pw), _dev_lut(lut), b, _dev_bf16(x),
                      rows).cpu().numpy()
        scale = np.abs(ref).max()
        assert np.abs(y - ref).max() <= 1e-5 * scale * max(1.0, cols / 1024)


# ---------------------------------------------------------------- whole layer

def _run_layer(pw, layer, T, batch=0, force_simple=False):
    os.environ["PW_FORCE_SIMPLE"] = "1" if force_simple else "0"
    try:
        dev = pw.upload_synth_layer(layer, max_tokens=max(T, 1))
    finally:
        os.environ.pop("PW_FORCE_SIMPLE", None)
    x = synth.tokens(layer.wl, T, seed=layer.seed, batch=batch)
    xd = _dev_bf16(x)
    wr = torch.from_numpy(layer.router_w).cuda()
    bias = None if layer.router_bias is None else torch.from_numpy(layer.router_bias).cuda()
    y = dev.forward(xd, wr, bias)
    idx, w = dev.routing(T)
    torch.cuda.synchronize()
    dev.check_device_error()
    yf = _to_f32(y)
    out = (yf, idx.cpu().numpy(), w.cpu().numpy(), x)
    dev.close()
    return out


def _oracle_forward(oracle, layer, x, threads=16):
    L = oracle_layer(oracle, layer)
    return L.forward(x, layer.router_w, layer.router_bias, threads=threads)


@pytest.mark.parametrize("force_simple", [False, True])
def test_tiny_layer(pw, oracle, force_simple):
    layer = synth.Layer(synth.WORKLOADS["tiny_h256_f512_e8k2"], seed=0)
    y, idx, w, x = _run_layer(pw, layer, 16, force_simple=force_simple)
    ref, ridx, rw = _oracle_forward(oracle, layer, x)
    np.testing.assert_array_equal(idx, ridx)
    np.testing.assert_allclose(w, rw, rtol=2e-6, atol=1e-7)
    assert_output_close(y, ref)


def test_tiny_layer_many_tokens_one_expert(pw, oracle):
    """A router bias sends every token to expert 3 first: 70 tokens -> three
    token tiles for that expert; the second slot spreads over the rest."""
    layer = synth.Layer(synth.WORKLOADS["tiny_h256_f512_e8k2"], seed=1)
    layer.router_bias = np.zeros(8, np.float32)
    layer.router_bias[3] = 50.0
    y, idx, w, x = _run_layer(pw, layer, 70)
    ref, ridx, rw = _oracle_forward(oracle, layer, x)
    assert np.all(idx[:, 0] == 3)
    np.testing.assert_array_equal(idx, ridx)
    assert_output_close(y, ref)


def test_hand_example_on_gpu(pw, oracle):
    """The 2-expert, 4x32 hand example (CUDA-core path: 1-word rows)."""
    from test_oracle_layer import _hand_layer
    L, Wr, x = _hand_layer(oracle)
    cfg = dict(hidden=32, ffn=4, n_experts=2, top_k=2, shared_ffn=0, n_max=3, renorm_topk=1,
               max_tokens=3)
    planes, slots, bits = [], [], []
    for (pl, lt, rows, cols, b) in L.block_list:
        planes.append(_dev_planes(pl, cols, pw))
        s0 = torch.zeros(rows << 3, dtype=torch.int16, device="cuda")
        s0[: lt.size].copy_(torch.from_numpy(lt.reshape(-1).view(np.int16)))
        slots.append((s0, torch.zeros_like(s0)))
        bits.append(b)
    dev = pw.MoELayer(cfg, planes, slots, bits)
    y = dev.forward(_dev_bf16(x), torch.from_numpy(Wr).cuda())
    idx, w = dev.routing(3)
    torch.cuda.synchronize()
    assert idx.cpu().numpy().tolist() == [[0, 1], [1, 0], [0, 1]]
    yf = _to_f32(y)
    want = [[-0.9035184, -0.9142537, 0.3580196, 0.3472844],
            [-0.6708742, -0.6615392, 0.5634112, 0.5727461],
            [-0.9166429, -0.9241294, 0.4995289, 0.4920425]]
    ref, _, _ = L.forward(x, Wr)
    np.testing.assert_allclose(ref[:, :4], want, atol=6e-8)
    assert_output_close(yf, ref)
    dev.close()


@pytest.mark.parametrize("T", [1, 8, 32])
def test_qwen_shaped_layer(pw, oracle, T):
    layer = synth.Layer(synth.WORKLOADS["qwen15_moe_a27b"], seed=0)
    y, idx, w, x = _run_layer(pw, layer, T, batch=T)
    ref, ridx, rw = _oracle_forward(oracle, layer, x)
    np.testing.assert_array_equal(idx, ridx)
    np.testing.assert_allclose(w, rw, rtol=2e-6, atol=1e-7)
    assert_output_close(y, ref)


@pytest.mark.parametrize("T", [1, 16, 64])
def test_mixtral_shaped_layer(pw, oracle, T):
    layer = synth.Layer(synth.WORKLOADS["mixtral_8x7b"], seed=0)
    y, idx, w, x = _run_layer(pw, layer, T, batch=T)
    ref, ridx, rw = _oracle_forward(oracle, layer, x, threads=32)
    np.testing.assert_array_equal(idx, ridx)
    assert_output_close(y, ref)


def test_repeat_runs_are_bitwise_identical(pw):
    layer = synth.Layer(synth.WORKLOADS["tiny_h256_f512_e8k2"], seed=2)
    dev = pw.upload_synth_layer(layer, max_tokens=16)
    x = _dev_bf16(synth.tokens(layer.wl, 16, seed=2))
    wr = torch.from_numpy(layer.router_w).cuda()
    a = dev.forward(x, wr).clone()
    b = dev.forward(x, wr).clone()
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    dev.close()


def test_zero_tokens_and_bad_T(pw):
    layer = synth.Layer(synth.WORKLOADS["tiny_h256_f512_e8k2"], seed=0)
    dev = pw.upload_synth_layer(layer, max_tokens=4)
    wr = torch.from_numpy(layer.router_w).cuda()
    x = torch.zeros((0, 256), dtype=torch.int16, device="cuda")
    y = dev.forward(x, wr)
    assert y.shape == (0, 256)
    with pytest.raises(pw.PwError):
        dev.forward(torch.zeros((5, 256), dtype=torch.int16, device="cuda"), wr)
    dev.close()


def test_bitwidth_switch_waits_at_lag_zero(pw, oracle):
    """max_lag 0: the forward issued right after the requests waits for the
    page moves and uses the new widths; it and the next match the oracle at
    those widths, and the widths reported before it are the old ones."""
    wl = synth.WORKLOADS["tiny_h256_f512_e8k2"]
    layer = synth.Layer(wl, seed=3)
    dev = pw.upload_synth_layer(layer, max_tokens=16, host_copies=True)
    dev.set_switch_lag(0)
    wr = torch.from_numpy(layer.router_w).cuda()
    side = torch.cuda.Stream()
    changes = {0: 8, 4: 2, 5: 6, 11: 1, 23: 8}
    x0 = synth.tokens(wl, 16, seed=3, batch=0)
    dev.forward(_dev_bf16(x0), wr)                      # forward 0
    old = list(layer.bits)
    assert dev.forward_bits() == old
    for blk, b in changes.items():
        dev.set_block_bits(blk, b, side)
        assert dev.get_block_bits(blk) == (old[blk], b)
    with pytest.raises(pw.PwError):
        dev.set_block_bits(0, 3, side)                  # still pending
    new = list(old)
    for blk, b in changes.items():
        new[blk] = b
    for f in (1, 2):
        x = synth.tokens(wl, 16, seed=3, batch=f)
        y = dev.forward(_dev_bf16(x), wr)
        assert dev.forward_bits() == new
        torch.cuda.synchronize()
        ref, _, _ = oracle_layer(oracle, layer, new).forward(x, layer.router_w, threads=8)
        assert_output_close(_to_f32(y), ref)
    for blk, b in changes.items():
        assert dev.get_block_bits(blk) == (b, 0)
    dev.check_device_error()
    dev.close()


def test_bitwidth_switch_async_replay(pw, oracle):
    """Default lag: a change takes effect at the first forward issued after
    its copy has landed (at the latest max_lag forwards after the request);
    every forward matches the oracle at the widths it reports."""
    wl = synth.WORKLOADS["tiny_h256_f512_e8k2"]
    layer = synth.Layer(wl, seed=6)
    dev = pw.upload_synth_layer(layer, max_tokens=16, host_copies=True)
    wr = torch.from_numpy(layer.router_w).cuda()
    side = torch.cuda.Stream()
    sched = {1: [(2, 8), (7, 1)], 3: [(2, 3), (13, 7), (20, 2)]}
    want = list(layer.bits)
    for f in range(12):
        for blk, b in sched.get(f, []):
            dev.set_block_bits(blk, b, side)
            want[blk] = b
        x = synth.tokens(wl, 16, seed=6, batch=f)
        y = dev.forward(_dev_bf16(x), wr)
        used = dev.forward_bits()
        torch.cuda.synchronize()   # lets the copies land before the next forward
        ref, _, _ = oracle_layer(oracle, layer, used).forward(x, layer.router_w, threads=8)
        assert_output_close(_to_f32(y), ref)
        if f in (2, 4) or f > 4:
            # the previous forward's synchronize let every copy requested
            # before it land, so this forward found them complete
            assert used == want, (f, used, want)
    dev.check_device_error()
    dev.close()


def test_switch_stress_replay_qwen_shaped(pw, oracle):
    """The Qwen-shaped switch stress (decode batch 32; before every 10th
    forward a quarter of the blocks change width, page moves on a side
    stream), 41 forwards issued back to back.  The widths each forward
    reports are replayed through the oracle: forward 0, every 10th, and the
    first forwards after each switch at which part and all of its changes
    had landed are compared."""
    wl = synth.WORKLOADS["qwen15_moe_a27b_switch"]
    T = wl.tokens[0]
    layer = synth.Layer(wl, seed=0)
    dev = pw.upload_synth_layer(layer, max_tokens=T, host_copies=True)
    wr = torch.from_numpy(layer.router_w).cuda()
    side = torch.cuda.Stream()
    n = 41
    sched = synth.switch_schedule(wl, layer.bits, n, every=10)
    assert all(len(v) == round(0.25 * wl.n_blocks) for v in sched.values())
    ys, used, want_after = [], [], {}
    want = list(layer.bits)
    for f in range(n):
        for blk, b in sched.get(f, []):
            dev.set_block_bits(blk, b, side)
            want[blk] = b
        if f in sched:
            want_after[f] = list(want)
        x = synth.tokens(wl, T, seed=0, batch=f)
        ys.append(dev.forward(_dev_bf16(x), wr))
        used.append(dev.forward_bits())
    torch.cuda.synchronize()
    dev.check_device_error()
    lag = 8
    pick = {0} | {f for f in range(0, n, 10)}
    for f0, w in want_after.items():
        # every change of the switch took effect within the lag
        full = [f for f in range(f0, min(n, f0 + lag + 1)) if used[f] == w]
        assert full, "switch before forward %d never completed within the lag" % f0
        pick.add(full[0])
        part = [f for f in range(f0, full[0] + 1) if used[f] != used[f - 1]]
        if part:
            pick.add(part[0])
    assert used[-1] == want
    for f in sorted(pick):
        x = synth.tokens(wl, T, seed=0, batch=f)
        ref, ridx, _ = oracle_layer(oracle, layer, used[f]).forward(x, layer.router_w, threads=32)
        assert_output_close(_to_f32(ys[f]), ref)
    dev.close()


def test_switch_rejects_missing_host_copies(pw):
    """Raising the width of a block without host planes, and a width without
    a host LUT, are rejected with nothing enqueued; the layer keeps working."""
    wl = synth.WORKLOADS["tiny_h256_f512_e8k2"]
    layer = synth.Layer(wl, seed=0)
    side = torch.cuda.Stream()
    b0 = layer.bits[0]
    bare = pw.upload_synth_layer(layer, max_tokens=4)     # no host copies at all
    with pytest.raises(pw.PwError) as e:
        bare.set_block_bits(0, b0 - 1, side)              # no host LUT for that width
    assert e.value.status == 1 and "LUT" in str(e.value)
    bare.close()
    dev = pw.upload_synth_layer(layer, max_tokens=4, host_copies=True, host_planes=False)
    with pytest.raises(pw.PwError) as e:
        dev.set_block_bits(0, b0 + 1, side)               # raising needs the host planes
    assert e.value.status == 1 and "planes" in str(e.value)
    assert dev.get_block_bits(0) == (b0, 0)
    dev.set_block_bits(0, b0 - 1, side)                   # lowering needs only the LUT
    assert dev.get_block_bits(0) == (b0, b0 - 1)
    wr = torch.from_numpy(layer.router_w).cuda()
    dev.forward(_dev_bf16(synth.tokens(wl, 4, seed=0)), wr)
    torch.cuda.synchronize()
    dev.check_device_error()
    dev.close()


def test_destroy_with_work_in_flight(pw):
    """pw_destroy while a forward and a page move are still queued waits for
    them and returns PW_OK."""
    wl = synth.WORKLOADS["tiny_h256_f512_e8k2"]
    layer = synth.Layer(wl, seed=0)
    dev = pw.upload_synth_layer(layer, max_tokens=16, host_copies=True)
    wr = torch.from_numpy(layer.router_w).cuda()
    side = torch.cuda.Stream()
    x = _dev_bf16(synth.tokens(wl, 16, seed=0))
    dev.forward(x, wr)
    dev.set_block_bits(1, 8, side)
    dev.forward(x, wr)
    dev.close()                                          # raises on a non-OK status
    torch.cuda.synchronize()


def test_forward_host_matches_device(pw):
    layer = synth.Layer(synth.WORKLOADS["tiny_h256_f512_e8k2"], seed=4)
    dev = pw.upload_synth_layer(layer, max_tokens=16)
    x = synth.tokens(layer.wl, 16, seed=4)
    wr = torch.from_numpy(layer.router_w).cuda()
    yd = dev.forward(_dev_bf16(x), wr).cpu()
    xh = torch.from_numpy(x.view(np.int16)).pin_memory()
    yh = dev.forward_host(xh, wr)
    assert torch.equal(yd, yh)
    dev.close()


def test_prefill_scale_layer_sampled(pw, oracle):
    """Mixtral-shaped layer at prefill scale (4096 tokens, Zipf(1.2)-skewed
    expert usage, experts 0 and 1 at 8 bits, the rest at 4): every token's
    routing is compared with the oracle's, expert 0's top-1 share is Zipf's
    0.429 +- 0.02, and the outputs of a stratified sample of 256 tokens (32
    whose first choice is each expert, so both 8-bit experts and every
    other) are compared (the oracle computes each token on its own)."""
    wl = synth.WORKLOADS["mixtral_8x7b_prefill"]
    layer = synth.Layer(wl, seed=0)
    T = 4096
    y, idx, w, x = _run_layer(pw, layer, T)
    logits = oracle.router_logits(x, layer.router_w, layer.router_bias)
    ridx, rw = oracle.topk_softmax(logits, wl.top_k, bool(wl.renorm_topk))
    np.testing.assert_array_equal(idx, ridx)
    np.testing.assert_allclose(w, rw, rtol=1e-5, atol=1e-7)
    top1 = np.bincount(idx[:, 0], minlength=wl.n_experts) / T
    assert abs(top1[0] - synth.zipf_pmf(wl.n_experts, wl.zipf_s)[0]) <= 0.02, top1
    rng = np.random.default_rng(7)
    per = 256 // wl.n_experts
    sample = np.sort(np.concatenate([
        rng.choice(np.flatnonzero(idx[:, 0] == e), per, replace=False)
        for e in range(wl.n_experts)]))
    assert sample.size == 256
    L = oracle_layer(oracle, layer)
    ref, sidx, _ = L.forward(x[sample], layer.router_w, layer.router_bias, threads=64)
    np.testing.assert_array_equal(sidx, idx[sample])
    assert_output_close(y[sample], ref)


def _run_layer_env(pw, layer, T, env, batch=0):
    old = {k: os.environ.get(k) for k in env}
    os.environ.update(env)
    try:
        return _run_layer(pw, layer, T, batch=batch)
    finally:
        for k, v in old.items():
            if v is None:
                os.environ.pop(k, None)
            else:
                os.environ[k] = v


@pytest.mark.parametrize("T,bias_expert", [(200, None), (300, 5)])
def test_prefill_passes_tiny_layer(pw, oracle, T, bias_expert):
    """The prefill passes (256-token chunks; gate, up and down launches) on
    the tiny layer, every output compared; with a router bias one expert gets
    every token (two chunks, the second partial)."""
    layer = synth.Layer(synth.WORKLOADS["tiny_h256_f512_e8k2"], seed=4)
    if bias_expert is not None:
        layer.router_bias = np.zeros(8, np.float32)
        layer.router_bias[bias_expert] = 50.0
    y, idx, w, x = _run_layer_env(pw, layer, T, {"PW_PREFILL": "1"})
    ref, ridx, rw = _oracle_forward(oracle, layer, x, threads=32)
    np.testing.assert_array_equal(idx, ridx)
    assert_output_close(y, ref)
    # the decode passes give the same routing and outputs within the same bound
    y2, idx2, _, _ = _run_layer_env(pw, layer, T, {"PW_PREFILL": "0"})
    np.testing.assert_array_equal(idx2, ridx)
    assert_output_close(y2, ref)


def test_prefill_passes_qwen_shaped_sampled(pw, oracle):
    """Qwen-shaped layer (shared expert of 5632) through the prefill passes at
    320 tokens: all routing, and the outputs of a token sample."""
    layer = synth.Layer(synth.WORKLOADS["qwen15_moe_a27b"], seed=5)
    T = 320
    y, idx, w, x = _run_layer_env(pw, layer, T, {"PW_PREFILL": "1"})
    wl = layer.wl
    ridx, _ = oracle.topk_softmax(oracle.router_logits(x, layer.router_w, None), wl.top_k,
                                  bool(wl.renorm_topk))
    np.testing.assert_array_equal(idx, ridx)
    sample = np.array([0, 1, 77, 150, 255, 256, 300, T - 1])
    L = oracle_layer(oracle, layer)
    ref, _, _ = L.forward(x[sample], layer.router_w, None, threads=32)
    assert_output_close(y[sample], ref)


@pytest.mark.parametrize("name,T,n_fwd", [("tiny_h256_f512_e8k2", 16, 1000),
                                          ("qwen15_moe_a27b", 32, 20)])
def test_routing_stats_accumulate_over_forwards(pw, oracle, name, T, n_fwd):
    """The route kernel's per-expert counters (assignments and routing-weight
    mass, the planner's online routing mass) over many forwards of distinct
    batches: counts equal the oracle's exactly, mass within 1e-5 relative;
    a read with reset zeroes them."""
    wl = synth.WORKLOADS[name]
    layer = synth.Layer(wl, seed=8)
    dev = pw.upload_synth_layer(layer, max_tokens=T)
    wr = torch.from_numpy(layer.router_w).cuda()
    counts = np.zeros(wl.n_experts, np.uint64)
    mass = np.zeros(wl.n_experts, np.float64)
    y = torch.empty((T, wl.hidden), dtype=torch.int16, device="cuda")
    for f in range(n_fwd):
        x = synth.tokens(wl, T, seed=8, batch=f)
        dev.forward(_dev_bf16(x), wr, None, y)
        idx, w = oracle.topk_softmax(oracle.router_logits(x, layer.router_w, None), wl.top_k,
                                     bool(wl.renorm_topk))
        oracle.routing_stats(idx, w, wl.n_experts, counts, mass)
    got_c, got_m = dev.routing_stats(reset=True)
    dev.check_device_error()
    np.testing.assert_array_equal(got_c, counts)
    np.testing.assert_allclose(got_m, mass, rtol=1e-5, atol=1e-9)
    assert int(got_c.sum()) == n_fwd * T * wl.top_k
    c2, m2 = dev.routing_stats()
    assert not c2.any() and not m2.any()
    dev.close()


def _plane_total(pw, layer, bits):
    return sum(b * pw.plane_bytes(*layer.shape(blk)) for blk, b in enumerate(bits))


def test_paging_offload_reload_parity(pw, oracle):
    """Library-owned plane storage: after pw_enable_paging the caller's plane
    buffers are overwritten with garbage and the layer still matches the
    oracle; lowering widths offloads planes (resident bytes fall by exactly
    the released plane pages), raising them reloads planes from the host
    copies, and every forward matches the oracle at the widths it used."""
    wl = synth.WORKLOADS["tiny_h256_f512_e8k2"]
    layer = synth.Layer(wl, seed=11)
    dev = pw.upload_synth_layer(layer, max_tokens=16, host_copies=True)
    dev.set_switch_lag(0)
    wr = torch.from_numpy(layer.router_w).cuda()
    side = torch.cuda.Stream()
    assert dev.resident_bytes()[0] == 8 * _plane_total(pw, layer, [1] * wl.n_blocks)
    dev.enable_paging()
    bits = list(layer.bits)
    assert dev.resident_bytes()[0] == _plane_total(pw, layer, bits)
    for t in dev._keep[0]:                 # the caller's plane buffers
        t.fill_(-1)
    torch.cuda.synchronize()

    def check(f):
        x = synth.tokens(wl, 16, seed=11, batch=f)
        y = dev.forward(_dev_bf16(x), wr)
        used = dev.forward_bits()
        torch.cuda.synchronize()
        ref, _, _ = oracle_layer(oracle, layer, used).forward(x, layer.router_w, threads=8)
        assert_output_close(_to_f32(y), ref)
        return used

    assert check(0) == bits
    down = {0: 1, 1: 2, 5: 1, 9: 2, 16: 1, 23: 2}
    for blk, b in down.items():
        dev.set_block_bits(blk, b, side)
        bits[blk] = b
    assert check(1) == bits
    assert dev.resident_bytes()[0] == _plane_total(pw, layer, bits)
    up = {0: 8, 5: 6, 9: 3, 12: 7}
    for blk, b in up.items():
        dev.set_block_bits(blk, b, side)
        bits[blk] = b
    assert check(2) == bits
    assert check(3) == bits
    plane, reserved = dev.resident_bytes(trim=True)
    assert plane == _plane_total(pw, layer, bits) and reserved >= plane
    dev.check_device_error()
    dev.close()


def test_paging_planner_frees_device_memory(pw, oracle):
    """Qwen-shaped layer with paging: routing mass from the library's own
    counters over 20 forwards, the planner frees a quarter of the resident
    plane bytes, the plan is applied as page moves, and (a) resident bytes
    fall by what the planner released in plane pages, (b) the pool still
    covers what stays resident after a trim, (c) the next forwards match the oracle
    at the widths they used.  (The pool reserves memory in 2 MB mappings,
    so how much of the released bytes it can hand back depends on
    fragmentation; only the accounting is exact.)"""
    wl = synth.WORKLOADS["qwen15_moe_a27b"]
    layer = synth.Layer(wl, seed=12)
    T = 32
    dev = pw.upload_synth_layer(layer, max_tokens=T, host_copies=True)
    dev.enable_paging()
    for t in dev._keep[0]:
        t.fill_(-1)
    wr = torch.from_numpy(layer.router_w).cuda()
    for f in range(20):
        dev.forward(_dev_bf16(synth.tokens(wl, T, seed=12, batch=f)), wr)
    counts, mass = dev.routing_stats()
    resident0, reserved0 = dev.resident_bytes(trim=True)
    rng = np.random.default_rng(12)
    blocks = []
    for blk in range(wl.n_blocks):
        rows, cols = layer.shape(blk)
        e = blk // 3
        sens = [0.0] + [float(rng.random() + 0.5) * 2.0 ** (8 - b) for b in range(1, 9)]
        blocks.append(dict(bits=layer.bits[blk], min_bits=2, plane_bytes=pw.plane_bytes(rows, cols),
                           rows=rows, mass=float(mass[e]) if e < wl.n_experts else 20.0 * T,
                           resid=0.0, sens=sens))
    plan = pw.plan_release(blocks, resident0 // 4)
    assert plan["reached"] and plan == oracle.plan_greedy(blocks, resident0 // 4)
    side = torch.cuda.Stream()
    dev.set_switch_lag(0)
    for blk, b in enumerate(plan["bits"]):
        dev.set_block_bits(blk, b, side)
    x = synth.tokens(wl, T, seed=12, batch=99)
    y = dev.forward(_dev_bf16(x), wr)
    used = dev.forward_bits()
    assert used == plan["bits"]
    torch.cuda.synchronize()
    released_planes = sum((layer.bits[i] - b) * blocks[i]["plane_bytes"]
                          for i, b in enumerate(plan["bits"]))
    resident1, reserved1 = dev.resident_bytes(trim=True)
    assert resident1 == resident0 - released_planes
    assert 0 < reserved1 and resident1 <= reserved1
    ref, _, _ = oracle_layer(oracle, layer, used).forward(x, layer.router_w, threads=32)
    assert_output_close(_to_f32(y), ref)
    dev.check_device_error()
    dev.close()


def test_bounded_wait_times_out_and_the_handle_recovers(pw, oracle):
    """Failure detection without a fault: with the test switches, one
    expert's down items in the fused decode launch wait for a gate/up count
    that never arrives, under a 5 ms limit.  The wait gives up, every role of
    the CTA drains what it has in flight, the kernel returns, and
    pw_check_device_error reports PW_ERR_TIMEOUT once (then the word is
    clear).  The same handle's next forward, switches off, matches the
    oracle."""
    wl = synth.WORKLOADS["tiny_h256_f512_e8k2"]
    layer = synth.Layer(wl, seed=0)
    dev = pw.upload_synth_layer(layer, max_tokens=16)
    wr = torch.from_numpy(layer.router_w).cuda()
    x = synth.tokens(wl, 16, seed=0)
    idx_ref, _ = oracle.topk_softmax(oracle.router_logits(x, layer.router_w, None), wl.top_k,
                                     bool(wl.renorm_topk))
    stalled = int(idx_ref[0, 0])            # an expert with routed tokens
    os.environ["PW_TEST_WAIT_US"] = "5000"
    os.environ["PW_TEST_STALL_GROUP"] = str(stalled)
    try:
        dev.forward(_dev_bf16(x), wr)
        torch.cuda.synchronize()
    finally:
        os.environ.pop("PW_TEST_WAIT_US", None)
        os.environ.pop("PW_TEST_STALL_GROUP", None)
    with pytest.raises(pw.PwError) as e:
        dev.check_device_error()
    assert e.value.status == 4                 # PW_ERR_TIMEOUT
    dev.check_device_error()                   # cleared
    y = dev.forward(_dev_bf16(x), wr)
    torch.cuda.synchronize()
    dev.check_device_error()
    ref, _, _ = oracle_layer(oracle, layer).forward(x, layer.router_w, threads=8)
    assert_output_close(_to_f32(y), ref)
    dev.close()


def test_workspace_is_sized_to_its_use(pw):
    """The workspace query matches what a handle allocates, and a
    Mixtral-shaped layer able to run 4096-token prefill needs well under a
    gigabyte: the down partials are sized for the splits the passes use and
    share their region with the prefill gate outputs."""
    wl = synth.WORKLOADS["mixtral_8x7b"]
    cfg = dict(hidden=wl.hidden, ffn=wl.ffn, n_experts=wl.n_experts, top_k=wl.top_k,
               shared_ffn=0, n_max=8, renorm_topk=1, max_tokens=4096)
    big = pw.workspace_bytes(cfg)
    # gate outputs (fp16) + SwiGLU activations (fp16) + gathered rows (fp16)
    # + the host-forward staging rows (bf16 in and out)
    P = 4096 * 2
    core = P * wl.ffn * 2 + P * wl.ffn * 2 + P * wl.hidden * 2 + 2 * 4096 * wl.hidden * 2
    assert core <= big <= core + 64 * 2 ** 20, (big, core)
    small = pw.workspace_bytes(dict(cfg, max_tokens=16))
    assert small < 64 * 2 ** 20
    layer = synth.Layer(synth.WORKLOADS["tiny_h256_f512_e8k2"], seed=0)
    dev = pw.upload_synth_layer(layer, max_tokens=300)
    tcfg = dict(dev.cfg)
    assert pw.workspace_bytes(tcfg) > 0
    dev.close()


@pytest.mark.parametrize("name,T,bias_expert", [("tiny_h256_f512_e8k2", 1, None),
                                                ("tiny_h256_f512_e8k2", 3, None),
                                                ("tiny_h256_f512_e8k2", 4, 2),
                                                ("qwen15_moe_a27b", 2, None),
                                                ("mixtral_8x7b", 2, None)])
def test_cuda_core_decode_passes(pw, oracle, name, T, bias_expert):
    """The CUDA-core decode passes (few tokens per expert: gather, gate/up
    with SwiGLU, split-K down) against the oracle, and against the
    tensor-core passes on the same inputs (PW_GV=0) within the same bound;
    with a router bias all tokens share one expert (one token chunk)."""
    layer = synth.Layer(synth.WORKLOADS[name], seed=9)
    if bias_expert is not None:
        layer.router_bias = np.zeros(layer.wl.n_experts, np.float32)
        layer.router_bias[bias_expert] = 50.0
    y, idx, w, x = _run_layer_env(pw, layer, T, {"PW_GV_T": str(T)}, batch=T)
    ref, ridx, rw = _oracle_forward(oracle, layer, x, threads=32)
    np.testing.assert_array_equal(idx, ridx)
    assert_output_close(y, ref)
    y2, idx2, _, _ = _run_layer_env(pw, layer, T, {"PW_GV": "0"}, batch=T)
    np.testing.assert_array_equal(idx2, ridx)
    assert_output_close(y2, ref)


def test_cuda_core_decode_token_chunks_and_paging(pw, oracle):
    """Groups with more tokens than one item carries (12 tokens on one
    expert: three chunks of four), on paged storage after page moves."""
    wl = synth.WORKLOADS["tiny_h256_f512_e8k2"]
    layer = synth.Layer(wl, seed=10)
    layer.router_bias = np.zeros(8, np.float32)
    layer.router_bias[5] = 50.0
    old = os.environ.get("PW_GV_T")
    os.environ["PW_GV_T"] = "12"
    try:
        dev = pw.upload_synth_layer(layer, max_tokens=12, host_copies=True)
    finally:
        if old is None:
            os.environ.pop("PW_GV_T", None)
        else:
            os.environ["PW_GV_T"] = old
    dev.enable_paging()
    dev.set_switch_lag(0)
    side = torch.cuda.Stream()
    for blk, b in {15: 2, 16: 6, 17: 8, 3: 5}.items():
        dev.set_block_bits(blk, b, side)
    wr = torch.from_numpy(layer.router_w).cuda()
    bias = torch.from_numpy(layer.router_bias).cuda()
    x = synth.tokens(wl, 12, seed=10)
    y = dev.forward(_dev_bf16(x), wr, bias)
    used = dev.forward_bits()
    assert dev.launches(12) == 5          # route, gather, gate/up, down, combine
    torch.cuda.synchronize()
    dev.check_device_error()
    ref, ridx, _ = oracle_layer(oracle, layer, used).forward(x, layer.router_w, layer.router_bias,
                                                            threads=8)
    assert np.all(ridx[:, 0] == 5)
    assert_output_close(_to_f32(y), ref)
    dev.close()


def test_paging_compaction_returns_memory(pw, oracle):
    """Lower every block's width on paged storage, then pack the resident
    planes into one allocation: after a trim the pool reserves less than
    before and at most one mapping chunk more than the resident bytes, and
    the forwards before and after match the oracle."""
    wl = synth.WORKLOADS["qwen15_moe_a27b"]
    layer = synth.Layer(wl, seed=13)
    T = 8
    dev = pw.upload_synth_layer(layer, max_tokens=T, host_copies=True)
    dev.enable_paging()
    wr = torch.from_numpy(layer.router_w).cuda()
    side = torch.cuda.Stream()
    dev.set_switch_lag(0)
    bits = [max(2, b - 2) for b in layer.bits]
    for blk, b in enumerate(bits):
        dev.set_block_bits(blk, b, side)
    x = synth.tokens(wl, T, seed=13)
    y1 = dev.forward(_dev_bf16(x), wr)
    assert dev.forward_bits() == bits
    torch.cuda.synchronize()
    resident, reserved_before = dev.resident_bytes(trim=True)
    dev.compact_pages()
    y2 = dev.forward(_dev_bf16(x), wr)
    torch.cuda.synchronize()
    resident2, reserved_after = dev.resident_bytes(trim=True)
    assert resident2 == resident == _plane_total(pw, layer, bits)
    # the pool maps memory in chunks (32 MiB on the B200s measured): after
    # the trim it holds the packed copy rounded up to its mapping granularity
    assert reserved_after < reserved_before, (reserved_after, reserved_before)
    assert reserved_after <= resident + 32 * 2 ** 20, (reserved_after, resident, reserved_before)
    assert torch.equal(y1, y2)
    ref, _, _ = oracle_layer(oracle, layer, bits).forward(x, layer.router_w, threads=32)
    assert_output_close(_to_f32(y2), ref)
    dev.check_device_error()
    dev.close()
