"""pw_route_static (routing with its scratch in a fixed device array, no
allocation) against the routing pw_moe_forward reports through
pw_get_routing on the same inputs, and against the oracle's top-k.

Collected last (file name) so it also runs after every other GPU test has
used the device; it passes on its own as well.
"""
import numpy as np
import pytest

from any_precision_weight_pw_b200 import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def pw():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from any_precision_weight_pw_b200 import binding, build
    build.build()
    return binding


def _forward_routing(pw, layer, dev, x, wr, bias):
    dev.forward(x, wr, bias)
    return dev.routing(x.shape[0])


@pytest.mark.parametrize("name,T1,T2", [
    ("tiny_h256_f512_e8k2", 37, 256),         # max token count on the second call
    ("tiny_h256_f512_e8k2", 1, 1),
    ("qwen15_moe_a27b", 32, 7),               # E = 60, k = 4, no renormalisation
    ("mixtral_8x7b_prefill", 256, 19),        # router bias (skewed expert popularity)
])
def test_two_calls_match_forward_routing(pw, oracle, name, T1, T2):
    wl = synth.WORKLOADS[name]
    layer = synth.Layer(wl, seed=3)
    dev = pw.upload_synth_layer(layer, max_tokens=max(T1, T2))
    wr = torch.from_numpy(layer.router_w).cuda()
    bias = None if layer.router_bias is None else torch.from_numpy(layer.router_bias).cuda()
    xs_h = [synth.tokens(wl, T1, seed=3, batch=0), synth.tokens(wl, T2, seed=3, batch=1)]
    xs = [torch.from_numpy(x.view(np.int16)).cuda() for x in xs_h]

    # the existing entry point: one forward per batch, routing read back
    ref = []
    for x in xs:
        i, w = _forward_routing(pw, layer, dev, x, wr, bias)
        ref.append((i.clone(), w.clone()))
    torch.cuda.synchronize()

    # two calls in a row on the same stream, no synchronisation between them
    outs = [pw.route_static(x, wr, wl.top_k, wl.renorm_topk, router_bias=bias) for x in xs]
    torch.cuda.synchronize()
    for (i, w), (ri, rw), xh in zip(outs, ref, xs_h):
        assert torch.equal(i, ri)
        assert torch.equal(w, rw)          # same kernel, same order: bit-identical
        oi, ow = oracle.topk_softmax(oracle.router_logits(xh, layer.router_w, layer.router_bias),
                                     wl.top_k, bool(wl.renorm_topk))
        np.testing.assert_array_equal(i.cpu().numpy(), oi)
        np.testing.assert_allclose(w.cpu().numpy(), ow, rtol=1e-5, atol=1e-7)
    dev.close()


def test_repeat_calls_reuse_scratch_without_allocating(pw):
    wl = synth.WORKLOADS["tiny_h256_f512_e8k2"]
    layer = synth.Layer(wl, seed=4)
    wr = torch.from_numpy(layer.router_w).cuda()
    x = torch.from_numpy(synth.tokens(wl, 64, seed=4).view(np.int16)).cuda()
    idx = torch.empty((64, wl.top_k), dtype=torch.int32, device="cuda")
    w = torch.empty((64, wl.top_k), dtype=torch.float32, device="cuda")
    pw.route_static(x, wr, wl.top_k, wl.renorm_topk, idx=idx, w=w)  # first call: set-up
    torch.cuda.synchronize()
    first = (idx.clone(), w.clone())
    free0 = torch.cuda.mem_get_info()[0]
    for _ in range(3):
        pw.route_static(x, wr, wl.top_k, wl.renorm_topk, idx=idx, w=w)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    assert torch.equal(idx, first[0]) and torch.equal(w, first[1])


def test_rejects_more_tokens_than_the_scratch_holds(pw):
    wl = synth.WORKLOADS["tiny_h256_f512_e8k2"]
    layer = synth.Layer(wl, seed=5)
    wr = torch.from_numpy(layer.router_w).cuda()
    x = torch.zeros((257, wl.hidden), dtype=torch.int16, device="cuda")
    with pytest.raises(pw.PwError):
        pw.route_static(x, wr, wl.top_k, wl.renorm_topk)


@pytest.mark.parametrize("T,E,H,k,bias", [
    (1, 9, 100, 2, False),      # hidden not a multiple of 8: plain staging loads
    (5, 7, 7, 3, True),         # hidden below one 32-column step
    (17, 1, 64, 1, False),      # one expert
    (33, 100, 264, 4, True),    # 13 experts per block, several clusters
    (200, 3, 40, 2, False),     # three single-expert blocks, 13 clusters
    (256, 60, 2048, 4, False),  # prefill geometry: 32-token clusters, 4 x 8 tiles
    (256, 128, 520, 8, True),   # 128 experts, 16 per block, several column chunks
])
def test_route_geometries_match_oracle(pw, oracle, T, E, H, k, bias):
    """Every launch geometry of the router (cluster size, tokens per cluster,
    register tile, column chunks, plain or 16-byte staging) gives the oracle's
    selections exactly; rows of zeros make every logit tie (lower index wins)."""
    rng = np.random.default_rng(T * 1000 + E)
    xf = rng.standard_normal((T, H)).astype(np.float32)
    xf[::4] = 0.0
    x_h = (xf.view(np.uint32) >> 16).astype(np.uint16)   # bf16 by truncation
    wr_h = (rng.standard_normal((E, H)) / np.sqrt(H)).astype(np.float32)
    b_h = (0.5 * rng.standard_normal(E)).astype(np.float32) if bias else None
    x = torch.from_numpy(x_h.view(np.int16)).cuda()
    wr = torch.from_numpy(wr_h).cuda()
    b = None if b_h is None else torch.from_numpy(b_h).cuda()
    i, w = pw.route_static(x, wr, k, 1, router_bias=b)
    torch.cuda.synchronize()
    oi, ow = oracle.topk_softmax(oracle.router_logits(x_h, wr_h, b_h), k, True)
    np.testing.assert_array_equal(i.cpu().numpy(), oi)
    np.testing.assert_allclose(w.cpu().numpy(), ow, rtol=1e-5, atol=1e-7)
