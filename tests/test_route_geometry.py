"""Host logic of the router's launch geometry (pw_route_geometry; no GPU
needed): for many shapes, the blocks of every cluster cover each (token,
expert) logit exactly once, every staged row and column read stays inside
the block's shared-memory buffers, each warp has at most one register tile,
the logits and the staged selections fit where the kernel puts them, and the
dynamic shared memory fits one B200 block.  The index arithmetic below is
the route kernel's, restated."""
import itertools

import numpy as np
import pytest

SMEM_LIMIT = 232448          # bytes of dynamic shared memory one block may use
WARPS = 8


@pytest.fixture(scope="module")
def pw():
    from any_precision_weight_pw_b200 import binding, build
    build.build()
    return binding


def _check(g, T, E, H, k):
    assert 1 <= g["cb"] <= 8 and g["ce"] >= 1 and g["cb"] % g["ce"] == 0
    assert g["tt"] in (1, 2, 4, 8) and g["te"] in (1, 4, 8)
    assert g["kc"] % 32 == 0 and g["kc"] >= 32
    assert g["smem"] <= SMEM_LIMIT
    n_chunks = -(-H // g["kc"])
    xbytes = (g["tbb"] * g["kc"] * 2 + 15) & ~15
    sbytes = xbytes + g["eb"] * g["kc"] * 4
    # staging buffers (one, or two when the columns come in several chunks)
    # end before the logits, which end within the allocation
    assert (2 if n_chunks > 1 else 1) * sbytes <= g["logits_off"]
    assert g["logits_off"] + g["tb"] * E * 4 <= g["smem"]
    if g["sel_staged"]:
        assert ((T * k + 15) & ~15) + 4 * T * k <= g["logits_off"]
    tasks_e = -(-g["eb"] // g["te"])
    n_tasks = -(-g["tbb"] // g["tt"]) * tasks_e
    assert n_tasks <= WARPS
    n_clusters = g["n_clusters"]
    assert n_clusters == (max(1, -(-T // g["tb"])))
    seen = np.zeros((T, E), dtype=np.int32)
    shift = 5 - int(np.log2(g["tt"] * g["te"]))
    for blk in range(n_clusters * g["cb"]):
        rank = blk % g["cb"]
        tc0 = blk // g["cb"] * g["tb"]
        tl0 = (rank // g["ce"]) * g["tbb"]
        t0 = tc0 + tl0
        e0 = (rank % g["ce"]) * g["eb"]
        nt = min(g["tbb"], g["tb"] - tl0, T - t0)
        ne = min(g["eb"], E - e0)
        for ci in range(n_chunks):          # staged rows and columns are in bounds
            k0 = ci * g["kc"]
            kc = min(g["kc"], H - k0)
            assert 0 < kc <= g["kc"]
            if nt > 0:
                assert (t0 + nt - 1) * H + k0 + kc <= T * H
            if ne > 0:
                assert (e0 + ne - 1) * H + k0 + kc <= E * H
        for warp in range(n_tasks):
            tt0 = (warp // tasks_e) * g["tt"]
            te0 = (warp % tasks_e) * g["te"]
            for lane in range(0, 32, 1 << shift):
                a = lane >> shift
                tl, el = tt0 + a // g["te"], te0 + a % g["te"]
                if tl < nt and el < ne:
                    seen[t0 + tl, e0 + el] += 1
                    assert (tl0 + tl) * E + e0 + el < g["tb"] * E
    assert (seen == 1).all()


SHAPES = [(T, E, H) for T, E, H in itertools.product(
    (0, 1, 2, 5, 8, 16, 17, 32, 64, 255, 256, 300, 1024, 4096),
    (1, 3, 8, 9, 60, 64, 128),
    (7, 100, 2048, 4096, 7168))]


@pytest.mark.parametrize("T,E,H", SHAPES)
def test_router_geometry_covers_every_logit_once(pw, T, E, H):
    k = min(E, 2 if E < 60 else 4)
    _check(pw.route_geometry(T, E, H, k), T, E, H, k)


def test_router_geometry_headline_shapes(pw):
    """The decode and prefill shapes of the benchmark workloads take the
    geometries the design describes."""
    g = pw.route_geometry(16, 8, 4096, 2)     # 16 Mixtral-shaped tokens
    assert (g["cb"], g["ce"], g["tbb"], g["eb"], g["n_clusters"]) == (8, 4, 8, 2, 1)
    g = pw.route_geometry(1, 60, 2048, 4)     # 1 Qwen-shaped token
    assert (g["cb"], g["ce"], g["tbb"], g["eb"]) == (8, 8, 1, 8)
    g = pw.route_geometry(4096, 8, 4096, 2)   # Mixtral-shaped prefill
    assert (g["cb"], g["tb"], g["tt"], g["te"], g["n_clusters"]) == (1, 32, 4, 8, 128)


def test_router_geometry_rejects_bad_shapes(pw):
    for args in ((-1, 8, 64, 2), (4, 0, 64, 1), (4, 129, 64, 2), (4, 8, 0, 2), (4, 8, 64, 9),
                 (4, 2, 64, 3)):
        with pytest.raises(pw.PwError):
            pw.route_geometry(*args)
