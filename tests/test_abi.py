"""The C ABI library loads, exports every function include/pw.h declares, and
rejects bad arguments on the host (no GPU needed for any of this)."""
import ctypes as C
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def pwlib():
    from any_precision_weight_pw_b200 import build, binding
    build.build()
    return binding


def declared_functions():
    src = open(os.path.join(ROOT, "include", "pw.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(pw_[a-z_]+)\s*\(", src)))


def test_every_declared_symbol_is_exported(pwlib):
    names = declared_functions()
    assert "pw_moe_create" in names and "pw_moe_forward" in names
    L = pwlib.lib()
    for n in names:
        assert hasattr(L, n), n
    assert sorted(pwlib.EXPORTED) == names


def test_abi_version(pwlib):
    assert pwlib.lib().pw_abi_version() == 1


def _cfg(pwlib, **kw):
    base = dict(hidden=256, ffn=512, n_experts=8, top_k=2, shared_ffn=0, n_max=8,
                renorm_topk=1, max_tokens=16)
    base.update(kw)
    return pwlib.Config(*[base[f] for f, _ in pwlib.Config._fields_])


@pytest.mark.parametrize("bad", [dict(hidden=100), dict(n_experts=0), dict(n_experts=129),
                                 dict(top_k=9), dict(top_k=0), dict(n_max=9), dict(max_tokens=0),
                                 dict(shared_ffn=-1)])
def test_create_rejects_bad_config(pwlib, bad):
    L = pwlib.lib()
    c = _cfg(pwlib, **bad)
    descs = (pwlib.BlockDesc * 24)()
    h = C.c_void_p()
    assert L.pw_moe_create(C.byref(c), descs, 24, C.byref(h)) == 1
    assert h.value is None
    assert L.pw_last_error()


def test_create_rejects_bad_blocks(pwlib):
    L = pwlib.lib()
    c = _cfg(pwlib)
    h = C.c_void_p()
    descs = (pwlib.BlockDesc * 24)()
    assert L.pw_moe_create(C.byref(c), descs, 23, C.byref(h)) == 1   # count
    assert L.pw_moe_create(C.byref(c), descs, 24, C.byref(h)) == 1   # null buffers
    for d in descs:
        d.d_planes, d.d_lut[0], d.d_lut[1], d.bits = 4096, 8192, 8200, 4
    assert L.pw_moe_create(C.byref(c), descs, 24, C.byref(h)) == 1   # misaligned LUT slot
    assert b"aligned" in L.pw_last_error()
    for d in descs:
        d.d_lut[1], d.bits = 8208, 9
    assert L.pw_moe_create(C.byref(c), descs, 24, C.byref(h)) == 1   # bits > n_max
    assert L.pw_moe_create(None, descs, 24, C.byref(h)) == 1


def test_null_handle_calls(pwlib):
    L = pwlib.lib()
    assert L.pw_destroy(None) == 0
    assert L.pw_set_block_bits(None, 0, 4, None) == 1
    assert L.pw_moe_forward(None, None, 1, None, None, None, None) == 1
    assert L.pw_moe_forward_host(None, None, 1, None, None, None, None) == 1
    assert L.pw_get_routing(None, None, None, None) == 1
    assert L.pw_check_device_error(None) == 1
    assert L.pw_forward_launches(None, 4) == 0
    assert L.pw_profile_enable(None, 1) == 1
    assert L.pw_profile_read(None, None, 4, None) == 1
    n, p = C.c_int32(), C.c_int32()
    assert L.pw_get_block_bits(None, 0, C.byref(n), C.byref(p)) == 1


def test_linear_rejects_bad_args(pwlib):
    L = pwlib.lib()
    assert L.pw_linear(4096, 4096, 0, 32, 8, 4, 4096, 1, 4096, None) == 1      # rows
    assert L.pw_linear(4096, 4096, 8, 32, 8, 9, 4096, 1, 4096, None) == 1      # bits > n_max
    assert L.pw_linear(4096, 4096, 8, 32, 3, 4, 4096, 1, 4096, None) == 1      # bits > n_max
    assert L.pw_linear(None, 4096, 8, 32, 8, 4, 4096, 1, 4096, None) == 1      # null planes
    assert L.pw_linear(4100, 4096, 8, 32, 8, 4, 4096, 1, 4096, None) == 1      # misaligned
    assert L.pw_linear(4096, 4096, 8, 32, 8, 4, None, 0, None, None) == 0      # T = 0: nothing to do
    assert L.pw_repack_planes(None, 4096, 8, 32, 1, None) == 1
    assert L.pw_repack_planes(4096, 4096, 8, 32, 9, None) == 1
    # pw_route_static: limits are checked before anything touches a device
    assert L.pw_route_static(4096, 4096, None, 257, 64, 8, 2, 1, 4096, 4096, None) == 1  # T > 256
    assert L.pw_route_static(4096, 4096, None, -1, 64, 8, 2, 1, 4096, 4096, None) == 1   # T < 0
    assert L.pw_route_static(4096, 4096, None, 4, 64, 129, 2, 1, 4096, 4096, None) == 1  # E > 128
    assert L.pw_route_static(4096, 4096, None, 4, 64, 4, 5, 1, 4096, 4096, None) == 1    # k > E
    assert L.pw_route_static(4096, 4096, None, 4, 64, 60, 9, 0, 4096, 4096, None) == 1   # k > 8
    assert L.pw_route_static(4096, 4096, None, 4, 64, 8, 2, 2, 4096, 4096, None) == 1    # renorm
    assert L.pw_route_static(4096, 4096, None, 4, 0, 8, 2, 1, 4096, 4096, None) == 1     # hidden
    assert L.pw_route_static(None, None, None, 0, 64, 8, 2, 1, None, None, None) == 0    # T = 0


def test_plane_bytes(pwlib):
    L = pwlib.lib()
    # 128 rows x 8 words per 4 KB tile
    assert L.pw_plane_bytes(128, 256) == 4096
    assert L.pw_plane_bytes(129, 256) == 8192
    assert L.pw_plane_bytes(128, 257) == 8192
    assert L.pw_plane_bytes(14336, 4096) == 14336 * 4096 // 8
    assert L.pw_plane_bytes(0, 32) == 0
