"""Thin ctypes binding of the C ABI in include/pw.h.

Argument marshalling only: every step of the layer runs in the CUDA library
``libpw_b200.so`` (built by ``any_precision_weight_pw_b200.build``).  PyTorch
supplies device memory, pinned host memory and streams.  There is no CPU or
PyTorch fallback: if the library is missing, loading raises.
"""
from __future__ import annotations

import ctypes as C
import os
from typing import List, Optional, Sequence

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libpw_b200.so")

PW_MAX_BITS = 8
STATUS = {0: "PW_OK", 1: "PW_ERR_INVALID_ARG", 2: "PW_ERR_CUDA", 3: "PW_ERR_OOM",
          4: "PW_ERR_TIMEOUT", 5: "PW_ERR_STATE", 6: "PW_ERR_UNSUPPORTED"}
EXPORTED = ["pw_moe_create", "pw_set_block_bits", "pw_moe_forward", "pw_destroy",
            "pw_moe_forward_host", "pw_linear", "pw_get_block_bits", "pw_get_routing",
            "pw_check_device_error", "pw_profile_enable", "pw_profile_read",
            "pw_forward_launches", "pw_plane_bytes", "pw_repack_planes", "pw_route_static",
            "pw_get_forward_bits", "pw_set_switch_lag", "pw_routing_stats", "pw_plan_release",
            "pw_enable_paging", "pw_resident_bytes", "pw_workspace_bytes", "pw_compact_pages",
            "pw_last_error", "pw_abi_version", "pw_route_geometry"]


class PwError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__("%s: %s" % (STATUS.get(status, status), message))
        self.status = status


class Config(C.Structure):
    _fields_ = [("hidden", C.c_int32), ("ffn", C.c_int32), ("n_experts", C.c_int32),
                ("top_k", C.c_int32), ("shared_ffn", C.c_int32), ("n_max", C.c_int32),
                ("renorm_topk", C.c_int32), ("max_tokens", C.c_int32)]


class PlanBlock(C.Structure):
    _fields_ = [("bits", C.c_int32), ("min_bits", C.c_int32), ("plane_bytes", C.c_int64),
                ("rows", C.c_int32), ("mass", C.c_double), ("resid", C.c_double),
                ("sens", C.c_double * (PW_MAX_BITS + 1))]


class BlockDesc(C.Structure):
    _fields_ = [("d_planes", C.c_void_p), ("d_lut", C.c_void_p * 2), ("h_planes", C.c_void_p),
                ("h_lut", C.c_void_p * (PW_MAX_BITS + 1)), ("bits", C.c_int32)]


_lib = None


def lib():
    """Load libpw_b200.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("libpw_b200.so is missing; build it with "
                               "any_precision_weight_pw_b200.build.build()")
        L = C.CDLL(LIB_PATH)
        P, i32 = C.c_void_p, C.c_int32
        L.pw_moe_create.argtypes = [C.POINTER(Config), C.POINTER(BlockDesc), i32, C.POINTER(P)]
        L.pw_set_block_bits.argtypes = [P, i32, i32, P]
        L.pw_moe_forward.argtypes = [P, P, i32, P, P, P, P]
        L.pw_destroy.argtypes = [P]
        L.pw_moe_forward_host.argtypes = [P, P, i32, P, P, P, P]
        L.pw_linear.argtypes = [P, P, i32, i32, i32, i32, P, i32, P, P]
        L.pw_get_block_bits.argtypes = [P, i32, C.POINTER(i32), C.POINTER(i32)]
        L.pw_get_forward_bits.argtypes = [P, C.POINTER(i32), i32]
        L.pw_set_switch_lag.argtypes = [P, i32]
        L.pw_routing_stats.argtypes = [P, P, P, i32, P]
        L.pw_enable_paging.argtypes = [P, P]
        L.pw_compact_pages.argtypes = [P, P]
        L.pw_workspace_bytes.argtypes = [C.POINTER(Config), C.POINTER(C.c_int64)]
        L.pw_resident_bytes.argtypes = [P, C.POINTER(C.c_int64), C.POINTER(C.c_int64)]
        L.pw_plan_release.argtypes = [C.POINTER(PlanBlock), i32, C.c_int64, C.POINTER(i32),
                                      C.POINTER(C.c_int64), C.POINTER(C.c_double),
                                      C.POINTER(i32)]
        L.pw_get_routing.argtypes = [P, P, P, P]
        L.pw_check_device_error.argtypes = [P]
        L.pw_profile_enable.argtypes = [P, i32]
        L.pw_profile_read.argtypes = [P, C.POINTER(C.c_float), i32, C.POINTER(i32)]
        L.pw_forward_launches.argtypes = [P, i32]
        L.pw_forward_launches.restype = i32
        L.pw_plane_bytes.argtypes = [i32, i32]
        L.pw_plane_bytes.restype = C.c_int64
        L.pw_repack_planes.argtypes = [P, P, i32, i32, i32, P]
        L.pw_route_static.argtypes = [P, P, P, i32, i32, i32, i32, i32, P, P, P]
        L.pw_route_geometry.argtypes = [i32, i32, i32, i32, C.POINTER(C.c_int64)]
        L.pw_last_error.restype = C.c_char_p
        L.pw_abi_version.restype = i32
        for name in EXPORTED:
            if name not in ("pw_forward_launches", "pw_last_error", "pw_abi_version",
                            "pw_plane_bytes"):
                getattr(L, name).restype = C.c_int
        _lib = L
    return _lib


def check(status: int) -> None:
    if status != 0:
        raise PwError(status, lib().pw_last_error().decode())


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> Optional[int]:
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def plane_bytes(rows: int, cols: int) -> int:
    """Bytes of one plane page of a rows x cols block."""
    return int(lib().pw_plane_bytes(rows, cols))


def repack_planes(planes, cols: int, stream=None):
    """Row-major planes (int32 device tensor [n][rows][ceil(cols/32)], uint32
    bit patterns) -> the paged layout of an n-plane block (flat int32 device
    tensor of n * plane_bytes / 4 words)."""
    import torch
    n, rows, _ = planes.shape
    out = torch.empty(n * plane_bytes(rows, cols) // 4, dtype=torch.int32, device=planes.device)
    check(lib().pw_repack_planes(_ptr(planes), _ptr(out), rows, cols, n, _stream(stream)))
    return out


def linear(planes, lut, bits: int, x, rows: int, y=None, stream=None):
    """y[t][o] = sum_i W_b[o][i] x[t][i] for one block.  planes: a block in
    the paged layout (repack_planes; its plane count follows from its size);
    lut: int16 [rows][2^bits] (fp16 bit patterns); x: bf16 [T][cols].
    Returns fp32 [T][rows]."""
    import torch
    T, cols = x.shape
    n_max = planes.numel() * 4 // plane_bytes(rows, cols)
    if y is None:
        y = torch.empty((T, rows), dtype=torch.float32, device=x.device)
    check(lib().pw_linear(_ptr(planes), _ptr(lut), rows, cols, n_max, bits, _ptr(x), T, _ptr(y),
                          _stream(stream)))
    return y


def route_static(x, router_w, top_k: int, renorm_topk: int, router_bias=None, idx=None, w=None,
                 stream=None):
    """Routing alone through pw_route_static (no device allocation inside
    the library): x bf16 [T][H], router_w fp32 [E][H] -> (idx int32 [T][k],
    w fp32 [T][k]).  Pass idx / w to reuse output buffers."""
    import torch
    T, H = x.shape
    E = router_w.shape[0]
    if idx is None:
        idx = torch.empty((T, top_k), dtype=torch.int32, device=x.device)
    if w is None:
        w = torch.empty((T, top_k), dtype=torch.float32, device=x.device)
    check(lib().pw_route_static(_ptr(x), _ptr(router_w), _ptr(router_bias), T, H, E, top_k,
                                renorm_topk, _ptr(idx), _ptr(w), _stream(stream)))
    return idx, w


def route_geometry(T: int, E: int, H: int, top_k: int) -> dict:
    """The route kernel's launch geometry for a shape (host arithmetic)."""
    out = (C.c_int64 * 12)()
    check(lib().pw_route_geometry(T, E, H, top_k, out))
    keys = ("cb", "ce", "tb", "tbb", "eb", "kc", "n_clusters", "tt", "te", "sel_staged",
            "logits_off", "smem")
    return dict(zip(keys, list(out)))


def workspace_bytes(cfg: dict) -> int:
    """Device workspace bytes a layer with this config allocates."""
    c = Config(cfg["hidden"], cfg["ffn"], cfg["n_experts"], cfg["top_k"], cfg["shared_ffn"],
               cfg["n_max"], cfg["renorm_topk"], cfg["max_tokens"])
    out = C.c_int64()
    check(lib().pw_workspace_bytes(C.byref(c), C.byref(out)))
    return out.value


def plan_release(blocks, target_bytes: int):
    """Greedy release plan through pw_plan_release.  blocks: dicts with bits,
    min_bits, plane_bytes, rows, mass, resid, sens (sens[b] for b = 0..8).
    Returns {"bits", "released", "damage", "reached"}."""
    n = len(blocks)
    arr = (PlanBlock * max(n, 1))()
    for j, b in enumerate(blocks):
        arr[j].bits, arr[j].min_bits = int(b["bits"]), int(b["min_bits"])
        arr[j].plane_bytes, arr[j].rows = int(b["plane_bytes"]), int(b["rows"])
        arr[j].mass, arr[j].resid = float(b["mass"]), float(b.get("resid", 0.0))
        for k in range(PW_MAX_BITS + 1):
            arr[j].sens[k] = float(b["sens"][k]) if k < len(b["sens"]) else 0.0
    bits = (C.c_int32 * max(n, 1))()
    rel, dmg, reached = C.c_int64(), C.c_double(), C.c_int32()
    check(lib().pw_plan_release(arr, n, int(target_bytes), bits, C.byref(rel), C.byref(dmg),
                                C.byref(reached)))
    return {"bits": list(bits)[:n], "released": rel.value, "damage": dmg.value,
            "reached": bool(reached.value)}


class MoELayer:
    """A layer over device-resident pages (torch tensors kept alive here)."""

    def __init__(self, cfg: dict, planes: Sequence, lut_slots: Sequence, bits: Sequence[int],
                 host_planes: Optional[Sequence] = None, host_luts: Optional[Sequence] = None):
        self.cfg = dict(cfg)
        self._keep: List = [planes, lut_slots, host_planes, host_luts]
        c = Config(cfg["hidden"], cfg["ffn"], cfg["n_experts"], cfg["top_k"], cfg["shared_ffn"],
                   cfg["n_max"], cfg["renorm_topk"], cfg["max_tokens"])
        n = len(planes)
        descs = (BlockDesc * n)()
        for j in range(n):
            d = descs[j]
            d.d_planes = _ptr(planes[j])
            d.d_lut[0] = _ptr(lut_slots[j][0])
            d.d_lut[1] = _ptr(lut_slots[j][1])
            d.h_planes = _ptr(host_planes[j]) if host_planes else None
            if host_luts:
                for b, t in host_luts[j].items():
                    d.h_lut[b] = _ptr(t)
            d.bits = int(bits[j])
        h = C.c_void_p()
        check(lib().pw_moe_create(C.byref(c), descs, n, C.byref(h)))
        self.h = h
        self.n_blocks = n

    def forward(self, x, router_w, bias=None, y=None, stream=None):
        import torch
        T = x.shape[0]
        if y is None:
            y = torch.empty_like(x)
        check(lib().pw_moe_forward(self.h, _ptr(x), T, _ptr(router_w), _ptr(bias), _ptr(y),
                                   _stream(stream)))
        return y

    def forward_host(self, x_host, router_w, bias=None, y_host=None, stream=None):
        """x_host: pinned CPU int16/bf16 tensor [T][H]; returns the host output."""
        import torch
        if y_host is None:
            y_host = torch.empty_like(x_host).pin_memory()
        check(lib().pw_moe_forward_host(self.h, _ptr(x_host), x_host.shape[0], _ptr(router_w),
                                        _ptr(bias), _ptr(y_host), _stream(stream)))
        return y_host

    def set_block_bits(self, block: int, bits: int, side_stream) -> None:
        check(lib().pw_set_block_bits(self.h, block, bits, side_stream.cuda_stream))

    def get_block_bits(self, block: int):
        """(bitwidth as of the last issued forward, pending width or 0)."""
        cur, pend = C.c_int32(), C.c_int32()
        check(lib().pw_get_block_bits(self.h, block, C.byref(cur), C.byref(pend)))
        return cur.value, pend.value

    def forward_bits(self) -> List[int]:
        """Bitwidth of every block in the most recently issued forward."""
        out = (C.c_int32 * self.n_blocks)()
        check(lib().pw_get_forward_bits(self.h, out, self.n_blocks))
        return list(out)

    def set_switch_lag(self, max_lag: int) -> None:
        check(lib().pw_set_switch_lag(self.h, max_lag))

    def routing(self, T: int, stream=None):
        import torch
        k = self.cfg["top_k"]
        idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
        w = torch.empty((T, k), dtype=torch.float32, device="cuda")
        check(lib().pw_get_routing(self.h, _ptr(idx), _ptr(w), _stream(stream)))
        return idx, w

    def enable_paging(self, stream=None) -> None:
        """Library-owned plane storage holding only each block's resident
        planes (the caller's plane buffers may be freed afterwards)."""
        check(lib().pw_enable_paging(self.h, _stream(stream)))

    def compact_pages(self, stream=None) -> None:
        """Pack the resident planes into one allocation (on the forward stream)."""
        check(lib().pw_compact_pages(self.h, _stream(stream)))

    def resident_bytes(self, trim: bool = False):
        """(plane bytes resident, pool bytes reserved after a trim or None)."""
        pb, pr = C.c_int64(), C.c_int64()
        check(lib().pw_resident_bytes(self.h, C.byref(pb), C.byref(pr) if trim else None))
        return pb.value, (pr.value if trim else None)

    def routing_stats(self, reset: bool = False, stream=None):
        """(counts uint64 [E], mass float64 [E]) accumulated over forwards."""
        E = self.cfg["n_experts"]
        counts = np.zeros(E, dtype=np.uint64)
        mass = np.zeros(E, dtype=np.float64)
        check(lib().pw_routing_stats(self.h, counts.ctypes.data, mass.ctypes.data,
                                     1 if reset else 0, _stream(stream)))
        return counts, mass

    def check_device_error(self) -> None:
        check(lib().pw_check_device_error(self.h))

    def profile(self, on: bool) -> None:
        check(lib().pw_profile_enable(self.h, 1 if on else 0))

    def profile_read(self):
        """(ms per launch slot summed since the last read, forwards summed)."""
        ms = (C.c_float * 4)()
        n = C.c_int32()
        check(lib().pw_profile_read(self.h, ms, 4, C.byref(n)))
        return list(ms), n.value

    def launches(self, T: int) -> int:
        return int(lib().pw_forward_launches(self.h, T))

    def close(self) -> None:
        if getattr(self, "h", None):
            check(lib().pw_destroy(self.h))
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def upload_synth_layer(layer, max_tokens: int, host_copies: bool = False,
                       device: str = "cuda", host_planes: bool = True) -> MoELayer:
    """Put a synth.Layer's pages on the device and create the library layer.
    With host_copies, pinned master copies of every LUT width, and of all
    planes unless host_planes is False, are kept for bitwidth switches."""
    import torch
    wl = layer.wl
    planes, slots, hp, hl = [], [], [], []
    for blk in range(wl.n_blocks):
        rows, cols = layer.shape(blk)
        pl = layer.planes(blk)
        paged = repack_planes(torch.from_numpy(pl.view(np.int32)).to(device), cols)
        planes.append(paged)
        s0 = torch.zeros(rows << wl.n_max, dtype=torch.int16, device=device)
        s1 = torch.zeros(rows << wl.n_max, dtype=torch.int16, device=device)
        lt = layer.lut(blk, layer.bits[blk])
        s0[: lt.size].copy_(torch.from_numpy(lt.reshape(-1).view(np.int16)))
        slots.append((s0, s1))
        if host_copies and host_planes:
            hp.append(paged.cpu().pin_memory())
        if host_copies:
            hl.append({b: torch.from_numpy(layer.lut(blk, b).reshape(-1).view(np.int16)).pin_memory()
                       for b in range(1, wl.n_max + 1)})
    cfg = dict(hidden=wl.hidden, ffn=wl.ffn, n_experts=wl.n_experts, top_k=wl.top_k,
               shared_ffn=wl.shared_ffn, n_max=wl.n_max, renorm_topk=wl.renorm_topk,
               max_tokens=max_tokens)
    return MoELayer(cfg, planes, slots, layer.bits, hp or None, hl or None)
