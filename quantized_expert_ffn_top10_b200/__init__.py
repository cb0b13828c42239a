"""Python binding of libmoe.so (include/moe.h): argument marshalling only.

Every step of the layer runs in the library's CUDA kernels; this module turns
torch tensors into pointers and sizes and raises on a non-zero return code.
There is no fallback: if libmoe.so is missing or fails to load, import fails.
"""
from __future__ import annotations

import ctypes
import os



class ArenaDesc(ctypes.Structure):
    """moe_arena_desc of include/moe.h."""
    _fields_ = [("H", ctypes.c_int32), ("I", ctypes.c_int32), ("block", ctypes.c_int32),
                ("bits_gate", ctypes.c_int32), ("bits_up", ctypes.c_int32), ("bits_down", ctypes.c_int32),
                ("slot_bytes", ctypes.c_int64), ("off_codes", ctypes.c_int64 * 3),
                ("off_scales", ctypes.c_int64 * 3), ("n_slots", ctypes.c_int32), ("reserved", ctypes.c_int32)]


def as_desc(d) -> ArenaDesc:
    """Copy any object with the descriptor's field names into an ArenaDesc."""
    if isinstance(d, ArenaDesc):
        return d
    o = ArenaDesc()
    for name, _ in ArenaDesc._fields_:
        v = getattr(d, name)
        if name in ("off_codes", "off_scales"):
            for i in range(3):
                getattr(o, name)[i] = v[i]
        else:
            setattr(o, name, v)
    return o

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe.so")

MOE_OK, MOE_ERR_ARG, MOE_ERR_SHAPE, MOE_ERR_RANGE = 0, -1, -2, -3
MOE_ERR_WS, MOE_ERR_CUDA, MOE_ERR_SLOT, MOE_ERR_TIMEOUT = -4, -5, -6, -7
MOE_ERR_STATIC = -8
MOE_DECODE_MAX_T, MOE_PREFILL_MAX_T, MOE_ROUTER_F64_MAX_T = 8, 8192, 128
MOE_ROUTE_STATIC_MAX_T, MOE_ROUTE_STATIC_BYTES = 8, 128 * 1024

EXPORTS = ("moe_workspace_bytes", "moe_route", "moe_forward_decode", "moe_forward_prefill",
           "moe_route_histogram", "moe_rank_experts", "moe_last_device_error", "moe_strerror",
           "moe_set_stage_events", "moe_launch_count", "moe_timeout_site", "moe_route_static",
           "moe_debug_set", "moe_workspace_offset", "moe_router_gamma", "moe_profile_bytes",
           "moe_profile_write", "moe_profile_read", "moe_profile_hit_rate", "moe_forward_partial",
           "moe_finish_rows")
MOE_SLOT_REMOTE = -2
MOE_DBG_SPIN_LIMIT, MOE_DBG_BARRIER_EXTRA = 1, 2
MOE_WS_FAST_LOGITS, MOE_WS_PAIR_OUT, MOE_WS_SLOW_COUNT = 1, 2, 3


class RouteOut(ctypes.Structure):
    _fields_ = [("topk_idx", ctypes.c_void_p), ("topk_w", ctypes.c_void_p),
                ("expert_offsets", ctypes.c_void_p), ("perm", ctypes.c_void_p),
                ("n_rechecked", ctypes.c_void_p)]


class MoeError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__(f"{where}: {code} ({strerror(code)})")
        self.code = code


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libmoe.so not built at {LIB_PATH}; run quantized_expert_ffn_top10_b200.build.build()")
        L = ctypes.CDLL(LIB_PATH)
        P, i32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        L.moe_workspace_bytes.restype = sz
        L.moe_workspace_bytes.argtypes = [i32, i32, i32, i32, i32]
        L.moe_route.restype = i32
        L.moe_route.argtypes = [P, i32, i32, P, P, i32, i32, P, P, P, P, P, sz, P]
        fwd = [P, P, P, i32, i32, P, i32, P, P, i32, i32, i32, P, P, P, P, P, sz, P]
        L.moe_forward_decode.restype = i32
        L.moe_forward_decode.argtypes = fwd
        L.moe_forward_prefill.restype = i32
        L.moe_forward_prefill.argtypes = fwd
        L.moe_forward_partial.restype = i32
        L.moe_forward_partial.argtypes = [i32, P, P, P, i32, i32, P, i32, P, P, i32, i32, P, P, P, P,
                                          ctypes.c_size_t, P]
        L.moe_finish_rows.restype = i32
        L.moe_finish_rows.argtypes = [P, P, i32, i32, i32, P, P, P]
        L.moe_route_histogram.restype = i32
        L.moe_route_histogram.argtypes = [P, i32, i32, i32, P, P]
        L.moe_rank_experts.restype = i32
        L.moe_rank_experts.argtypes = [P, i32, i32, P]
        L.moe_last_device_error.restype = i32
        L.moe_last_device_error.argtypes = [P]
        L.moe_strerror.restype = ctypes.c_char_p
        L.moe_strerror.argtypes = [i32]
        L.moe_set_stage_events.restype = i32
        L.moe_set_stage_events.argtypes = [P, i32]
        L.moe_launch_count.restype = ctypes.c_uint64
        L.moe_launch_count.argtypes = []
        L.moe_timeout_site.restype = i32
        L.moe_timeout_site.argtypes = [P]
        L.moe_route_static.restype = i32
        L.moe_route_static.argtypes = [P, i32, i32, P, P, i32, i32, P, P, P, P, P]
        L.moe_debug_set.restype = i32
        L.moe_debug_set.argtypes = [i32, i32]
        L.moe_workspace_offset.restype = sz
        L.moe_workspace_offset.argtypes = [i32, i32, i32, i32, i32, i32]
        L.moe_router_gamma.restype = ctypes.c_double
        L.moe_router_gamma.argtypes = [i32, i32, i32]
        L.moe_profile_bytes.restype = ctypes.c_int64
        L.moe_profile_bytes.argtypes = [i32, i32, i32]
        L.moe_profile_write.restype = ctypes.c_int64
        L.moe_profile_write.argtypes = [P, i32, i32, i32, P, sz]
        L.moe_profile_read.restype = i32
        L.moe_profile_read.argtypes = [P, sz, P, P, P, P, P]
        L.moe_profile_hit_rate.restype = ctypes.c_double
        L.moe_profile_hit_rate.argtypes = [P, i32, i32, i32, i32, P]
        _lib = L
    return _lib


def strerror(code: int) -> str:
    return lib().moe_strerror(int(code)).decode()


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return stream if isinstance(stream, int) else stream.cuda_stream


def _check(rc: int, where: str, raise_on_error: bool):
    if rc != MOE_OK and raise_on_error:
        raise MoeError(rc, where)
    return rc


def moe_workspace_bytes(T: int, E: int, top_k: int, H: int, I: int) -> int:
    return int(lib().moe_workspace_bytes(T, E, top_k, H, I))


def moe_route(x, router_w, router_bias, top_k, topk_idx, topk_w, expert_offsets, perm, ws,
              stream=None, raise_on_error=True) -> int:
    """x [T, H] bf16, router_w [E, H] fp32, router_bias [E] fp32 or None (CUDA tensors)."""
    T, H = x.shape
    E = router_w.shape[0]
    rc = lib().moe_route(_ptr(x), T, H, _ptr(router_w), _ptr(router_bias), E, top_k, _ptr(topk_idx),
                         _ptr(topk_w), _ptr(expert_offsets), _ptr(perm), _ptr(ws), ws.numel() * ws.element_size(),
                         _stream(stream))
    return _check(rc, "moe_route", raise_on_error)


def moe_route_static(x, router_w, router_bias, top_k, topk_idx, topk_w, expert_offsets, perm,
                     stream=None, raise_on_error=True) -> int:
    """moe_route with the library's fixed device scratch instead of a workspace
    (T <= MOE_ROUTE_STATIC_MAX_T).  Calls that overlap on the GPU race."""
    T, H = x.shape
    E = router_w.shape[0]
    rc = lib().moe_route_static(_ptr(x), T, H, _ptr(router_w), _ptr(router_bias), E, top_k, _ptr(topk_idx),
                                _ptr(topk_w), _ptr(expert_offsets), _ptr(perm), _stream(stream))
    return _check(rc, "moe_route_static", raise_on_error)


def _forward(fn, name, desc, arena, slot_table, L, layer, x, router_w, router_bias, top_k, residual, out,
             hist, route_out, ws, stream, raise_on_error, steer=None, T=None, E=None):
    T = x.shape[0] if T is None else T
    E = router_w.shape[0] if E is None else E
    ro = None
    if route_out is not None:
        ro = RouteOut(*[_ptr(route_out.get(k)) for k in ("topk_idx", "topk_w", "expert_offsets", "perm",
                                                          "n_rechecked")])
    rc = fn(ctypes.byref(as_desc(desc)), _ptr(arena), _ptr(slot_table), L, layer, _ptr(x), T, _ptr(router_w),
            _ptr(router_bias), E, top_k, int(bool(residual)), _ptr(steer), _ptr(out), _ptr(hist),
            ctypes.byref(ro) if ro is not None else None, _ptr(ws),
            ws.numel() * ws.element_size() if hasattr(ws, "numel") else 0, _stream(stream))
    return _check(rc, name, raise_on_error)


def moe_forward_decode(desc: ArenaDesc, arena, slot_table, L, layer, x, router_w, router_bias, top_k,
                       residual, out, hist=None, route_out=None, ws=None, stream=None, raise_on_error=True,
                       steer=None):
    """One MoE layer for a decode window (T <= 8).  route_out: optional dict of
    device tensors topk_idx / topk_w / expert_offsets / perm / n_rechecked;
    steer: optional fp32 [H] direction projected out of every output row."""
    return _forward(lib().moe_forward_decode, "moe_forward_decode", desc, arena, slot_table, L, layer, x,
                    router_w, router_bias, top_k, residual, out, hist, route_out, ws, stream, raise_on_error,
                    steer=steer)


def moe_forward_prefill(desc: ArenaDesc, arena, slot_table, L, layer, x, router_w, router_bias, top_k,
                        residual, out, hist=None, route_out=None, ws=None, stream=None, raise_on_error=True,
                        steer=None):
    """One MoE layer for a prefill chunk (T <= 8192), tensor-core grouped GEMMs."""
    return _forward(lib().moe_forward_prefill, "moe_forward_prefill", desc, arena, slot_table, L, layer, x,
                    router_w, router_bias, top_k, residual, out, hist, route_out, ws, stream, raise_on_error,
                    steer=steer)


def moe_forward_partial(prefill, desc: ArenaDesc, arena, slot_table, L, layer, x, router_w, router_bias, top_k,
                        partial, hist=None, route_out=None, ws=None, stream=None, raise_on_error=True):
    """Expert parallelism: partial [T, H] fp32 receives each token's gate-weighted
    sum over the experts held here (slot != MOE_SLOT_REMOTE), no residual."""
    T, E = x.shape[0], router_w.shape[0]
    ro = None
    if route_out is not None:
        ro = RouteOut(*[_ptr(route_out.get(k)) for k in ("topk_idx", "topk_w", "expert_offsets", "perm",
                                                          "n_rechecked")])
    rc = lib().moe_forward_partial(int(bool(prefill)), ctypes.byref(as_desc(desc)), _ptr(arena), _ptr(slot_table),
                                   L, layer, _ptr(x), T, _ptr(router_w), _ptr(router_bias), E, top_k, _ptr(partial),
                                   _ptr(hist), ctypes.byref(ro) if ro is not None else None, _ptr(ws),
                                   ws.numel() * ws.element_size() if hasattr(ws, "numel") else 0, _stream(stream))
    return _check(rc, "moe_forward_partial", raise_on_error)


def moe_finish_rows(x, total, residual, out, steer=None, stream=None, raise_on_error=True) -> int:
    """out = bf16((residual ? x : 0) + total), steering projection first when given."""
    T, H = total.shape
    rc = lib().moe_finish_rows(_ptr(x), _ptr(total), T, H, int(bool(residual)), _ptr(steer), _ptr(out),
                               _stream(stream))
    return _check(rc, "moe_finish_rows", raise_on_error)


def moe_route_histogram(expert_offsets, E, L, layer, hist, stream=None, raise_on_error=True) -> int:
    rc = lib().moe_route_histogram(_ptr(expert_offsets), E, L, layer, _ptr(hist), _stream(stream))
    return _check(rc, "moe_route_histogram", raise_on_error)


def moe_rank_experts(hist_host):
    """hist_host: numpy uint32 [L, E] -> numpy uint16 [L*E, 2] (layer, expert), most routed first."""
    import numpy as np
    h = np.ascontiguousarray(hist_host, dtype=np.uint32)
    L, E = h.shape
    pairs = np.zeros((L * E, 2), np.uint16)
    rc = lib().moe_rank_experts(h.ctypes.data_as(ctypes.c_void_p), L, E, pairs.ctypes.data_as(ctypes.c_void_p))
    _check(rc, "moe_rank_experts", True)
    return pairs


def moe_last_device_error(stream=None) -> int:
    return int(lib().moe_last_device_error(_stream(stream)))


def moe_set_stage_events(events) -> int:
    """events: list of 5 torch.cuda.Event(enable_timing=True) (or [] to turn off);
    later forward calls record them at the stage boundaries."""
    for e in events:
        if e.cuda_event == 0:
            e.record()  # make sure the event exists before its handle is taken
    n = len(events)
    arr = (ctypes.c_void_p * max(n, 1))(*[e.cuda_event for e in events])
    return _check(lib().moe_set_stage_events(arr if n else None, n), "moe_set_stage_events", True)


def moe_launch_count() -> int:
    return int(lib().moe_launch_count())


def moe_timeout_site(stream=None) -> int:
    return int(lib().moe_timeout_site(_stream(stream)))


def moe_debug_set(key: int, value: int) -> int:
    """Test hook: see include/moe.h (MOE_DBG_SPIN_LIMIT, MOE_DBG_BARRIER_EXTRA)."""
    return _check(lib().moe_debug_set(int(key), int(value)), "moe_debug_set", True)


def moe_workspace_offset(T: int, E: int, top_k: int, H: int, I: int, field: int) -> int:
    """Byte offset of a workspace field (MOE_WS_FAST_LOGITS, MOE_WS_PAIR_OUT)."""
    v = int(lib().moe_workspace_offset(T, E, top_k, H, I, field))
    if v == ctypes.c_size_t(-1).value:
        raise MoeError(MOE_ERR_ARG, "moe_workspace_offset")
    return v


def moe_router_gamma(T: int, E: int, H: int) -> float:
    """Bound factor of a chunk router's fast logits (include/moe.h)."""
    return float(lib().moe_router_gamma(T, E, H))


def moe_profile_write(pairs, L: int, E: int) -> bytes:
    """STRP v1 expert profile (include/moe.h) of the ranked (layer, expert)
    pairs (numpy uint16 [n, 2], rank order)."""
    import numpy as np
    pr = np.ascontiguousarray(pairs, dtype=np.uint16).reshape(-1, 2)
    n = pr.shape[0]
    size = int(lib().moe_profile_bytes(n, L, E))
    if size < 0:
        raise MoeError(MOE_ERR_RANGE, "moe_profile_bytes")
    buf = np.zeros(size, np.uint8)
    rc = int(lib().moe_profile_write(pr.ctypes.data_as(ctypes.c_void_p), n, L, E,
                                     buf.ctypes.data_as(ctypes.c_void_p), size))
    if rc < 0:
        raise MoeError(rc, "moe_profile_write")
    return buf.tobytes()


def moe_profile_read(data: bytes):
    """(L, E, pairs uint16 [n, 2], inverse int32 [L, E]) of an STRP v1 file."""
    import numpy as np
    raw = np.frombuffer(data, np.uint8).copy()
    Lc, Ec, nc = ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
    P = ctypes.c_void_p
    rc = lib().moe_profile_read(raw.ctypes.data_as(P), raw.size, ctypes.byref(Lc), ctypes.byref(Ec),
                                ctypes.byref(nc), None, None)
    _check(rc, "moe_profile_read", True)
    pairs = np.zeros((nc.value, 2), np.uint16)
    inv = np.zeros((Lc.value, Ec.value), np.int32)
    rc = lib().moe_profile_read(raw.ctypes.data_as(P), raw.size, ctypes.byref(Lc), ctypes.byref(Ec),
                                ctypes.byref(nc), pairs.ctypes.data_as(P), inv.ctypes.data_as(P))
    _check(rc, "moe_profile_read", True)
    return Lc.value, Ec.value, pairs, inv


def moe_profile_hit_rate(pairs, L: int, E: int, slots: int, hist) -> float:
    """Fraction of the routed reads in hist [L, E] that land in the first
    `slots` ranked pairs."""
    import numpy as np
    pr = np.ascontiguousarray(pairs, dtype=np.uint16).reshape(-1, 2)
    h = np.ascontiguousarray(hist, dtype=np.uint32)
    v = float(lib().moe_profile_hit_rate(pr.ctypes.data_as(ctypes.c_void_p), pr.shape[0], L, E, slots,
                                         h.ctypes.data_as(ctypes.c_void_p)))
    if v < 0:
        raise MoeError(MOE_ERR_ARG, "moe_profile_hit_rate")
    return v
