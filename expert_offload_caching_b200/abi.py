"""Thin ctypes binding of libmoeoffload.so: the C ABI of include/moe_offload.h under
the same names.  Argument marshalling only -- every step of the routed-expert
path runs in the library's CUDA kernels.  Pointer arguments accept a torch
tensor, a numpy array, a raw integer address or None."""
from __future__ import annotations

import ctypes
import os

from . import build as _build

MOE_OK, MOE_ERR_ARG, MOE_ERR_CUDA, MOE_ERR_NOT_PINNED = 0, 1, 2, 3
MOE_ERR_CAPACITY, MOE_ERR_TIMEOUT, MOE_ERR_STATE, MOE_ERR_UNSUPPORTED = 4, 5, 6, 7
MOE_CACHE_RESET, MOE_CACHE_PREFETCH_NEXT = 1, 2
MOE_CACHE_STATIC_SPLIT = 4
MOE_FMT_NVFP4, MOE_FMT_MXFP4, MOE_FMT_BF16 = 0, 1, 2
MOE_K_ROUTE, MOE_K_GATEUP, MOE_K_DOWN, MOE_K_COMBINE = 0, 1, 2, 3
MOE_K_PREFILL_ROUTE, MOE_K_PREFILL_GATEUP, MOE_K_PREFILL_DOWN = 4, 5, 6
MOE_K_LAYER, MOE_K_LAYER_HITS, MOE_K_MISS, MOE_K_COUNT = 7, 8, 9, 10
KERNEL_NAMES = ["route_lookup", "gate_up", "down", "combine", "prefill_route", "prefill_gate_up",
                "prefill_down", "expert_layer", "expert_hits", "expert_miss"]
ROUTE_PHASES = ["logits", "elect", "topk", "jobs", "table_read", "select_write", "publish",
                "wait_previous_layer"]


class moe_dims(ctypes.Structure):
    _fields_ = [("L", ctypes.c_int32), ("E", ctypes.c_int32), ("k", ctypes.c_int32),
                ("d", ctypes.c_int32), ("F", ctypes.c_int32), ("has_shared", ctypes.c_int32),
                ("renormalize", ctypes.c_int32), ("max_rows", ctypes.c_int32),
                ("pool_records", ctypes.c_int64), ("weight_format", ctypes.c_int32),
                ("shared_format", ctypes.c_int32)]


class moe_cache_event(ctypes.Structure):
    _fields_ = [("layer", ctypes.c_int32), ("expert", ctypes.c_int32), ("slot", ctypes.c_int32),
                ("hit", ctypes.c_int32), ("evicted_key", ctypes.c_int64),
                ("prefetch", ctypes.c_int32), ("reserved", ctypes.c_int32)]


class moe_layer_trace(ctypes.Structure):
    _fields_ = [("events", ctypes.POINTER(moe_cache_event)), ("capacity", ctypes.c_int32),
                ("count", ctypes.c_int32)]


class moe_stats(ctypes.Structure):
    _fields_ = [("lookups", ctypes.c_int64), ("hits", ctypes.c_int64), ("misses", ctypes.c_int64),
                ("evictions", ctypes.c_int64), ("prefetch_lookups", ctypes.c_int64),
                ("prefetch_misses", ctypes.c_int64), ("h2d_copies", ctypes.c_int64),
                ("h2d_bytes", ctypes.c_int64), ("forward_calls", ctypes.c_int64),
                ("kernel_launches", ctypes.c_int64 * MOE_K_COUNT),
                ("kernel_ms", ctypes.c_double * MOE_K_COUNT),
                ("kernel_bytes", ctypes.c_double * MOE_K_COUNT),
                ("route_phase_us", ctypes.c_double * 8),
                ("host_us", ctypes.c_double * 3),
                ("kernel_span_ms", ctypes.c_double * MOE_K_COUNT)]


class moe_split(ctypes.Structure):
    _fields_ = [("q", ctypes.c_int32), ("cpu", ctypes.c_int32), ("mode", ctypes.c_int32),
                ("reserved", ctypes.c_int32), ("q_real", ctypes.c_double),
                ("t_finish", ctypes.c_double)]


EXPORTS = ["moe_record_bytes", "moe_shared_record_bytes", "moe_record_layout", "moe_workspace_bytes", "moe_arena_bytes",
           "moe_layer_init", "cache_configure", "moe_layer_forward", "moe_layer_forward_host",
           "moe_get_routing", "moe_cache_export", "moe_get_stats", "moe_set_timing",
           "moe_set_wait_limit", "moe_set_expert_shard", "moe_debug_inject", "moe_debug_trace", "plan_split",
           "moe_measure_h2d",
           "moe_measure_h2d_sm",
           "moe_route_noalloc", "moe_status_str", "moe_last_error", "moe_layer_destroy"]

_lib = None


def lib():
    """Load the CUDA library (building it first when sources are newer).  There is
    no fallback: without the library every call raises."""
    global _lib
    if _lib is None:
        if not _build.up_to_date():
            _build.build()
        if not os.path.exists(_build.LIB):
            raise RuntimeError(f"CUDA extension missing: {_build.LIB}")
        L = ctypes.CDLL(_build.LIB)
        vp, i32, i64, u32, dbl, sz = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64,
                                      ctypes.c_uint32, ctypes.c_double, ctypes.c_size_t)
        D = ctypes.POINTER(moe_dims)
        L.moe_record_bytes.restype = sz
        L.moe_record_bytes.argtypes = [D]
        L.moe_shared_record_bytes.restype = sz
        L.moe_shared_record_bytes.argtypes = [D]
        L.moe_record_layout.restype = ctypes.c_int
        L.moe_record_layout.argtypes = [D, vp]
        L.moe_workspace_bytes.restype = sz
        L.moe_workspace_bytes.argtypes = [D]
        L.moe_arena_bytes.restype = sz
        L.moe_arena_bytes.argtypes = [D, i64]
        L.moe_layer_init.restype = ctypes.c_int
        L.moe_layer_init.argtypes = [D, vp, sz, vp, vp, vp, sz, vp, vp, ctypes.POINTER(vp)]
        L.cache_configure.restype = ctypes.c_int
        L.cache_configure.argtypes = [vp, i64, vp, sz, u32]
        L.moe_layer_forward.restype = ctypes.c_int
        L.moe_layer_forward.argtypes = [vp, i32, vp, i32, vp, ctypes.POINTER(moe_layer_trace)]
        L.moe_layer_forward_host.restype = ctypes.c_int
        L.moe_layer_forward_host.argtypes = [vp, i32, vp, i32, vp,
                                             ctypes.POINTER(moe_layer_trace)]
        L.moe_get_routing.restype = ctypes.c_int
        L.moe_get_routing.argtypes = [vp, vp, vp, i32]
        L.moe_cache_export.restype = ctypes.c_int
        L.moe_cache_export.argtypes = [vp, vp, vp, vp, vp]
        L.moe_get_stats.restype = ctypes.c_int
        L.moe_get_stats.argtypes = [vp, ctypes.POINTER(moe_stats)]
        L.moe_set_timing.restype = ctypes.c_int
        L.moe_set_timing.argtypes = [vp, i32]
        L.moe_set_wait_limit.restype = ctypes.c_int
        L.moe_set_wait_limit.argtypes = [vp, dbl]
        L.moe_set_expert_shard.restype = ctypes.c_int
        L.moe_set_expert_shard.argtypes = [vp, i32, i32]
        L.moe_debug_inject.restype = ctypes.c_int
        L.moe_debug_inject.argtypes = [vp, i32, i64]
        L.moe_debug_trace.restype = ctypes.c_int
        L.moe_debug_trace.argtypes = [vp, ctypes.POINTER(ctypes.c_uint64), i32]
        L.plan_split.restype = ctypes.c_int
        L.plan_split.argtypes = [i32, dbl, dbl, dbl, dbl, ctypes.POINTER(moe_split)]
        L.moe_measure_h2d.restype = ctypes.c_int
        L.moe_measure_h2d.argtypes = [vp, vp, sz, sz, i32, vp, ctypes.POINTER(dbl)]
        L.moe_measure_h2d_sm.restype = ctypes.c_int
        L.moe_measure_h2d_sm.argtypes = [vp, vp, sz, sz, i32, vp, ctypes.POINTER(dbl)]
        L.moe_route_noalloc.restype = ctypes.c_int
        L.moe_route_noalloc.argtypes = [vp, vp, i32, i32, i32, i32, i32, vp, vp, vp]
        L.moe_status_str.restype = ctypes.c_char_p
        L.moe_status_str.argtypes = [ctypes.c_int]
        L.moe_last_error.restype = ctypes.c_char_p
        L.moe_last_error.argtypes = [vp]
        L.moe_layer_destroy.restype = None
        L.moe_layer_destroy.argtypes = [vp]
        _lib = L
    return _lib


class MoeError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str = ""):
        self.status = status
        msg = f"{where}: {lib().moe_status_str(status).decode()} ({status})"
        super().__init__(msg + (f": {detail}" if detail else ""))


def _ptr(x) -> int | None:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if hasattr(x, "data_ptr"):
        return x.data_ptr()
    if hasattr(x, "ctypes"):
        return x.ctypes.data
    if hasattr(x, "cuda_stream"):
        return x.cuda_stream
    raise TypeError(f"cannot take the address of {type(x)}")


def _stream(s) -> int:
    return s.cuda_stream if hasattr(s, "cuda_stream") else int(s)


def _check(rc: int, where: str, ctx=None):
    if rc != MOE_OK:
        detail = lib().moe_last_error(ctx).decode() if ctx else ""
        raise MoeError(rc, where, detail)


def make_dims(L, E, k, d, F, has_shared=False, renormalize=True, max_rows=1, pool_records=0,
              weight_format=MOE_FMT_NVFP4, shared_format=None):
    """shared_format None: the routed format."""
    sf = weight_format if shared_format is None else shared_format
    return moe_dims(L, E, k, d, F, int(has_shared), int(renormalize), max_rows, pool_records,
                    weight_format, sf)


def moe_record_bytes(dims: moe_dims) -> int:
    return lib().moe_record_bytes(ctypes.byref(dims))


def moe_shared_record_bytes(dims: moe_dims) -> int:
    return lib().moe_shared_record_bytes(ctypes.byref(dims))


def moe_record_layout(dims: moe_dims) -> tuple[int, ...]:
    off = (ctypes.c_int64 * 6)()
    _check(lib().moe_record_layout(ctypes.byref(dims), off), "moe_record_layout")
    return tuple(off)


def moe_workspace_bytes(dims: moe_dims) -> int:
    return lib().moe_workspace_bytes(ctypes.byref(dims))


def moe_arena_bytes(dims: moe_dims, num_slots: int) -> int:
    return lib().moe_arena_bytes(ctypes.byref(dims), num_slots)


def moe_layer_init(dims, host_pool, host_pool_bytes, router_w, shared_recs, workspace,
                   workspace_bytes, compute_stream, copy_stream) -> int:
    out = ctypes.c_void_p()
    rc = lib().moe_layer_init(ctypes.byref(dims), _ptr(host_pool), host_pool_bytes,
                              _ptr(router_w), _ptr(shared_recs), _ptr(workspace), workspace_bytes,
                              _stream(compute_stream), _stream(copy_stream), ctypes.byref(out))
    _check(rc, "moe_layer_init")
    return out.value


def cache_configure(ctx: int, num_slots: int, slot_arena, arena_bytes: int, flags: int) -> None:
    _check(lib().cache_configure(ctx, num_slots, _ptr(slot_arena), arena_bytes, flags),
           "cache_configure", ctx)


def moe_layer_forward(ctx: int, layer: int, x, T: int, y, trace: moe_layer_trace | None = None):
    rc = lib().moe_layer_forward(ctx, layer, _ptr(x), T, _ptr(y),
                                 ctypes.byref(trace) if trace is not None else None)
    _check(rc, "moe_layer_forward", ctx)


def moe_layer_forward_host(ctx: int, layer: int, x_host, T: int, y_host,
                           trace: moe_layer_trace | None = None):
    rc = lib().moe_layer_forward_host(ctx, layer, _ptr(x_host), T, _ptr(y_host),
                                      ctypes.byref(trace) if trace is not None else None)
    _check(rc, "moe_layer_forward_host", ctx)


def moe_get_routing(ctx: int, idx, gates, T: int) -> None:
    _check(lib().moe_get_routing(ctx, _ptr(idx), _ptr(gates), T), "moe_get_routing", ctx)


def moe_cache_export(ctx: int, map_=None, owner=None, stamp=None):
    clock = ctypes.c_uint64()
    _check(lib().moe_cache_export(ctx, _ptr(map_), _ptr(owner), _ptr(stamp),
                                  ctypes.addressof(clock)), "moe_cache_export", ctx)
    return clock.value


def moe_get_stats(ctx: int) -> moe_stats:
    s = moe_stats()
    _check(lib().moe_get_stats(ctx, ctypes.byref(s)), "moe_get_stats", ctx)
    return s


def moe_set_timing(ctx: int, enable: bool) -> None:
    _check(lib().moe_set_timing(ctx, int(enable)), "moe_set_timing", ctx)


def moe_set_wait_limit(ctx: int, seconds: float) -> None:
    _check(lib().moe_set_wait_limit(ctx, seconds), "moe_set_wait_limit", ctx)


def moe_set_expert_shard(ctx: int, rank: int, size: int) -> None:
    _check(lib().moe_set_expert_shard(ctx, rank, size), "moe_set_expert_shard", ctx)


def moe_debug_inject(ctx: int, what: int, n: int) -> None:
    _check(lib().moe_debug_inject(ctx, what, n), "moe_debug_inject", ctx)


def moe_debug_trace(ctx: int, n: int = 160 * 32):
    """The last traced launch's stamps (see moe_debug_inject what = 9) as a list of ints."""
    buf = (ctypes.c_uint64 * n)()
    _check(lib().moe_debug_trace(ctx, buf, n), "moe_debug_trace", ctx)
    return list(buf)


def plan_split(m: int, B_P: float, B_H: float, threshold: float = 2.0,
               expert_bytes: float = 1.0) -> moe_split:
    out = moe_split()
    _check(lib().plan_split(m, B_P, B_H, threshold, expert_bytes, ctypes.byref(out)), "plan_split")
    return out


def moe_measure_h2d(dev_buf, host_buf, nbytes: int, chunk_bytes: int = 0, reps: int = 10,
                    stream=None) -> float:
    gbs = ctypes.c_double()
    _check(lib().moe_measure_h2d(_ptr(dev_buf), _ptr(host_buf), nbytes, chunk_bytes, reps,
                                 _stream(stream), ctypes.byref(gbs)), "moe_measure_h2d")
    return gbs.value


def moe_measure_h2d_sm(dev_buf, host_buf, nbytes: int, chunk_bytes: int = 0, reps: int = 10,
                       stream=None) -> float:
    """moe_measure_h2d with the copy done by an SM kernel reading mapped host memory."""
    gbs = ctypes.c_double()
    _check(lib().moe_measure_h2d_sm(_ptr(dev_buf), _ptr(host_buf), nbytes, chunk_bytes, reps,
                                    _stream(stream), ctypes.byref(gbs)), "moe_measure_h2d_sm")
    return gbs.value


def moe_route_noalloc(router_w, x, T: int, E: int, d: int, k: int, renormalize: bool, idx, gates,
                      stream) -> None:
    """Routing with no workspace (see include/moe_offload.h): the scratch lives in
    an array inside the library, so the call allocates nothing."""
    _check(lib().moe_route_noalloc(_ptr(router_w), _ptr(x), T, E, d, k, int(renormalize),
                                   _ptr(idx), _ptr(gates), _stream(stream)), "moe_route_noalloc")


def moe_status_str(s: int) -> str:
    return lib().moe_status_str(s).decode()


def moe_last_error(ctx: int) -> str:
    return lib().moe_last_error(ctx).decode()


def moe_layer_destroy(ctx: int) -> None:
    lib().moe_layer_destroy(ctx)
