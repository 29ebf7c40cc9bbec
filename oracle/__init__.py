"""CPU oracle of the per-layer routed-expert step (plain C, fp64) -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg
may import this package.  The product path (``expert_offload_caching_b200``)
never does, and shares no code with it: this is the independent definition the
CUDA kernels are checked against.

What it computes, and where the FreeToken pages say so:
  * router logits, softmax and top-k with renormalised gates
    (florigen.ai: 10 of 512 routed experts + 1 shared per token; gaming-st.com,
    "技術的背景": 6 of 256 per layer; pirouter.ai: 4 per layer)
  * NVFP4 decode (E2M1 codes, one E4M3 scale per 16 elements, fp32 tensor
    scale; florigen.ai, "NVFP4で約135GBまで縮める" names E2M1 + block scaling)
  * SwiGLU expert FFN, gate-weighted combine with the shared expert
  * global LRU cache over (layer, expert) slots (ai-hardware-zukan,
    "GPUに載らない分をどう間に合わせるか"; gaming-st.com, "技術的背景")
  * the hybrid split planner q = m*B_P/B_H and the 2.0 auto threshold
    (ai-hardware-zukan, same section; florigen.ai, "CPU/PCIe ratio 1.70x")

Each function is pinned by ``tests/test_oracle_pins.py`` against hand-worked
values, library routines, closed forms and brute force.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liborc.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile liborc.so (gcc -O2, OpenMP, no FP contraction) next to its source."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-ffp-contract=off",
                               "-fno-fast-math", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        i32, i64, u64, dbl, flt, vp = (ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64,
                                       ctypes.c_double, ctypes.c_float, ctypes.c_void_p)
        ip = ctypes.POINTER(ctypes.c_int)
        dp = ctypes.POINTER(ctypes.c_double)
        L.orc_e2m1.restype = dbl
        L.orc_e2m1.argtypes = [ctypes.c_int]
        L.orc_e4m3.restype = dbl
        L.orc_e4m3.argtypes = [ctypes.c_int]
        L.orc_record_layout.argtypes = [ctypes.c_int, ctypes.c_int, vp]
        L.orc_dequant_matrix.argtypes = [vp, ctypes.c_int, ctypes.c_int, ctypes.c_int, vp]
        L.orc_route.restype = ctypes.c_int
        L.orc_route.argtypes = [vp, vp, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                ctypes.c_int, vp, vp, vp, vp]
        L.orc_expert_w4a16.argtypes = [vp, ctypes.c_int, ctypes.c_int, vp, vp, vp]
        L.orc_expert_w4a4.argtypes = [vp, ctypes.c_int, ctypes.c_int, vp, vp]
        L.orc_tensor_scale_f32.restype = flt
        L.orc_tensor_scale_f32.argtypes = [vp, i64]
        L.orc_e4m3_rne.restype = ctypes.c_int
        L.orc_e4m3_rne.argtypes = [flt]
        L.orc_e2m1_rne.restype = ctypes.c_int
        L.orc_e2m1_rne.argtypes = [flt]
        L.orc_nvfp4_quantize.argtypes = [vp, i64, flt, vp, vp]
        L.orc_moe_layer.restype = ctypes.c_int
        L.orc_moe_layer.argtypes = [vp, i64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                    ctypes.c_int, ctypes.c_int, ctypes.c_int, vp, vp, vp,
                                    ctypes.c_int, ctypes.c_int, vp, vp, vp]
        L.orc_lru_new.restype = vp
        L.orc_lru_new.argtypes = [i64, i64, i64]
        L.orc_lru_free.argtypes = [vp]
        L.orc_lru_state.argtypes = [vp, vp, vp, vp, vp]
        L.orc_lru_batch.restype = ctypes.c_int
        L.orc_lru_batch.argtypes = [vp, ctypes.c_int, vp, ctypes.c_int, vp, vp, vp]
        L.orc_plan_split.restype = ctypes.c_int
        L.orc_plan_split.argtypes = [ctypes.c_int, dbl, dbl, dbl, dbl, ip, ip, ip, dp, dp]
        L.orc_e8m0.restype = dbl
        L.orc_e8m0.argtypes = [ctypes.c_int]
        L.orc_mx_record_layout.argtypes = [ctypes.c_int, ctypes.c_int, vp]
        L.orc_dequant_matrix_mx.argtypes = [vp, ctypes.c_int, ctypes.c_int, ctypes.c_int, vp]
        L.orc_expert_mx_w4a16.argtypes = [vp, ctypes.c_int, ctypes.c_int, vp, vp]
        L.orc_expert_bf16.argtypes = [vp, ctypes.c_int, ctypes.c_int, vp, vp]
        L.orc_mx_quantize.argtypes = [vp, ctypes.c_int64, vp, vp]
        L.orc_expert_mx_w4a4.argtypes = [vp, ctypes.c_int, ctypes.c_int, vp, vp]
        L.orc_moe_layer_fmt.argtypes = [vp, ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                        ctypes.c_int, ctypes.c_int, ctypes.c_int, vp, vp, vp, ctypes.c_int,
                                        ctypes.c_int, ctypes.c_int, ctypes.c_int, vp, vp, vp]
        _lib = L
    return _lib


def _p(a) -> int | None:
    if a is None:
        return None
    assert isinstance(a, np.ndarray) and a.flags["C_CONTIGUOUS"], type(a)
    return a.ctypes.data


# --------------------------------------------------------------- formats --
def e2m1(code: int) -> float:
    return lib().orc_e2m1(int(code))


def e4m3(byte: int) -> float:
    return lib().orc_e4m3(int(byte))


def e4m3_rne(r: float) -> int:
    return lib().orc_e4m3_rne(float(r))


def e2m1_rne(v: float) -> int:
    return lib().orc_e2m1_rne(float(v))


def tensor_scale(x: np.ndarray) -> np.float32:
    x = np.ascontiguousarray(x, dtype=np.float32)
    return np.float32(lib().orc_tensor_scale_f32(_p(x), x.size))


def nvfp4_quantize(x: np.ndarray, s_t: float) -> tuple[np.ndarray, np.ndarray]:
    x = np.ascontiguousarray(x, dtype=np.float32).ravel()
    assert x.size % 16 == 0
    codes = np.empty(x.size // 2, dtype=np.uint8)
    scales = np.empty(x.size // 16, dtype=np.uint8)
    lib().orc_nvfp4_quantize(_p(x), x.size, float(s_t), _p(codes), _p(scales))
    return codes, scales


def record_layout(d: int, F: int) -> tuple[int, ...]:
    off = np.zeros(6, dtype=np.int64)
    lib().orc_record_layout(d, F, _p(off))
    return tuple(int(v) for v in off)


def dequant_matrix(rec: np.ndarray, d: int, F: int, which: int) -> np.ndarray:
    """which = 0 gate [F, d], 1 up [F, d], 2 down [d, F], fp64."""
    out = np.empty(F * d, dtype=np.float64)
    lib().orc_dequant_matrix(_p(np.ascontiguousarray(rec)), d, F, which, _p(out))
    return out.reshape((F, d) if which < 2 else (d, F))


# --------------------------------------------------------------- routing --
def route(Wr: np.ndarray, x: np.ndarray, k: int, renorm: bool = True):
    """Wr bf16 bits [E, d], x bf16 bits [T, d] -> (idx [T,k] ascending, gates [T,k],
    logits [T,E], gap [T] = z_(k) - z_(k+1))."""
    Wr = np.ascontiguousarray(Wr, dtype=np.uint16)
    x = np.ascontiguousarray(np.atleast_2d(x), dtype=np.uint16)
    E, d = Wr.shape
    T = x.shape[0]
    idx = np.empty((T, k), dtype=np.int32)
    gates = np.empty((T, k), dtype=np.float64)
    logits = np.empty((T, E), dtype=np.float64)
    gap = np.empty(T, dtype=np.float64)
    rc = lib().orc_route(_p(Wr), _p(x), T, E, d, k, int(renorm), _p(idx), _p(gates),
                         _p(logits), _p(gap))
    if rc:
        raise ValueError("orc_route: bad arguments")
    return idx, gates, logits, gap


def expert_w4a16(rec: np.ndarray, d: int, F: int, x: np.ndarray):
    """One expert on one bf16 row: (y [d], h [F]) in fp64."""
    y = np.empty(d, dtype=np.float64)
    h = np.empty(F, dtype=np.float64)
    lib().orc_expert_w4a16(_p(np.ascontiguousarray(rec)), d, F,
                           _p(np.ascontiguousarray(x, dtype=np.uint16)), _p(y), _p(h))
    return y, h


def expert_w4a4(rec: np.ndarray, d: int, F: int, x: np.ndarray) -> np.ndarray:
    y = np.empty(d, dtype=np.float64)
    lib().orc_expert_w4a4(_p(np.ascontiguousarray(rec)), d, F,
                          _p(np.ascontiguousarray(x, dtype=np.uint16)), _p(y))
    return y


def e8m0(code: int) -> float:
    return lib().orc_e8m0(int(code))


def mx_record_layout(d: int, F: int) -> tuple[int, ...]:
    off = np.zeros(5, dtype=np.int64)
    lib().orc_mx_record_layout(d, F, _p(off))
    return tuple(int(v) for v in off)


def dequant_matrix_mx(rec: np.ndarray, d: int, F: int, which: int) -> np.ndarray:
    """Dequantised matrix of an MXFP4 record: 0 gate [F, d], 1 up [F, d], 2 down [d, F]."""
    out = np.empty((F, d) if which < 2 else (d, F), dtype=np.float64)
    lib().orc_dequant_matrix_mx(_p(np.ascontiguousarray(rec)), d, F, which, _p(out))
    return out


def expert_mx_w4a16(rec: np.ndarray, d: int, F: int, x: np.ndarray) -> np.ndarray:
    """One expert over an MXFP4 record on one bf16 row, fp64."""
    y = np.empty(d, dtype=np.float64)
    lib().orc_expert_mx_w4a16(_p(np.ascontiguousarray(rec)), d, F,
                              _p(np.ascontiguousarray(x, dtype=np.uint16)), _p(y))
    return y


def mx_quantize(x: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """MXFP4 codes (n/2 bytes) and E8M0 scales (n/32) of fp32 values (OCP rule)."""
    x = np.ascontiguousarray(x, dtype=np.float32).ravel()
    codes = np.empty(x.size // 2, dtype=np.uint8)
    scales = np.empty(x.size // 32, dtype=np.uint8)
    lib().orc_mx_quantize(_p(x), x.size, _p(codes), _p(scales))
    return codes, scales


def expert_mx_w4a4(rec: np.ndarray, d: int, F: int, x: np.ndarray) -> np.ndarray:
    """One expert over an MXFP4 record on one bf16 row, activations MXFP4-quantized (prefill)."""
    y = np.empty(d, dtype=np.float64)
    lib().orc_expert_mx_w4a4(_p(np.ascontiguousarray(rec)), d, F,
                             _p(np.ascontiguousarray(x, dtype=np.uint16)), _p(y))
    return y


def expert_bf16(rec: np.ndarray, d: int, F: int, x: np.ndarray) -> np.ndarray:
    """One expert over a BF16 record (W13 rows interleaved, then W2) on one bf16 row, fp64."""
    y = np.empty(d, dtype=np.float64)
    lib().orc_expert_bf16(_p(np.ascontiguousarray(rec, dtype=np.uint16)), d, F,
                          _p(np.ascontiguousarray(x, dtype=np.uint16)), _p(y))
    return y


FMT_NVFP4, FMT_MXFP4, FMT_BF16 = 0, 1, 2


def moe_layer(pool: np.ndarray, P: int, layer: int, E: int, d: int, F: int, k: int,
              Wr_layer: np.ndarray, shared_rec: np.ndarray | None, x: np.ndarray,
              w4a4: bool = False, renorm: bool = True, fmt: int = FMT_NVFP4,
              shared_fmt: int | None = None):
    """One layer on T independent rows: (idx [T,k], gates [T,k], y [T,d] fp64).

    fmt: the routed records' format (NVFP4 or MXFP4); shared_fmt: the shared
    record's (None: the routed format; or BF16)."""
    x = np.ascontiguousarray(np.atleast_2d(x), dtype=np.uint16)
    T = x.shape[0]
    sf = fmt if shared_fmt is None else shared_fmt
    idx = np.empty((T, k), dtype=np.int32)
    gates = np.empty((T, k), dtype=np.float64)
    y = np.empty((T, d), dtype=np.float64)
    if shared_rec is not None:
        shared_rec = np.ascontiguousarray(shared_rec).view(np.uint8)
    rc = lib().orc_moe_layer_fmt(_p(pool), P, layer, E, d, F, k, int(renorm),
                                 _p(np.ascontiguousarray(Wr_layer, dtype=np.uint16)),
                                 _p(shared_rec), _p(x), T, int(w4a4), fmt, sf, _p(idx), _p(gates),
                                 _p(y))
    if rc:
        raise ValueError("orc_moe_layer_fmt: bad arguments")
    return idx, gates, y


# ------------------------------------------------------------------- LRU --
class LRU:
    """Global LRU cache of (layer, expert) slots; key = layer*E + expert."""

    def __init__(self, L: int, E: int, C: int):
        self.L, self.E, self.C = L, E, C
        self._h = lib().orc_lru_new(L, E, C)
        if not self._h:
            raise ValueError("bad LRU dimensions")

    def __del__(self):
        h = getattr(self, "_h", None)
        if h and _lib is not None:
            _lib.orc_lru_free(h)
            self._h = None

    def batch(self, layer: int, experts) -> list[tuple[int, int, int, int]]:
        """Lookup batch of distinct ascending experts -> [(expert, slot, hit, evicted_key)]."""
        ex = np.ascontiguousarray(experts, dtype=np.int32)
        n = ex.size
        slot = np.empty(n, dtype=np.int32)
        hit = np.empty(n, dtype=np.int32)
        ev = np.empty(n, dtype=np.int64)
        rc = lib().orc_lru_batch(self._h, layer, _p(ex), n, _p(slot), _p(hit), _p(ev))
        if rc < 0:
            raise ValueError("LRU batch rejected (order, range or size)")
        return [(int(e), int(s), int(h), int(v)) for e, s, h, v in zip(ex, slot, hit, ev)]

    def state(self):
        m = np.empty(self.L * self.E, dtype=np.int32)
        o = np.empty(self.C, dtype=np.int32)
        s = np.empty(self.C, dtype=np.uint64)
        c = np.zeros(1, dtype=np.uint64)
        lib().orc_lru_state(self._h, _p(m), _p(o), _p(s), _p(c))
        return m, o, s, int(c[0])


# --------------------------------------------------------------- planner --
def plan_split(m: int, B_P: float, B_H: float, threshold: float = 2.0,
               expert_bytes: float = 1.0) -> dict:
    q, cpu, mode = ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
    qr, tf = ctypes.c_double(), ctypes.c_double()
    rc = lib().orc_plan_split(m, B_P, B_H, threshold, expert_bytes, ctypes.byref(q),
                              ctypes.byref(cpu), ctypes.byref(mode), ctypes.byref(qr),
                              ctypes.byref(tf))
    if rc:
        raise ValueError("plan_split: bad arguments")
    return dict(q=q.value, cpu=cpu.value, mode=mode.value, q_real=qr.value, t_finish=tf.value)


from . import workloads  # noqa: E402,F401  (input conditioning and trace helpers)
