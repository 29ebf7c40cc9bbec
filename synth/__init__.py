"""Seeded synthetic inputs for the per-layer routed-expert step.

Inputs only: SplitMix64 counter-based draws, Box-Muller normals, NVFP4 (and
MXFP4 / BF16) encoding of the synthetic expert weights, bf16 rounding and the
AR(1) hidden-state recurrence.  None of the step's own arithmetic lives here; both the CPU oracle
(``oracle/``) and the CUDA path read the bytes this module writes.

Workload recipes (shapes from the FreeToken pages' models; weights N(0, 0.02)):
  * routed expert records: purpose 1, keyed by (layer, expert, matrix)
  * shared expert records: purpose 5, keyed by (layer, 0, matrix)
  * router weights: purpose 2, keyed by layer, rounded to bf16
  * decode hidden states: purpose 3, one AR(1) chain (rho = 0.9) per (stream, layer)
  * prefill rows: purpose 4, i.i.d. N(0, 1) per (layer, row)
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_LIB = os.path.join(_HERE, "libsynth.so")
_lib = None

MASTER_SEED = 20260901
PURPOSE_EXPERT, PURPOSE_ROUTER, PURPOSE_DECODE, PURPOSE_PREFILL, PURPOSE_SHARED = 1, 2, 3, 4, 5


def build(force: bool = False) -> str:
    """Compile libsynth.so next to its source (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-ffp-contract=off",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        u64, i32, i64, dbl, vp = (ctypes.c_uint64, ctypes.c_int32, ctypes.c_int64,
                                  ctypes.c_double, ctypes.c_void_p)
        L.synth_key.restype = u64
        L.synth_key.argtypes = [u64] * 6
        L.synth_normals_f32.argtypes = [u64, i64, dbl, vp]
        L.synth_to_bf16.argtypes = [vp, i64, vp]
        L.synth_router_bf16.argtypes = [u64, i32, i32, i32, dbl, vp]
        L.synth_noise_f32.argtypes = [u64, i32, i32, i32, i64, i32, i32, vp]
        L.synth_ar1_step.argtypes = [vp, vp, i32, i64, ctypes.c_float, vp]
        L.synth_record_layout.argtypes = [i32, i32, vp]
        L.synth_expert_record.argtypes = [u64, i32, i32, i32, i32, i32, dbl, vp]
        L.synth_expert_matrix_f32.argtypes = [u64, i32, i32, i32, i32, i32, i32, dbl, vp]
        L.synth_replicate_records.argtypes = [vp, i64, i64, i64]
        L.synth_prefill_rows_bf16.argtypes = [u64, i32, i32, i32, vp]
        L.synth_mx_record_layout.argtypes = [i32, i32, vp]
        L.synth_mx_encode.argtypes = [vp, i64, i64, vp, vp]
        L.synth_expert_record_mx.argtypes = [u64, i32, i32, i32, i32, i32, dbl, vp]
        L.synth_expert_record_bf16.argtypes = [u64, i32, i32, i32, i32, i32, dbl, vp]
        _lib = L
    return _lib


def _p(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


@dataclass(frozen=True)
class LayerShape:
    """Shape of one MoE layer stack: L layers of E routed experts, top-k, width d, FFN F."""
    name: str
    L: int
    E: int
    k: int
    d: int
    F: int
    shared: bool
    tokens: int
    cache_slots: int
    sigma: float = 0.02


def record_layout(d: int, F: int) -> tuple[int, int, int, int, int, int]:
    """(w13 codes, w13 scales, w2 codes, w2 scales, tensor scales, total) byte offsets."""
    off = np.zeros(6, dtype=np.int64)
    lib().synth_record_layout(d, F, _p(off))
    return tuple(int(v) for v in off)


def record_bytes(d: int, F: int) -> int:
    return record_layout(d, F)[5]


def expert_record(layer: int, expert: int, d: int, F: int, *, seed: int = MASTER_SEED,
                  shared: bool = False, sigma: float = 0.02, out=None) -> np.ndarray:
    """The NVFP4 record of routed expert (layer, expert), or of layer's shared expert."""
    nb = record_bytes(d, F)
    if out is None:
        out = np.empty(nb, dtype=np.uint8)
    purpose = PURPOSE_SHARED if shared else PURPOSE_EXPERT
    lib().synth_expert_record(seed, purpose, layer, 0 if shared else expert, d, F, sigma, _p(out))
    return out


def expert_record_into(ptr: int, layer: int, expert: int, d: int, F: int, *,
                       seed: int = MASTER_SEED, shared: bool = False, sigma: float = 0.02) -> None:
    """Same as expert_record, written at a raw host address (e.g. a pinned pool)."""
    purpose = PURPOSE_SHARED if shared else PURPOSE_EXPERT
    lib().synth_expert_record(seed, purpose, layer, 0 if shared else expert, d, F, sigma, ptr)


def expert_matrix_f32(layer: int, expert: int, m: int, d: int, F: int, *, seed: int = MASTER_SEED,
                      shared: bool = False, sigma: float = 0.02) -> np.ndarray:
    """The fp32 normal draws behind matrix m (0 gate [F,d], 1 up [F,d], 2 down [d,F])."""
    out = np.empty(F * d, dtype=np.float32)
    purpose = PURPOSE_SHARED if shared else PURPOSE_EXPERT
    lib().synth_expert_matrix_f32(seed, purpose, layer, 0 if shared else expert, m, d, F, sigma,
                                  _p(out))
    return out.reshape((F, d) if m < 2 else (d, F))


def mx_record_layout(d: int, F: int) -> tuple[int, int, int, int, int]:
    """MXFP4 record: (w13 codes, w13 E8M0 scales, w2 codes, w2 scales, total) byte offsets."""
    off = np.zeros(5, dtype=np.int64)
    lib().synth_mx_record_layout(d, F, _p(off))
    return tuple(int(v) for v in off)


def mx_encode(w: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """MXFP4 codes [rows, K/2] and E8M0 scales [rows, K/32] of an fp32 [rows, K] matrix."""
    w = np.ascontiguousarray(np.atleast_2d(w), dtype=np.float32)
    rows, K = w.shape
    codes = np.empty((rows, K // 2), dtype=np.uint8)
    scales = np.empty((rows, K // 32), dtype=np.uint8)
    lib().synth_mx_encode(_p(w), rows, K, _p(codes), _p(scales))
    return codes, scales


def expert_record_mx(layer: int, expert: int, d: int, F: int, *, seed: int = MASTER_SEED,
                     shared: bool = False, sigma: float = 0.02) -> np.ndarray:
    """The MXFP4 record (E2M1, one E8M0 scale per 32) of the same draws as expert_record."""
    out = np.empty(mx_record_layout(d, F)[4], dtype=np.uint8)
    purpose = PURPOSE_SHARED if shared else PURPOSE_EXPERT
    lib().synth_expert_record_mx(seed, purpose, layer, 0 if shared else expert, d, F, sigma, _p(out))
    return out


def expert_record_bf16(layer: int, expert: int, d: int, F: int, *, seed: int = MASTER_SEED,
                       shared: bool = True, sigma: float = 0.02) -> np.ndarray:
    """A BF16 record of the same draws: W13 [2F x d] (rows interleaved gate/up), then W2 [d x F]."""
    out = np.empty(3 * d * F, dtype=np.uint16)
    purpose = PURPOSE_SHARED if shared else PURPOSE_EXPERT
    lib().synth_expert_record_bf16(seed, purpose, layer, 0 if shared else expert, d, F, sigma, _p(out))
    return out


def replicate_records(ptr: int, rec_bytes: int, n_src: int, n_dst: int) -> None:
    lib().synth_replicate_records(ptr, rec_bytes, n_src, n_dst)


def router_bf16(layer: int, E: int, d: int, *, seed: int = MASTER_SEED,
                sigma: float = 0.02) -> np.ndarray:
    """Router weights of one layer, [E, d] bf16 bit patterns (uint16)."""
    out = np.empty((E, d), dtype=np.uint16)
    lib().synth_router_bf16(seed, layer, E, d, sigma, _p(out))
    return out


def noise_f32(purpose: int, stream: int, layer: int, t: int, attempt: int, d: int, *,
              seed: int = MASTER_SEED) -> np.ndarray:
    out = np.empty(d, dtype=np.float32)
    lib().synth_noise_f32(seed, purpose, stream, layer, t, attempt, d, _p(out))
    return out


def ar1_step(x_prev: np.ndarray | None, eps: np.ndarray, t: int, rho: float = 0.9) -> np.ndarray:
    d = eps.shape[0]
    out = np.empty(d, dtype=np.float32)
    prev = np.zeros(d, dtype=np.float32) if x_prev is None else np.ascontiguousarray(x_prev,
                                                                                   np.float32)
    lib().synth_ar1_step(_p(prev), _p(np.ascontiguousarray(eps, np.float32)), d, t, rho, _p(out))
    return out


def to_bf16(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.uint16)
    lib().synth_to_bf16(_p(x), x.size, _p(out))
    return out


def bf16_to_f32(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32)


def decode_hidden_bf16(stream: int, layer: int, T: int, d: int, *, seed: int = MASTER_SEED,
                       rho: float = 0.9, accept=None) -> tuple[np.ndarray, int]:
    """T AR(1) hidden states of one (stream, layer) chain as bf16 [T, d].

    ``accept(x_bf16_row) -> bool`` may reject a candidate row; the row's noise
    is then redrawn with the attempt counter + 1 and the chain continues from
    the accepted row.  Returns (rows, number of redraws).
    """
    out = np.empty((T, d), dtype=np.uint16)
    x_prev = None
    redraws = 0
    for t in range(T):
        attempt = 0
        while True:
            eps = noise_f32(PURPOSE_DECODE, stream, layer, t, attempt, d, seed=seed)
            x = ar1_step(x_prev, eps, t, rho)
            xb = to_bf16(x)
            if accept is None or accept(xb):
                break
            attempt += 1
            redraws += 1
            if attempt > 64:
                raise RuntimeError("input conditioning did not converge")
        out[t] = xb
        x_prev = x
    return out, redraws


def prefill_rows_bf16(layer: int, T: int, d: int, *, seed: int = MASTER_SEED,
                      accept=None) -> tuple[np.ndarray, int]:
    """T i.i.d. N(0, 1) rows for one layer's prefill chunk, bf16 [T, d]."""
    out = np.empty((T, d), dtype=np.uint16)
    redraws = 0
    for t in range(T):
        attempt = 0
        while True:
            xb = to_bf16(noise_f32(PURPOSE_PREFILL, 0, layer, t, attempt, d, seed=seed))
            if accept is None or accept(xb):
                break
            attempt += 1
            redraws += 1
            if attempt > 64:
                raise RuntimeError("input conditioning did not converge")
        out[t] = xb
    return out, redraws


def prefill_rows_fast(layer: int, T: int, d: int, *, seed: int = MASTER_SEED) -> np.ndarray:
    """The rows of prefill_rows_bf16 with no conditioning (attempt 0 everywhere), in C."""
    out = np.empty((T, d), dtype=np.uint16)
    lib().synth_prefill_rows_bf16(seed, layer, T, d, _p(out))
    return out


# The workloads (shapes of the models on the FreeToken pages; cache sizes as fractions of
# the routed pool).  "tokens" is the decode length per stream.
TINY = LayerShape("tiny", L=1, E=16, k=2, d=256, F=512, shared=False, tokens=64, cache_slots=4)
GPT_OSS = LayerShape("gpt-oss-120b-shaped", L=36, E=128, k=4, d=2880, F=2880, shared=False,
                     tokens=512, cache_slots=int(0.40 * 36 * 128))
QWEN38 = LayerShape("qwen3.8-flash-next-shaped", L=48, E=512, k=10, d=2048, F=768, shared=True,
                    tokens=256, cache_slots=int(0.25 * 48 * 512))
DSV4 = LayerShape("deepseek-v4-flash-shaped", L=43, E=256, k=6, d=4096, F=2048, shared=True,
                  tokens=256, cache_slots=int(0.11 * 43 * 256))
SHAPES = {s.name: s for s in (TINY, GPT_OSS, QWEN38, DSV4)}
