"""Assemble seeded synthetic workloads in host/device memory (inputs only).

A workload is a LayerShape plus:
  * the pinned host pool of P expert records (record i = routed expert
    (i // E, i % E)); with ``distinct`` < P only the first ``distinct`` records
    are generated and record i repeats record i mod distinct (same bytes,
    same transfer cost; it bounds generation time for 64-156 GB pools);
  * router weights, bf16 [L, E, d], on the device;
  * shared-expert records [L] on the device (when the shape has them);
  * hidden states: decode AR(1) chains or prefill rows, bf16.
"""
from __future__ import annotations

import numpy as np
import torch

from . import (LayerShape, MASTER_SEED, decode_hidden_bf16, expert_record, expert_record_bf16,
               expert_record_into, expert_record_mx, mx_record_layout, record_bytes, replicate_records,
               router_bf16)

# record formats (the values of the library's MOE_FMT_* constants)
FMT_NVFP4, FMT_MXFP4, FMT_BF16 = 0, 1, 2


def format_record_bytes(fmt: int, d: int, F: int) -> int:
    if fmt == FMT_MXFP4:
        return mx_record_layout(d, F)[4]
    if fmt == FMT_BF16:
        return 6 * d * F
    return record_bytes(d, F)


def pinned_pool(shape: LayerShape, P: int | None = None, distinct: int | None = None,
                seed: int = MASTER_SEED) -> torch.Tensor:
    P = shape.L * shape.E if P is None else P
    distinct = P if distinct is None else min(distinct, P)
    rb = record_bytes(shape.d, shape.F)
    pool = torch.empty(P * rb, dtype=torch.uint8, pin_memory=True)
    base = pool.data_ptr()
    for i in range(distinct):
        expert_record_into(base + i * rb, i // shape.E, i % shape.E, shape.d, shape.F, seed=seed)
    if distinct < P:
        replicate_records(base, rb, distinct, P)
    return pool


def pinned_pool_fmt(shape: LayerShape, fmt: int, P: int | None = None, distinct: int | None = None,
                    seed: int = MASTER_SEED) -> torch.Tensor:
    """pinned_pool with the records in NVFP4 or MXFP4 (same draws)."""
    if fmt == FMT_NVFP4:
        return pinned_pool(shape, P, distinct, seed)
    P = shape.L * shape.E if P is None else P
    distinct = P if distinct is None else min(distinct, P)
    rb = format_record_bytes(fmt, shape.d, shape.F)
    pool = torch.empty(P * rb, dtype=torch.uint8, pin_memory=True)
    arr = pool.numpy()
    for i in range(distinct):
        arr[i * rb:(i + 1) * rb] = expert_record_mx(i // shape.E, i % shape.E, shape.d, shape.F, seed=seed)
    if distinct < P:
        replicate_records(pool.data_ptr(), rb, distinct, P)
    return pool


def shared_records_fmt(shape: LayerShape, fmt: int, seed: int = MASTER_SEED) -> np.ndarray | None:
    """The L shared-expert records (uint8) in NVFP4, MXFP4 or BF16 (same draws)."""
    if not shape.shared:
        return None
    if fmt == FMT_NVFP4:
        return shared_records(shape, seed)
    if fmt == FMT_MXFP4:
        return np.concatenate([expert_record_mx(l, 0, shape.d, shape.F, shared=True, seed=seed)
                               for l in range(shape.L)])
    return np.concatenate([expert_record_bf16(l, 0, shape.d, shape.F, shared=True, seed=seed).view(np.uint8)
                           for l in range(shape.L)])


def router_weights(shape: LayerShape, seed: int = MASTER_SEED) -> np.ndarray:
    return np.stack([router_bf16(l, shape.E, shape.d, seed=seed) for l in range(shape.L)])


def shared_records(shape: LayerShape, seed: int = MASTER_SEED) -> np.ndarray | None:
    if not shape.shared:
        return None
    return np.concatenate([expert_record(l, 0, shape.d, shape.F, shared=True, seed=seed)
                           for l in range(shape.L)])


def to_device(a: np.ndarray | None, device="cuda") -> torch.Tensor | None:
    if a is None:
        return None
    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


def decode_inputs(shape: LayerShape, T: int, streams: int = 1, seed: int = MASTER_SEED,
                  stream0: int = 0) -> np.ndarray:
    """bf16 bits [T, L, streams, d]: one AR(1) chain per (stream, layer), no conditioning."""
    out = np.empty((T, shape.L, streams, shape.d), dtype=np.uint16)
    for s in range(streams):
        for l in range(shape.L):
            out[:, l, s, :] = decode_hidden_bf16(stream0 + s, l, T, shape.d, seed=seed)[0]
    return out


class RegisteredPool:
    """A host pool in ordinary (malloc'd) memory, page-locked with cudaHostRegister.

    Used for pools of tens of GB: it pins exactly the bytes asked for (a
    cudaHostAlloc through torch's caching host allocator may round the size up).
    ``tensor`` is a uint8 view; call ``close()`` (or drop the object) to unpin."""

    def __init__(self, shape: LayerShape, P: int | None = None, distinct: int | None = None,
                 seed: int = MASTER_SEED, fmt: int = FMT_NVFP4):
        P = shape.L * shape.E if P is None else P
        distinct = P if distinct is None else min(distinct, P)
        rb = format_record_bytes(fmt, shape.d, shape.F)
        self.nbytes = P * rb
        self.array = np.empty(self.nbytes, dtype=np.uint8)
        base = self.array.ctypes.data
        for i in range(distinct):
            if fmt == FMT_NVFP4:
                expert_record_into(base + i * rb, i // shape.E, i % shape.E, shape.d, shape.F,
                                   seed=seed)
            else:
                self.array[i * rb:(i + 1) * rb] = expert_record_mx(i // shape.E, i % shape.E, shape.d,
                                                                   shape.F, seed=seed)
        if distinct < P:
            replicate_records(base, rb, distinct, P)
        rc = torch.cuda.cudart().cudaHostRegister(base, self.nbytes, 0)
        if int(rc) != 0:
            raise RuntimeError(f"cudaHostRegister failed ({rc})")
        self.registered = True
        self.tensor = torch.from_numpy(self.array)

    def close(self) -> None:
        if getattr(self, "registered", False):
            torch.cuda.cudart().cudaHostUnregister(self.array.ctypes.data)
            self.registered = False

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
