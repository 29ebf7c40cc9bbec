"""Workload assembly for the tests: seeded inputs conditioned with the oracle's
router, and cache traces from the oracle's LRU simulator.  TEST INFRASTRUCTURE.

Input conditioning (the k-th/(k+1)-th gap rule): a hidden-state row whose
oracle logits have z_(k) - z_(k+1) < GAP_MIN has its noise redrawn with the
attempt counter + 1; a decode chain continues from the redrawn row.  The gap
makes the selected set independent of the fp32 summation order of any
correct router, so expert indices can be compared bit for bit.
"""
from __future__ import annotations

import numpy as np

import synth
from . import LRU, route

GAP_MIN = 1e-4


def router_weights(shape: synth.LayerShape, layers=None, seed: int = synth.MASTER_SEED):
    layers = range(shape.L) if layers is None else layers
    return {l: synth.router_bf16(l, shape.E, shape.d, seed=seed) for l in layers}


def decode_chain(stream: int, layer: int, T: int, d: int, attempts: dict[int, int],
                 seed: int = synth.MASTER_SEED, rho: float = 0.9) -> np.ndarray:
    out = np.empty((T, d), dtype=np.uint16)
    x_prev = None
    for t in range(T):
        eps = synth.noise_f32(synth.PURPOSE_DECODE, stream, layer, t, attempts.get(t, 0), d,
                              seed=seed)
        x = synth.ar1_step(x_prev, eps, t, rho)
        out[t] = synth.to_bf16(x)
        x_prev = x
    return out


def conditioned_decode(Wr: np.ndarray, k: int, stream: int, layer: int, T: int,
                       seed: int = synth.MASTER_SEED):
    """AR(1) rows of one (stream, layer) chain with every row's gap >= GAP_MIN.
    Returns (x bf16 [T, d], attempts {t: attempt})."""
    d = Wr.shape[1]
    attempts: dict[int, int] = {}
    while True:
        x = decode_chain(stream, layer, T, d, attempts, seed)
        gap = route(Wr, x, k)[3]
        bad = np.nonzero(gap < GAP_MIN)[0]
        if bad.size == 0:
            return x, attempts
        t = int(bad[0])
        attempts[t] = attempts.get(t, 0) + 1
        if attempts[t] > 64:
            raise RuntimeError("input conditioning did not converge")


def conditioned_prefill(Wr: np.ndarray, k: int, layer: int, T: int,
                        seed: int = synth.MASTER_SEED):
    """T i.i.d. N(0,1) rows for one layer, each with gap >= GAP_MIN."""
    d = Wr.shape[1]
    x = np.empty((T, d), dtype=np.uint16)
    for t in range(T):
        x[t] = synth.to_bf16(synth.noise_f32(synth.PURPOSE_PREFILL, 0, layer, t, 0, d, seed=seed))
    attempt = np.zeros(T, dtype=np.int64)
    while True:
        gap = route(Wr, x, k)[3]
        bad = np.nonzero(gap < GAP_MIN)[0]
        if bad.size == 0:
            return x, {int(t): int(attempt[t]) for t in np.nonzero(attempt)[0]}
        for t in bad:
            attempt[t] += 1
            if attempt[t] > 64:
                raise RuntimeError("input conditioning did not converge")
            x[t] = synth.to_bf16(synth.noise_f32(synth.PURPOSE_PREFILL, 0, layer, int(t),
                                                 int(attempt[t]), d, seed=seed))


def decode_trace(idx: np.ndarray, L: int, E: int, C: int, lru: LRU | None = None,
                 shard: tuple[int, int] = (0, 1)):
    """Replay decode lookups through the oracle LRU.

    idx: [T, L, rows, k] selected experts per (token step, layer, row).  One
    lookup batch per (step, layer): the distinct experts over the rows, in
    ascending id -- with shard = (rank, size), only those with e % size == rank
    (the cache of one rank of an expert-parallel layer).
    Returns (events [(t, layer, expert, slot, hit, evicted)], lru).
    """
    lru = LRU(L, E, C) if lru is None else lru
    events = []
    T = idx.shape[0]
    rank, size = shard
    for t in range(T):
        for l in range(L):
            batch = np.unique(idx[t, l].ravel())
            batch = batch[batch % size == rank]
            for e, s, h, v in lru.batch(l, batch):
                events.append((t, l, e, s, h, v))
    return events, lru


def prefill_trace(idx: np.ndarray, L: int, E: int, C: int, prefetch: bool = True,
                  lru: LRU | None = None, shard: tuple[int, int] = (0, 1)):
    """Replay a prefill chunk: idx [L, T, k].  Per layer one routed batch (the
    distinct experts of all rows, ascending), then, with prefetch, one batch of
    all E experts of the next layer -- with shard = (rank, size), only the
    experts e % size == rank in both.  Events carry a kind: 0 routed, 1 prefetch."""
    lru = LRU(L, E, C) if lru is None else lru
    events = []
    rank, size = shard
    for l in range(L):
        batch = np.unique(idx[l].ravel())
        for e, s, h, v in lru.batch(l, batch[batch % size == rank]):
            events.append((0, l, e, s, h, v))
        if prefetch and l + 1 < L:
            allx = np.arange(E, dtype=np.int32)
            for e, s, h, v in lru.batch(l + 1, allx[allx % size == rank]):
                events.append((1, l + 1, e, s, h, v))
    return events, lru


def static_split_trace(idx: np.ndarray, L: int, E: int, C: int, scratch: int):
    """The static per-layer split (ai-hardware-zukan.com, "GPUに載らない分をどう間に合わせるか":
    the comparison policy that splits the expert cache over the layers without
    looking at the routing), as the C ABI's MOE_CACHE_STATIC_SPLIT defines it:
    s = min((C - scratch) // L, E) experts per layer are resident -- layer l's
    experts 0 .. s-1 in slots l*s .. l*s+s-1 -- and never change; in each lookup
    batch (the distinct experts over the rows, ascending) an expert e < s is a
    hit in slot l*s + e, any other is the m-th miss of the batch and goes to
    scratch slot L*s + m; nothing is evicted.

    idx: [T, L, rows, k].  Returns events [(t, layer, expert, slot, hit, evicted)]."""
    s = min((C - scratch) // L, E)
    events = []
    for t in range(idx.shape[0]):
        for l in range(L):
            m = 0
            for e in np.unique(idx[t, l].ravel()):
                e = int(e)
                if e < s:
                    events.append((t, l, e, l * s + e, 1, -1))
                else:
                    events.append((t, l, e, L * s + m, 0, -1))
                    m += 1
    return events
