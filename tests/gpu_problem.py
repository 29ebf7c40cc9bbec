"""Test harness for the device parity tests: build a seeded problem, run the
CUDA path through the C ABI, and compute the oracle's answers on the same
inputs.  (Test infrastructure: imports the oracle.)"""
from __future__ import annotations

import dataclasses

import numpy as np
import torch

import oracle
import synth
from oracle.workloads import conditioned_decode, decode_trace
from synth import problem as sp
from expert_offload_caching_b200 import abi
from expert_offload_caching_b200.runtime import LayerStack, new_trace, trace_events

REL_L2_MAX = 1e-3  # layer outputs: relative L2 error bound (fp32 accumulation)


def rel_l2(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


@dataclasses.dataclass
class DecodeRun:
    events: list          # (t, layer, expert, slot, hit, evicted)
    y: torch.Tensor       # [T, L, S, d] fp32 on device
    idx: np.ndarray | None
    gates: np.ndarray | None
    table: tuple          # (map, owner, stamp, clock)
    stats: object


class DecodeProblem:
    def __init__(self, shape: synth.LayerShape, T: int, streams: int = 1, P: int | None = None,
                 distinct: int | None = None, C: int | None = None, stream0: int = 0,
                 fmt: int = sp.FMT_NVFP4, shared_fmt: int | None = None):
        self.shape, self.T, self.S = shape, T, streams
        self.fmt = fmt
        self.shared_fmt = fmt if shared_fmt is None else shared_fmt
        self.P = shape.L * shape.E if P is None else P
        self.C = shape.cache_slots if C is None else C
        self.rb = sp.format_record_bytes(fmt, shape.d, shape.F)
        self.srb = sp.format_record_bytes(self.shared_fmt, shape.d, shape.F)
        self.Wr = sp.router_weights(shape)
        self.shared = sp.shared_records_fmt(shape, self.shared_fmt)
        self.pool = sp.pinned_pool_fmt(shape, fmt, self.P, distinct)
        self.pool_np = self.pool.numpy()
        x = np.empty((T, shape.L, streams, shape.d), dtype=np.uint16)
        for s in range(streams):
            for l in range(shape.L):
                x[:, l, s, :] = conditioned_decode(self.Wr[l], shape.k, stream0 + s, l, T)[0]
        self.x = x

    # ---------------------------------------------------------- oracle --
    def oracle_routing(self):
        sh = self.shape
        idx = np.empty((self.T, sh.L, self.S, sh.k), dtype=np.int32)
        gates = np.empty((self.T, sh.L, self.S, sh.k), dtype=np.float64)
        for l in range(sh.L):
            rows = self.x[:, l].reshape(-1, sh.d)
            i, g, _, _ = oracle.route(self.Wr[l], rows, sh.k)
            idx[:, l] = i.reshape(self.T, self.S, sh.k)
            gates[:, l] = g.reshape(self.T, self.S, sh.k)
        return idx, gates

    def oracle_trace(self, idx):
        return decode_trace(idx, self.shape.L, self.shape.E, self.C)

    def oracle_y(self, t: int, l: int) -> np.ndarray:
        sh = self.shape
        shared = None if self.shared is None else self.shared[l * self.srb:(l + 1) * self.srb]
        return oracle.moe_layer(self.pool_np, self.P, l, sh.E, sh.d, sh.F, sh.k, self.Wr[l],
                                shared, self.x[t, l], fmt=self.fmt, shared_fmt=self.shared_fmt)[2]

    # ------------------------------------------------------------- GPU --
    def dims(self):
        sh = self.shape
        return abi.make_dims(sh.L, sh.E, sh.k, sh.d, sh.F, sh.shared, True, self.S,
                             0 if self.P == sh.L * sh.E else self.P, weight_format=self.fmt,
                             shared_format=self.shared_fmt)

    def stack(self) -> LayerStack:
        return LayerStack(self.dims(), self.pool, sp.to_device(self.Wr),
                          sp.to_device(self.shared), self.C)

    def run(self, stack: LayerStack | None = None, routing: bool = False, tokens=None,
            host_io: bool = False) -> DecodeRun:
        sh = self.shape
        own = stack is None
        st = self.stack() if own else stack
        T = self.T if tokens is None else tokens
        xd = torch.from_numpy(self.x[:T]).cuda()
        y = torch.zeros((T, sh.L, self.S, sh.d), dtype=torch.float32, device="cuda")
        if host_io:
            xh = torch.from_numpy(self.x[:T]).pin_memory()
            yh = torch.zeros((T, sh.L, self.S, sh.d), dtype=torch.float32).pin_memory()
        torch.cuda.synchronize()
        tr, arr = new_trace(2 * sh.E + 8)
        events = []
        idx = np.empty((T, sh.L, self.S, sh.k), dtype=np.int32) if routing else None
        gates = np.empty((T, sh.L, self.S, sh.k), dtype=np.float32) if routing else None
        for t in range(T):
            for l in range(sh.L):
                if host_io:
                    st.forward_host(l, xh[t, l], yh[t, l], tr)
                else:
                    st.forward(l, xd[t, l], y[t, l], tr)
                events += [(t, l, e[1], e[2], e[3], e[4]) for e in trace_events(tr, arr)]
                if routing:
                    abi.moe_get_routing(st.ctx, idx[t, l], gates[t, l], self.S)
        st.synchronize()
        if host_io:
            y.copy_(yh)
        m = np.empty(sh.L * sh.E, dtype=np.int32)
        o = np.empty(self.C, dtype=np.int32)
        s = np.empty(self.C, dtype=np.uint64)
        clock = abi.moe_cache_export(st.ctx, m, o, s)
        stats = abi.moe_get_stats(st.ctx)
        run = DecodeRun(events, y, idx, gates, (m, o, s, clock), stats)
        if own:
            self._last_stack = st
        return run

    def check_slots(self, st: LayerStack, owner: np.ndarray, sample: int | None = None):
        """Slot contents: each resident slot holds its owner's record, byte for byte."""
        sh = self.shape
        slots = np.nonzero(owner >= 0)[0]
        if sample is not None and slots.size > sample:
            slots = np.random.default_rng(0).choice(slots, sample, replace=False)
        for s in slots:
            key = int(owner[s])
            r = key % self.P
            want = self.pool[r * self.rb:(r + 1) * self.rb].cuda()
            got = st.arena[int(s) * self.rb:(int(s) + 1) * self.rb]
            assert torch.equal(got, want), f"slot {s} (key {key}) differs from its record"
