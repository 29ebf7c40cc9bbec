"""Benchmark of the per-layer routed-expert step (decode, batch 1) on B200.

Workload (default): DeepSeek-V4-Flash-shaped decode -- 43 layers x 256 routed
experts, top-6 + 1 shared expert, d = 4096, SwiGLU F = 2048, NVFP4 expert
records (14.156 MB each; a 155.8 GB pool, held in page-locked host memory as
far as the host RAM allows, the rest aliased: expert (l, e) reads record
(l*E + e) mod P, so every miss still moves a whole record), router weights
bf16, AR(1) bf16 hidden states (rho = 0.9), 256 tokens at batch 1, HBM cache
of 11% of the pool (1210 slots), cold at the start of the timed region.
Other shapes: --config (gpt-oss-120b-shaped, qwen3.8-flash-next-shaped, ...);
record formats: --format mxfp4, --shared-format bf16.

A step is one token through all layers: router + top-k + LRU lookup, miss
copies over PCIe, expert GEMVs, combine.  value = tokens/s on the device
clock (CUDA events on the library's compute stream, max over ranks).
e2e = the same run through moe_layer_forward_host (x from pinned host memory,
y back to pinned host memory every layer).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402
from synth import problem as sp  # noqa: E402

METRIC = "MoE decode tok/s at batch 1; % of HBM+H2D roofline; expert miss rate"
H2D_SM = {}  # SM-driven H2D rates measured by open_stack
DISTINCT_RECORDS = 32  # generated records; the rest of the pool repeats them (same bytes moved)
PREFILL_ROWS = 4096     # rows of one prefill chunk
STREAMS = 16            # concurrent decode streams
# mode -> (steps, warm-up steps, workload)
MODE_DEFAULTS = {"decode": (256, 8, "deepseek-v4-flash-shaped"),
                 "prefill": (3, 3, "qwen3.8-flash-next-shaped"),
                 "concurrent": (128, 4, "qwen3.8-flash-next-shaped")}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--mode", default="decode", choices=["decode", "prefill", "concurrent"],
                    help="decode: batch-1 tokens (default); prefill: 4096-row chunks, cold cache, "
                         "next-layer prefetch; concurrent: 16 decode streams after one prefill chunk")
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=None)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default=None, choices=list(synth.SHAPES))
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-kernel-timing", action="store_true")
    ap.add_argument("--layers", type=int, default=0, help="override L (small profiling cases)")
    ap.add_argument("--slots", type=int, default=0, help="override the HBM cache slots")
    ap.add_argument("--pool-records", type=int, default=0, help="override the host pool records")
    ap.add_argument("--policy", default="lru", choices=["lru", "static"],
                    help="cache policy: the global LRU (default) or the static per-layer split")
    ap.add_argument("--warm", action="store_true",
                    help="warm up on the timed inputs and keep the cache (all-hit runs)")
    ap.add_argument("--format", default="nvfp4", choices=["nvfp4", "mxfp4"],
                    help="routed expert records (decode): NVFP4 (default) or MXFP4")
    ap.add_argument("--shared-format", default="same", choices=["same", "bf16"],
                    help="shared expert records: the routed format (default) or BF16")
    ap.add_argument("--layer-kernel", action="store_true",
                    help="decode through the persistent layer kernel (one launch per layer, misses gated "
                         "by copy flags) instead of the default launches (hit experts, then a gate/up and "
                         "a down launch per miss, gated by copy events)")
    ap.add_argument("--split-k", action="store_true",
                    help="the default decode launches with the split-K expert kernels instead of the "
                         "streaming ones")
    ap.add_argument("--copy-streams", type=int, default=0, choices=[0, 1, 2],
                    help="decode misses on 1 or 2 copy streams (0: the library's default)")
    ap.add_argument("--head-bytes", type=int, default=0,
                    help="decode: the hit launch's SMs copy this many bytes of each layer's first miss from "
                         "the host pool while the copy engine moves the rest (0: off)")
    ap.add_argument("--split-record-copies", action="store_true",
                    help="decode: two copies per missed record (gate/up prefix, W2) instead of one")
    ap.add_argument("--ep", action="store_true",
                    help="decode with N > 1: expert parallelism (rank r serves experts e %% N == r, its "
                         "own cache; the partial outputs all-reduced per layer) instead of replicas")
    a = ap.parse_args()
    d_steps, d_warm, d_cfg = MODE_DEFAULTS[a.mode]
    a.steps = d_steps if a.steps is None else a.steps
    a.warmup = d_warm if a.warmup is None else a.warmup
    a.config = d_cfg if a.config is None else a.config
    return a


def dist_setup(n, backend: str = "nccl"):
    """One process per GPU (torchrun env).  Replicas only: the process group
    carries the barriers and the max/sum over ranks, no data-path collective.
    backend "gloo" runs the same logic on host tensors (CPU tests)."""
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local = int(os.environ.get("LOCAL_RANK", 0))
    if world > 1:
        import datetime
        if backend == "nccl":
            torch.cuda.set_device(local)
            torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=600),
                                                 device_id=torch.device("cuda", local))
        else:
            torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return rank, world, local


def _reduce_device():
    return "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"


def replica_pool_records(L: int, E: int, world: int) -> int:
    """Host-pool records per replica: the whole pool alone, else an aliased share
    (expert (l, e) -> record (l*E + e) mod P) so that the host RAM holds about one pool."""
    return L * E if world == 1 else max(DISTINCT_RECORDS, (L * E) // world)


def ep_owned(e, rank: int, world: int) -> bool:
    """Expert parallelism: rank r serves the routed experts e with e % world == r."""
    return e % world == rank


def ep_reduce(y, world: int, stream=None) -> None:
    """Sum the ranks' partial layer outputs in place (expert parallelism): an
    all-reduce, ordered on the library's compute stream on GPUs."""
    if world == 1:
        return
    if stream is not None:
        with torch.cuda.stream(stream):
            torch.distributed.all_reduce(y)
    else:
        torch.distributed.all_reduce(y)


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(v: float, world: int) -> float:
    if world == 1:
        return v
    t = torch.tensor([v], dtype=torch.float64, device=_reduce_device())
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(v: float, world: int) -> float:
    if world == 1:
        return v
    t = torch.tensor([v], dtype=torch.float64, device=_reduce_device())
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.SUM)
    return float(t.item())


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms during a region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device: int):
        self.uuid = str(torch.cuda.get_device_properties(device).uuid)
        self.proc = None

    def start(self):
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        uid = self.uuid if self.uuid.startswith("GPU-") else "GPU-" + self.uuid
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", uid, f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        self.proc.wait(timeout=10)
        self.f.seek(0)
        rows = [r.split(",") for r in self.f.read().strip().splitlines() if r.strip()]
        os.unlink(self.f.name)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                smax.append(float(r[2]))
            except (ValueError, IndexError):
                continue
            for nm, v in zip(names, r[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": float(np.median(sm)) if sm else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": sorted(reasons),
                "samples": len(sm)}


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


FP4_PER_BF16 = 4.0  # nominal dense FP4 / BF16 tensor throughput of B200 (9 / 2.25 PFLOP/s)


def measured_fp4_peak():
    """Dense NVFP4 tensor TFLOP/s: the measured bf16 burst figure (the prefill
    GEMMs run between long copy waits) times the nominal FP4/BF16 ratio."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return (FP4_PER_BF16 * float(json.load(f)["bf16_tflops"]),
                    "measured bf16_tflops (burst) x 4 (nominal fp4/bf16)")
    return FP4_PER_BF16 * 1590.0, "fallback bf16 (burst) x 4 (nominal fp4/bf16)"


def make_inputs(shape, T, stream0):
    return sp.decode_inputs(shape, T, 1, stream0=stream0)


def run_tokens(stack, x, y, L, host=False, mark=None, ep_world=1):
    """Tokens t = 0.. through all L layers; mark = (t0, event): the event is
    recorded on the compute stream before token t0.  ep_world > 1: expert
    parallelism, each layer's partial output summed over the ranks before the
    next layer runs."""
    for t in range(x.shape[0]):
        if mark is not None and t == mark[0]:
            mark[1].record(stack.compute)
        for l in range(L):
            if host:
                stack.forward_host(l, x[t, l], y[t, l])
            else:
                stack.forward(l, x[t, l], y[t, l])
            if ep_world > 1:
                ep_reduce(y[t, l], ep_world, None if host else stack.compute)


LAST_STEADY = {}  # steady-window time of the last timed() call: {"t0": first token, "s": seconds}


def timed(stack, x, y, L, world, host=False, ep_world=1):
    """Device seconds of all tokens; also records the steady window (tokens from
    T/4 on, after the cold cache has filled) in LAST_STEADY."""
    barrier(world)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    eq = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    t0 = x.shape[0] // 4
    e0.record(stack.compute)
    torch.cuda.nvtx.range_push("timed")  # lets a profiler select the timed region's launches
    run_tokens(stack, x, y, L, host, mark=(t0, eq) if t0 > 0 else None, ep_world=ep_world)
    torch.cuda.nvtx.range_pop()
    e1.record(stack.compute)
    torch.cuda.synchronize()
    barrier(world)
    LAST_STEADY.clear()
    if t0 > 0:
        LAST_STEADY.update(t0=t0, s=eq.elapsed_time(e1) * 1e-3)
    return e0.elapsed_time(e1) * 1e-3


def oracle_trace_counts(shape, Wr, x, policy, scratch):
    """The oracle's routing of every (token, layer) of the timed input and its
    cache simulator replayed over them (LRU, or the static split): routed
    lookups, hits, misses, evictions.  These are the counts the step's roofline
    is computed from, independent of the GPU's own counters.  x: [T, L, 1, d]."""
    import oracle
    from oracle import LRU
    from oracle.workloads import static_split_trace
    L, E, k = shape.L, shape.E, shape.k
    T = x.shape[0]
    idx = np.empty((T, L, 1, k), dtype=np.int32)
    for l in range(L):  # one call per layer: the oracle routes the rows in parallel
        idx[:, l, 0] = oracle.route(Wr[l], np.ascontiguousarray(x[:, l, 0]), k)[0]
    if policy == "static":
        ev = static_split_trace(idx, L, E, shape.cache_slots, scratch)
        hits = sum(e[4] for e in ev)
        return {"lookups": len(ev), "hits": hits, "misses": len(ev) - hits, "evictions": 0,
                "calls": T * L}
    lru = LRU(L, E, shape.cache_slots)
    lookups = hits = evictions = 0
    for t in range(T):
        for l in range(L):
            for _, _, h, v in lru.batch(l, np.unique(idx[t, l])):
                lookups += 1
                hits += h
                evictions += v >= 0
    return {"lookups": lookups, "hits": hits, "misses": lookups - hits, "evictions": evictions,
            "calls": T * L}


def cpu_baseline(shape, pool_np, P, Wr, shared, x, fmt=sp.FMT_NVFP4, sfmt=sp.FMT_NVFP4,
                 budget_s=12.0):
    """The oracle as it stands, on this host's cores: whole tokens (all layers:
    routing, LRU simulation, W4A16 expert FFNs of the selected experts, combine),
    reading the host pool directly, until about budget_s seconds have passed."""
    import oracle
    from oracle import LRU
    L, E = shape.L, shape.E
    lru = LRU(L, E, shape.cache_slots)
    t0 = time.perf_counter()
    tokens = 0
    layers = 0
    srb = sp.format_record_bytes(sfmt, shape.d, shape.F)
    while True:
        for l in range(L):
            sh = None if shared is None else shared[l * srb:(l + 1) * srb]
            idx, _, _ = oracle.moe_layer(pool_np, P, l, E, shape.d, shape.F, shape.k, Wr[l], sh,
                                         x[tokens % x.shape[0], l], fmt=fmt, shared_fmt=sfmt)
            lru.batch(l, np.unique(idx))
            layers += 1
        tokens += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count()))
    return {"value": tokens / el, "unit": "tok/s", "cores": cores, "kind": "oracle",
            "sample": f"{tokens} token(s) x {L} layers of the same workload, first tokens of "
                      f"the timed input, {el:.1f} s of CPU work"}


def reference_arm(args, shape):
    """The oracle timed on the host cores; each step = one layer of one batch of
    the mode's rows (decode: 1 row, concurrent: STREAMS rows, prefill: a sample
    of 64 rows of the chunk, W4A4)."""
    rank = int(os.environ.get("RANK", 0))
    if rank != 0:
        return
    import oracle
    fmt, sfmt = formats(args)
    if args.mode == "decode" and fmt != sp.FMT_NVFP4:
        rec = synth.expert_record_mx
    else:
        rec, fmt, sfmt = synth.expert_record, sp.FMT_NVFP4, sp.FMT_NVFP4
    srb = sp.format_record_bytes(sfmt, shape.d, shape.F)
    P = min(shape.L * shape.E, DISTINCT_RECORDS)
    pool = np.concatenate([rec(i // shape.E, i % shape.E, shape.d, shape.F) for i in range(P)])
    Wr = sp.router_weights(shape)
    shared = sp.shared_records_fmt(shape, sfmt)
    R = {"decode": 1, "concurrent": STREAMS, "prefill": 64}[args.mode]
    n_tok = max(1, (args.steps + args.warmup) // shape.L + 1)
    if args.mode == "prefill":
        x = np.stack([np.stack([synth.prefill_rows_fast(l, R, shape.d, seed=synth.MASTER_SEED + t)
                                for l in range(shape.L)]) for t in range(n_tok)])
    else:
        x = sp.decode_inputs(shape, n_tok, R)

    def step(i):
        l, t = i % shape.L, i // shape.L
        sh = None if shared is None else shared[l * srb:(l + 1) * srb]
        oracle.moe_layer(pool, P, l, shape.E, shape.d, shape.F, shape.k, Wr[l], sh,
                         np.ascontiguousarray(x[t, l]), w4a4=args.mode == "prefill", fmt=fmt,
                         shared_fmt=sfmt)

    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        step(args.warmup + i)
    el = time.perf_counter() - t0
    per_layer = el / args.steps
    tok_s = R / (per_layer * shape.L)
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count()))
    metric = {"decode": METRIC,
              "prefill": "MoE prefill tok/s (4096-row chunk, cold cache, next-layer prefetch); "
                         "% of HBM+H2D roofline",
              "concurrent": f"MoE concurrent decode tok/s ({STREAMS} streams, aggregate); "
                            "% of HBM+H2D roofline; expert miss rate"}[args.mode]
    line = {"impl": "reference", "metric": metric, "value": tok_s, "unit": "tok/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": per_layer * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "warm_cache": bool(args.warm),
            "config": {"workload": f"{shape.name} {args.mode}",
                       "step": f"one layer of {R} row(s) (oracle)"},
            "cpu_baseline": {"value": tok_s, "unit": "tok/s", "cores": cores, "kind": "oracle",
                             "sample": f"{args.steps} layer evaluations of {R} row(s) each; "
                                       f"tok/s = {R} / (mean layer time x {shape.L} layers)"},
            "e2e": {"value": tok_s, "unit": "tok/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


FMT = {"nvfp4": sp.FMT_NVFP4, "mxfp4": sp.FMT_MXFP4, "bf16": sp.FMT_BF16}
POOL_RAM_SHARE = 0.5  # at most this share of the host's available RAM is pinned for the pool


def host_available_bytes() -> int:
    try:
        with open("/proc/meminfo") as f:
            for ln in f:
                if ln.startswith("MemAvailable:"):
                    return int(ln.split()[1]) * 1024
    except OSError:
        pass
    return 0


def formats(args):
    """(routed format, shared format) codes of the run."""
    fmt = FMT[getattr(args, "format", "nvfp4")]
    sf = getattr(args, "shared_format", "same")
    return fmt, (fmt if sf == "same" else FMT[sf])


def pool_records(args, shape, world, rb) -> tuple[int, str]:
    """Records of the pinned host pool: the whole pool (L*E) when it fits in
    POOL_RAM_SHARE of the available host RAM, else as many as fit, aliased
    (expert (l, e) -> record (l*E + e) mod P: the bytes each miss moves do not
    change).  With several ranks on one host each replica takes a share."""
    L, E = shape.L, shape.E
    if args.pool_records:
        return min(args.pool_records, L * E), "--pool-records"
    P = replica_pool_records(L, E, world)
    avail = host_available_bytes()
    if avail:
        fit = int(POOL_RAM_SHARE * avail / world) // rb
        if fit < P:
            return max(DISTINCT_RECORDS, fit), (f"aliased: {POOL_RAM_SHARE:.0%} of the host's "
                                                f"{avail / 2**30:.0f} GiB available RAM")
    return P, "whole pool" if P == L * E else "replica share"


def open_stack(args, shape, world, max_rows, prefetch=False):
    """The pinned pool, the layer stack and this box's measured H2D bandwidth."""
    from expert_offload_caching_b200 import abi
    from expert_offload_caching_b200.runtime import LayerStack
    L, E = shape.L, shape.E
    fmt, sfmt = formats(args)
    rb = sp.format_record_bytes(fmt, shape.d, shape.F)
    P, args.pool_note = pool_records(args, shape, world, rb)
    pool = sp.RegisteredPool(shape, P, distinct=DISTINCT_RECORDS, fmt=fmt)
    Wr = sp.router_weights(shape)
    shared = sp.shared_records_fmt(shape, sfmt)
    dims = abi.make_dims(L, E, shape.k, shape.d, shape.F, shape.shared, True, max_rows,
                         0 if P == L * E else P, weight_format=fmt, shared_format=sfmt)
    rank = int(os.environ.get("RANK", 0))
    shard = (rank, world) if getattr(args, "ep", False) and world > 1 else (0, 1)
    stack = LayerStack(dims, pool.tensor, sp.to_device(Wr), sp.to_device(shared),
                       shape.cache_slots, prefetch=prefetch,
                       static_split=getattr(args, "policy", "lru") == "static", shard=shard)
    if getattr(args, "layer_kernel", False):
        abi.moe_debug_inject(stack.ctx, 3, 1)
    if getattr(args, "split_k", False):
        abi.moe_debug_inject(stack.ctx, 7, 0)
    if getattr(args, "copy_streams", 0):
        abi.moe_debug_inject(stack.ctx, 6, args.copy_streams)
    if getattr(args, "head_bytes", 0):
        abi.moe_debug_inject(stack.ctx, 10, args.head_bytes)
    if getattr(args, "split_record_copies", False):
        abi.moe_debug_inject(stack.ctx, 11, 1)

    # H2D bandwidth of this machine, measured now (the roofline's PCIe term)
    nb = 1 << 30
    hbuf = torch.empty(nb, dtype=torch.uint8, pin_memory=True)
    dbuf = torch.empty(nb, dtype=torch.uint8, device="cuda")
    h2d = abi.moe_measure_h2d(dbuf, hbuf, nb, 0, 10, stack.copy)
    h2d_rec = abi.moe_measure_h2d(dbuf, hbuf, (nb // rb) * rb, rb, 5, stack.copy)
    # the same through SM loads of mapped host memory (a device-initiated fetch)
    global H2D_SM
    try:
        H2D_SM = {"h2d_sm_gbs": abi.moe_measure_h2d_sm(dbuf, hbuf, nb, 0, 5, stack.copy),
                  "h2d_sm_record_gbs": abi.moe_measure_h2d_sm(dbuf, hbuf, (nb // rb) * rb, rb, 3,
                                                              stack.copy)}
    except abi.MoeError as e:
        H2D_SM = {"h2d_sm_gbs": None, "h2d_sm_note": str(e)}
    del dbuf, hbuf
    return stack, pool, P, rb, Wr, shared, h2d, h2d_rec


def expert_kernels_label(args) -> str:
    if getattr(args, "layer_kernel", False):
        return "persistent layer kernel (misses gated by copy flags)"
    if getattr(args, "split_k", False):
        return "split-K expert kernels: a gate/up and a down launch for the hit experts and per miss"
    if getattr(args, "split_record_copies", False):
        return "streaming expert kernels: one launch for the hit experts, a gate/up and a down launch per miss"
    return "streaming expert kernels: one launch for the hit experts, one per miss (gate/up, then down)"


def main():
    args = parse()
    shape = synth.SHAPES[args.config]
    if args.layers or args.slots:
        import dataclasses
        shape = dataclasses.replace(shape, L=args.layers or shape.L,
                                    cache_slots=args.slots or shape.cache_slots)
    if args.impl == "reference":
        reference_arm(args, shape)
        return
    rank, world, local = dist_setup(args.gpus)
    {"decode": bench_decode, "prefill": bench_prefill,
     "concurrent": bench_concurrent}[args.mode](args, shape, rank, world, local)
    if world > 1:
        torch.distributed.destroy_process_group()


def bench_decode(args, shape, rank, world, local):
    from expert_offload_caching_b200 import abi
    L, E, k, d, F = shape.L, shape.E, shape.k, shape.d, shape.F
    stack, pool, P, rb, Wr, shared, h2d, h2d_rec = open_stack(args, shape, world, 1)
    # expert parallelism: every rank runs the same tokens (one model over N GPUs)
    ep = args.ep and world > 1
    epw = world if ep else 1
    x_warm = torch.from_numpy(make_inputs(shape, max(args.warmup, 1), 1000 + (0 if ep else rank))).cuda()
    x = torch.from_numpy(make_inputs(shape, args.steps, 0 if ep else rank)).cuda()
    y = torch.empty((args.steps, L, 1, d), dtype=torch.float32, device="cuda")
    yw = torch.empty((x_warm.shape[0], L, 1, d), dtype=torch.float32, device="cuda")
    torch.cuda.synchronize()

    # warm-up on other inputs, then a cold cache
    if args.warm:
        run_tokens(stack, x, y, L, ep_world=epw)
        stack.synchronize()
        abi.moe_get_stats(stack.ctx)
        base = abi.moe_get_stats(stack.ctx)
    else:
        run_tokens(stack, x_warm[:args.warmup], yw, L, ep_world=epw)
        stack.synchronize()
        stack.reset()
    clocks = ClockSampler(local if world > 1 else 0)
    clocks.start()
    el = timed(stack, x, y, L, world, ep_world=epw)
    steady = dict(LAST_STEADY)
    clk = clocks.stop()
    st = abi.moe_get_stats(stack.ctx)
    if args.warm:  # counters of the timed region only
        for f in ("lookups", "hits", "misses", "evictions", "h2d_copies", "h2d_bytes", "forward_calls"):
            setattr(st, f, getattr(st, f) - getattr(base, f))
        for i in range(8):
            st.route_phase_us[i] -= base.route_phase_us[i]
    # the same run again (cold cache again) with CUDA events around every kernel
    # launch on the compute stream: per-kernel device time for the roofline
    kst = None
    if not args.no_kernel_timing:
        if not args.warm:
            stack.reset()
        before = abi.moe_get_stats(stack.ctx)
        abi.moe_set_timing(stack.ctx, True)
        timed(stack, x, y, L, world, ep_world=epw)
        kst = stats_delta(abi.moe_get_stats(stack.ctx), before)
        abi.moe_set_timing(stack.ctx, False)
    el_max = max_over_ranks(el, world)
    # replicas: every rank's own tokens; expert parallelism: the same tokens on all ranks
    tokens_total = float(args.steps) if ep else sum_over_ranks(float(args.steps), world)
    value = tokens_total / el_max
    steady_line = None
    if steady:  # tokens T/4 .. T-1, after the cold cache has filled (every rank takes part)
        s_max = max_over_ranks(steady["s"], world)
        steady_tok = float(args.steps - steady["t0"])
        steady_line = {"from_token": steady["t0"], "unit": "tok/s",
                       "value": (steady_tok if ep else sum_over_ranks(steady_tok, world)) / s_max}

    # end to end: host buffers through moe_layer_forward_host
    e2e = None
    if not args.no_e2e and not ep:  # (with expert parallelism the partials are reduced on the device)
        stack.reset()
        xh = x.cpu().pin_memory()
        yh = torch.empty((args.steps, L, 1, d), dtype=torch.float32).pin_memory()
        el2 = timed(stack, xh, yh, L, world, host=True)
        e2e = {"value": tokens_total / max_over_ranks(el2, world), "unit": "tok/s",
               "h2d_bytes_per_step": L * d * 2, "d2h_bytes_per_step": L * d * 4}

    # the CPU-baseline leg (rank 0, one GPU): the oracle's routing + cache
    # simulation over the whole timed input gives the hit and miss counts of
    # the roofline; then the oracle's whole-token throughput on a sample
    fmt, sfmt = formats(args)
    cpu, counts = None, None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        xn = x.cpu().numpy()
        counts = oracle_trace_counts(shape, Wr, xn, args.policy, min(k, E))
        cpu = cpu_baseline(shape, pool.array, P, Wr, shared, xn, fmt, sfmt)
    gpu_counts = {"lookups": st.lookups, "hits": st.hits, "misses": st.misses,
                  "evictions": st.evictions, "calls": st.forward_calls}
    if counts is None or args.warm:
        counts, source = gpu_counts, "gpu counters"
    else:
        source = "oracle trace"

    # roofline of the step: max(hit bytes / HBM BW, miss bytes / H2D BW); hit
    # bytes = routed hits + the shared expert of every call, in the shared format
    hbm_peak, peak_kind = measured_peaks()
    srb = sp.format_record_bytes(sfmt, d, F)
    hit_bytes = counts["hits"] * rb + (counts["calls"] * srb if shape.shared else 0)
    miss_bytes = counts["misses"] * rb
    t_roof = max(hit_bytes / (hbm_peak * 1e9), miss_bytes / (h2d * 1e9))
    t_roof_8tb = max(hit_bytes / 8000e9, miss_bytes / (h2d * 1e9))

    # dominant kernel by device time (from the timed pass with per-kernel timing)
    roof, kernels = None, {}
    if kst is not None:
        roof = hbm_roofline(kst, hbm_peak, peak_kind)
        kernels = kernel_table(kst)
    route_phases = {n: round(v / max(st.forward_calls, 1), 3)
                    for n, v in zip(abi.ROUTE_PHASES, st.route_phase_us)}
    host_phases = host_us_per_call(st)
    launches = launch_count(kst, st)

    if rank == 0:
        fname = {sp.FMT_NVFP4: "NVFP4", sp.FMT_MXFP4: "MXFP4", sp.FMT_BF16: "BF16"}
        shared_txt = (f" + shared ({fname[sfmt]}, {srb} B)" if shape.shared else "")
        line = {
            "metric": METRIC, "value": value, "unit": "tok/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": el_max / args.steps * 1e3,
            "higher_is_better": True, "scaling": "strong" if ep else "weak", "vs_baseline": None,
            "dtype": f"{fname[fmt].lower()} x bf16 -> f32 (w4a16)", "data": "synthetic",
            "warm_cache": bool(args.warm),
            "config": {"workload": f"{shape.name} decode: {L} layers x {E} experts, top-{k}"
                                   f"{shared_txt}, d={d}, F={F}, {fname[fmt]} records of {rb} B, "
                                   f"batch 1, {args.steps} tokens, HBM cache {shape.cache_slots} "
                                   f"slots ({shape.cache_slots / (L * E):.0%} of the pool), pool "
                                   f"{L * E * rb / 1e9:.1f} GB as {P} pinned records "
                                   f"({P * rb / 1e9:.1f} GB; {args.pool_note})",
                       "l2": "inputs larger than L2 (each step reads "
                             f"{k * L * rb / 1e9:.2f} GB of expert records)",
                       "cold_cache": not args.warm,
                       "parallelism": (f"expert parallel x{world} (experts e % {world} per rank, "
                                       f"partial outputs all-reduced per layer)") if ep else f"replicas x{world}",
                       "pool_distinct_records": DISTINCT_RECORDS, "policy": args.policy,
                       "expert_kernels": expert_kernels_label(args),
                       "copy_streams": args.copy_streams or "default",
                       "sm_head_bytes": args.head_bytes,
                       "copies_per_miss": 2 if args.split_record_copies else 1},
            "miss_rate": counts["misses"] / max(counts["lookups"], 1),
            "counts": {"source": source, **counts,
                       "gpu_counters_match": all(gpu_counts[f] == counts[f] for f in counts)},
            "steady_window": steady_line,
            "h2d_gbs": h2d, "h2d_record_gbs": h2d_rec, **H2D_SM,
            "layer_roofline": {"t_roof_s": t_roof, "t_measured_s": el,
                               "frac": t_roof / el, "frac_at_8tbs": t_roof_8tb / el,
                               "hbm_term_s": hit_bytes / (hbm_peak * 1e9),
                               "h2d_term_s": miss_bytes / (h2d * 1e9),
                               "bw_hbm_gbs": hbm_peak, "bw_h2d_gbs": h2d,
                               "hit_bytes": hit_bytes, "miss_bytes": miss_bytes},
            "roofline": roof, "kernels": kernels, "route_phase_us_per_call": route_phases,
            "host_us_per_call": host_phases,
            "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": launches, "clocks": clk,
        }
        print(json.dumps(line), flush=True)
    stack.close()
    pool.close()



def launch_count(kst, st):
    """The library's kernel launches in a timed run: counted per class by the
    timing pass (the same work as the timed run; with the layer kernel, the
    hit-phase class is a part of its launches, not launches of its own);
    without that pass, the per-call structure of the decode path (route + hit
    launch) plus one launch per miss."""
    from expert_offload_caching_b200 import abi
    if kst is not None:
        part = abi.MOE_K_LAYER_HITS if kst.kernel_launches[abi.MOE_K_LAYER] else -1
        return int(sum(kst.kernel_launches[i] for i in range(abi.MOE_K_COUNT) if i != part))
    return int(st.forward_calls * 2 + st.misses)


def host_us_per_call(st):
    """Host time per forward call: inside the call, waiting for the miss list, issuing after it."""
    n = max(st.forward_calls, 1)
    return {k: round(v / n, 2) for k, v in zip(("in_call", "wait_miss_list", "issue_after_list"),
                                                st.host_us)}


def kernel_ms(kst, i):
    """Device time of kernel class i: the summed device spans (first CTA start after
    its dependency wait to last CTA end) where the class is instrumented, else the
    CUDA-event time around the launches (which also counts launch latency and any
    wait for the host or for the previous kernel)."""
    return kst.kernel_span_ms[i] if kst.kernel_span_ms[i] > 0 else kst.kernel_ms[i]


def kernel_table(kst):
    from expert_offload_caching_b200 import abi
    out = {}
    for i in range(abi.MOE_K_COUNT):
        if not kst.kernel_launches[i]:
            continue
        t = kernel_ms(kst, i)
        out[abi.KERNEL_NAMES[i]] = {
            "launches": int(kst.kernel_launches[i]), "ms": round(t, 3),
            "ms_events": round(kst.kernel_ms[i], 3),
            "timing": "device span" if kst.kernel_span_ms[i] > 0 else "events",
            "GBps": kst.kernel_bytes[i] / (t * 1e-3) / 1e9 if t > 0 else None}
    return out


# DRAM traffic per algorithmic byte of a kernel class, from one committed ncu
# capture (dram__bytes_read.sum + dram__bytes_write.sum over the launch's
# algorithmic bytes) of the kernel as it is now; a launch's traffic is this
# ratio times its algorithmic bytes (traffic grows with the weight bytes
# streamed).  A class absent here reports null.
TRAFFIC_RATIO = {
    "expert_hits": (1.0476, "profiles/expert_stream_resident_deepseek-shaped.md"),
}


# Kernel classes whose device time is not bounded by HBM: the whole decode layer
# kernel waits for the PCIe copies of the misses (its HBM-bound part, the
# resident experts, is the class expert_hits).
NOT_HBM_BOUND = {"expert_layer"}


def hbm_roofline(kst, hbm_peak, peak_kind):
    """roofline object of the dominant (most device time) HBM-bound kernel class."""
    from expert_offload_caching_b200 import abi
    times = [0.0 if abi.KERNEL_NAMES[i] in NOT_HBM_BOUND else kernel_ms(kst, i)
             for i in range(abi.MOE_K_COUNT)]
    dom = int(np.argmax(times))
    if not kst.kernel_launches[dom] or times[dom] <= 0:
        return None
    achieved = kst.kernel_bytes[dom] / (times[dom] * 1e-3) / 1e9
    name = abi.KERNEL_NAMES[dom]
    per_launch = kst.kernel_bytes[dom] / kst.kernel_launches[dom]
    ratio = TRAFFIC_RATIO.get(name)
    return {"kernel": name, "bound": "hbm", "achieved": achieved,
            "peak": hbm_peak, "unit": "GB/s", "frac": achieved / hbm_peak,
            "peak_kind": f"{peak_kind} hbm_gbs (burst copy)",
            "traffic": ratio[0] * per_launch if ratio else None,
            "traffic_source": (f"{ratio[1]}: ncu DRAM bytes / algorithmic bytes = {ratio[0]}, "
                               f"times this run's algorithmic bytes per launch") if ratio else None,
            "timing": "device span" if kst.kernel_span_ms[dom] > 0 else "events",
            "launches": int(kst.kernel_launches[dom]),
            "avg_launch_us": times[dom] * 1e3 / kst.kernel_launches[dom],
            "bytes_per_launch": kst.kernel_bytes[dom] / kst.kernel_launches[dom]}


def stats_combine(a, b, sign):
    """Field-wise a + sign * b of two moe_stats."""
    from expert_offload_caching_b200 import abi
    out = abi.moe_stats()
    for f in (f[0] for f in abi.moe_stats._fields_):
        va, vb = getattr(a, f), getattr(b, f)
        if isinstance(va, (int, float)):
            setattr(out, f, va + sign * vb)
        else:
            arr = getattr(out, f)
            for i in range(len(arr)):
                arr[i] = va[i] + sign * vb[i]
    return out


def stats_delta(after, before):
    """Counters of after minus those of before (same context, no reset in between)."""
    return stats_combine(after, before, -1)


def prefill_rows_device(shape, T, seed):
    """[L, T, d] bf16 bit patterns of the prefill chunk (i.i.d. N(0, 1) rows per layer)."""
    x = torch.empty((shape.L, T, shape.d), dtype=torch.int16, device="cuda")
    for l in range(shape.L):
        x[l].copy_(torch.from_numpy(synth.prefill_rows_fast(l, T, shape.d, seed=seed).view(np.int16)))
    return x


def run_chunk(stack, x, y, L, host=False):
    for l in range(L):
        if host:
            stack.forward_host(l, x[l], y)
        else:
            stack.forward(l, x[l], y)


def bench_prefill(args, shape, rank, world, local):
    """Steps of one prefill chunk (PREFILL_ROWS rows) through all L layers, each
    from a cold cache with next-layer prefetch.  value = rows / s."""
    from expert_offload_caching_b200 import abi
    L, E, k, d, F, T = shape.L, shape.E, shape.k, shape.d, shape.F, PREFILL_ROWS
    stack, pool, P, rb, Wr, shared, h2d, h2d_rec = open_stack(args, shape, world, T, prefetch=True)
    xw = prefill_rows_device(shape, T, synth.MASTER_SEED + 1000 + rank)
    x = prefill_rows_device(shape, T, synth.MASTER_SEED + rank)
    y = torch.empty((T, d), dtype=torch.float32, device="cuda")
    torch.cuda.synchronize()
    for _ in range(args.warmup):
        stack.reset()
        run_chunk(stack, xw, y, L)
    stack.synchronize()

    def one_pass(timing, host=False, xs=x, ys=y):
        """args.steps cold-cache chunks; device seconds summed over the chunks, counters summed."""
        total, acc = 0.0, None
        for _ in range(args.steps):
            stack.reset()  # synchronises the previous chunk, empties the cache, zeroes counters
            abi.moe_set_timing(stack.ctx, timing)
            barrier(world)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stack.compute)
            torch.cuda.nvtx.range_push("timed")
            run_chunk(stack, xs, ys, L, host)
            torch.cuda.nvtx.range_pop()
            e1.record(stack.compute)
            torch.cuda.synchronize()
            total += e0.elapsed_time(e1) * 1e-3
            st = abi.moe_get_stats(stack.ctx)
            abi.moe_set_timing(stack.ctx, False)
            acc = st if acc is None else stats_combine(acc, st, 1)
        barrier(world)
        return total, acc

    clocks = ClockSampler(local if world > 1 else 0)
    clocks.start()
    el, st = one_pass(False)
    clk = clocks.stop()
    kst = None if args.no_kernel_timing else one_pass(True)[1]
    el_max = max_over_ranks(el, world)
    rows_total = sum_over_ranks(float(args.steps * T), world)
    value = rows_total / el_max

    hbm_peak, peak_kind = measured_peaks()
    # HBM: every distinct routed expert of a layer (and the shared one) is read at least once
    hit_bytes = (st.lookups + (st.forward_calls if shape.shared else 0)) * rb
    miss_bytes = st.h2d_bytes  # routed misses + next-layer prefetch misses
    t_roof = max(hit_bytes / (hbm_peak * 1e9), miss_bytes / (h2d * 1e9))
    # expert FLOPs: every row x (k routed + shared) experts x (gate, up, down)
    sel = T * (k + (1 if shape.shared else 0))
    flops_gu = 2.0 * sel * 2 * F * d * args.steps * L
    flops_dn = 2.0 * sel * d * F * args.steps * L
    roof, kernels = None, {}
    if kst is not None:
        kernels = kernel_table(kst)
        tpeak, tkind = measured_fp4_peak()
        i_gu, i_dn = abi.KERNEL_NAMES.index("prefill_gate_up"), abi.KERNEL_NAMES.index("prefill_down")
        dom, fl = (i_gu, flops_gu) if kernel_ms(kst, i_gu) >= kernel_ms(kst, i_dn) else (i_dn, flops_dn)
        if kst.kernel_launches[dom] and kernel_ms(kst, dom) > 0:
            # the binding roof of the grouped GEMM: its FLOPs against the FP4 tensor peak, or
            # the expert weights it streams (each read once per layer) against HBM -- with
            # about k*T/E rows per expert its arithmetic intensity sits below the ridge point
            span = kernel_ms(kst, dom) * 1e-3
            wbytes = kst.kernel_bytes[dom]
            tflops, gbs = fl / span / 1e12, wbytes / span / 1e9
            hbm_bound = wbytes / (hbm_peak * 1e9) > fl / (tpeak * 1e12)
            roof = {"kernel": abi.KERNEL_NAMES[dom], "bound": "hbm" if hbm_bound else "tensor",
                    "achieved": gbs if hbm_bound else tflops,
                    "peak": hbm_peak if hbm_bound else tpeak, "unit": "GB/s" if hbm_bound else "TFLOP/s",
                    "frac": gbs / hbm_peak if hbm_bound else tflops / tpeak,
                    "peak_kind": f"{peak_kind} hbm_gbs (burst copy)" if hbm_bound else tkind,
                    "traffic": None,
                    "tensor_tflops": tflops, "tensor_frac": tflops / tpeak, "tensor_peak": tpeak,
                    "hbm_gbs": gbs, "hbm_frac": gbs / hbm_peak,
                    "flop_per_weight_byte": fl / max(wbytes, 1.0),
                    "launches": int(kst.kernel_launches[dom]),
                    "avg_launch_us": kernel_ms(kst, dom) * 1e3 / kst.kernel_launches[dom],
                    "timing": "device span" if kst.kernel_span_ms[dom] > 0 else "events",
                    "flops_per_launch": fl / kst.kernel_launches[dom],
                    "bytes_per_launch": wbytes / kst.kernel_launches[dom],
                    "note": "grouped tcgen05.mma block-scaled FP4 (E2M1 x E2M1), TMA-fed, fp32 "
                            "accumulation in tensor memory"}
        for name, f in (("prefill_gate_up", flops_gu), ("prefill_down", flops_dn)):
            i = abi.KERNEL_NAMES.index(name)
            if kernel_ms(kst, i) > 0 and name in kernels:
                kernels[name]["TFLOPs"] = f / (kernel_ms(kst, i) * 1e-3) / 1e12

    e2e = None
    if not args.no_e2e:
        xh = x.cpu().pin_memory()
        yh = torch.empty((T, d), dtype=torch.float32).pin_memory()
        el2, _ = one_pass(False, host=True, xs=xh, ys=yh)
        e2e = {"value": rows_total / max_over_ranks(el2, world), "unit": "tok/s",
               "h2d_bytes_per_step": L * T * d * 2, "d2h_bytes_per_step": L * T * d * 4}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline_rows(shape, pool.array, P, Wr, shared, x, rows=64, w4a4=True)
    if rank == 0:
        # per layer: logits GEMM, top-k, lookup, scatter, tile plan, quant x, gate/up GEMM,
        # quant h, down GEMM, combine (+ a BF16 shared expert's GEMM, SwiGLU split, GEMM)
        bf16_shared = shape.shared and formats(args)[1] == sp.FMT_BF16
        launches = int(st.forward_calls * (10 + (3 if bf16_shared else 0)))
        line = {
            "metric": "MoE prefill tok/s (4096-row chunk, cold cache, next-layer prefetch); "
                      "% of HBM+H2D roofline",
            "value": value, "unit": "tok/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": el_max / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "nvfp4 x nvfp4 -> f32 (w4a4)", "data": "synthetic",
            "config": {"workload": f"{shape.name} prefill: {T}-row chunk of i.i.d. N(0,1) bf16 rows "
                                   f"through {L} layers x {E} experts, top-{k}"
                                   f"{' + shared' if shape.shared else ''}, d={d}, F={F}, NVFP4 "
                                   f"records of {rb} B, cold cache of {shape.cache_slots} slots per "
                                   f"chunk, next-layer prefetch on",
                       "l2": "inputs larger than L2 (each chunk moves "
                             f"{miss_bytes / max(args.steps, 1) / 1e9:.1f} GB over PCIe)",
                       "cold_cache": True, "parallelism": f"replicas x{world}",
                       "pool_distinct_records": DISTINCT_RECORDS},
            "miss_rate": st.misses / max(st.lookups, 1),
            "prefetch_miss_rate": st.prefetch_misses / max(st.prefetch_lookups, 1),
            "h2d_gbs": h2d, "h2d_record_gbs": h2d_rec, **H2D_SM,
            "layer_roofline": {"t_roof_s": t_roof, "t_measured_s": el, "frac": t_roof / el,
                               "hbm_term_s": hit_bytes / (hbm_peak * 1e9),
                               "h2d_term_s": miss_bytes / (h2d * 1e9),
                               "bw_hbm_gbs": hbm_peak, "bw_h2d_gbs": h2d,
                               "hit_bytes": hit_bytes, "miss_bytes": miss_bytes,
                               "h2d_achieved_gbs": miss_bytes / el / 1e9},
            "expert_tflop": (flops_gu + flops_dn) / 1e12,
            "host_us_per_call": host_us_per_call(st),
            "roofline": roof, "kernels": kernels, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": launches, "clocks": clk,
        }
        print(json.dumps(line), flush=True)
    stack.close()
    pool.close()


def bench_concurrent(args, shape, rank, world, local):
    """STREAMS decode streams at batch STREAMS after one (untimed) prefill chunk
    on the same cache: each step is one token of every stream through all L layers."""
    from expert_offload_caching_b200 import abi
    L, E, k, d, F, S = shape.L, shape.E, shape.k, shape.d, shape.F, STREAMS
    stack, pool, P, rb, Wr, shared, h2d, h2d_rec = open_stack(args, shape, world, PREFILL_ROWS,
                                                              prefetch=True)
    xp = prefill_rows_device(shape, PREFILL_ROWS, synth.MASTER_SEED + rank)
    yp = torch.empty((PREFILL_ROWS, d), dtype=torch.float32, device="cuda")
    x_warm = torch.from_numpy(sp.decode_inputs(shape, max(args.warmup, 1), S,
                                               stream0=1000 + S * rank)).cuda()
    x = torch.from_numpy(sp.decode_inputs(shape, args.steps, S, stream0=S * rank)).cuda()
    y = torch.empty((args.steps, L, S, d), dtype=torch.float32, device="cuda")
    yw = torch.empty((x_warm.shape[0], L, S, d), dtype=torch.float32, device="cuda")
    torch.cuda.synchronize()
    run_tokens(stack, x_warm[:args.warmup], yw, L)

    def prefilled():
        stack.reset()
        run_chunk(stack, xp, yp, L)
        stack.synchronize()
        return abi.moe_get_stats(stack.ctx)

    base = prefilled()
    clocks = ClockSampler(local if world > 1 else 0)
    clocks.start()
    el = timed(stack, x, y, L, world)
    clk = clocks.stop()
    st = stats_delta(abi.moe_get_stats(stack.ctx), base)
    kst = None
    if not args.no_kernel_timing:
        b2 = prefilled()
        abi.moe_set_timing(stack.ctx, True)
        timed(stack, x, y, L, world)
        abi.moe_set_timing(stack.ctx, False)
        kst = stats_delta(abi.moe_get_stats(stack.ctx), b2)
    el_max = max_over_ranks(el, world)
    tokens_total = sum_over_ranks(float(args.steps * S), world)
    value = tokens_total / el_max

    hbm_peak, peak_kind = measured_peaks()
    hit_bytes = (st.hits + (st.forward_calls if shape.shared else 0)) * rb
    miss_bytes = st.misses * rb
    t_roof = max(hit_bytes / (hbm_peak * 1e9), miss_bytes / (h2d * 1e9))
    roof, kernels = None, {}
    if kst is not None:
        kernels = kernel_table(kst)
        roof = hbm_roofline(kst, hbm_peak, peak_kind)

    e2e = None
    if not args.no_e2e:
        prefilled()
        xh = x.cpu().pin_memory()
        yh = torch.empty((args.steps, L, S, d), dtype=torch.float32).pin_memory()
        el2 = timed(stack, xh, yh, L, world, host=True)
        e2e = {"value": tokens_total / max_over_ranks(el2, world), "unit": "tok/s",
               "h2d_bytes_per_step": L * S * d * 2, "d2h_bytes_per_step": L * S * d * 4}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline_rows(shape, pool.array, P, Wr, shared, x[0], rows=S, w4a4=False)
    if rank == 0:
        line = {
            "metric": f"MoE concurrent decode tok/s ({S} streams, aggregate); "
                      "% of HBM+H2D roofline; expert miss rate",
            "value": value, "unit": "tok/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": el_max / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "nvfp4 x bf16 -> f32 (w4a16)", "data": "synthetic",
            "per_stream_tok_s": value / (S * world),
            "config": {"workload": f"{shape.name} concurrent decode: {S} AR(1) streams x "
                                   f"{args.steps} tokens at batch {S}, after one {PREFILL_ROWS}-row "
                                   f"prefill chunk on the same cache; {L} layers x {E} experts, "
                                   f"top-{k}{' + shared' if shape.shared else ''}, d={d}, F={F}, "
                                   f"cache {shape.cache_slots} slots",
                       "l2": "inputs larger than L2 (each step reads the union of the streams' "
                             "experts over all layers)",
                       "cold_cache": False, "parallelism": f"replicas x{world}",
                       "pool_distinct_records": DISTINCT_RECORDS},
            "miss_rate": st.misses / max(st.lookups, 1),
            "experts_per_layer_step": st.lookups / max(st.forward_calls, 1),
            "host_us_per_call": host_us_per_call(st),
            "h2d_gbs": h2d, "h2d_record_gbs": h2d_rec, **H2D_SM,
            "layer_roofline": {"t_roof_s": t_roof, "t_measured_s": el, "frac": t_roof / el,
                               "hbm_term_s": hit_bytes / (hbm_peak * 1e9),
                               "h2d_term_s": miss_bytes / (h2d * 1e9),
                               "bw_hbm_gbs": hbm_peak, "bw_h2d_gbs": h2d,
                               "hit_bytes": hit_bytes, "miss_bytes": miss_bytes},
            "roofline": roof, "kernels": kernels, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": launch_count(kst, st), "clocks": clk,
        }
        print(json.dumps(line), flush=True)
    stack.close()
    pool.close()


def cpu_baseline_rows(shape, pool_np, P, Wr, shared, x, rows, w4a4, budget_s=12.0):
    """The oracle on this host's cores over batches of `rows` rows, layer after
    layer, until about budget_s seconds have passed; tok/s = rows per whole pass
    of all layers.  x: device or host [L, >=rows, d] bf16 bits."""
    import oracle
    L, E = shape.L, shape.E
    rb = synth.record_bytes(shape.d, shape.F)
    xs = x[:, :rows].cpu().numpy().view(np.uint16) if hasattr(x, "cpu") else x[:, :rows]
    t0 = time.perf_counter()
    layers = 0
    while True:
        l = layers % L
        sh = None if shared is None else shared[l * rb:(l + 1) * rb]
        oracle.moe_layer(pool_np, P, l, E, shape.d, shape.F, shape.k, Wr[l], sh,
                         np.ascontiguousarray(xs[l]), w4a4=w4a4)
        layers += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count()))
    return {"value": rows * layers / L / el, "unit": "tok/s", "cores": cores, "kind": "oracle",
            "sample": f"{layers} layer evaluation(s) of {rows} rows (first rows of the timed "
                      f"input), {el:.1f} s of CPU work; tok/s = rows x layers / {L} / s"}


if __name__ == "__main__":
    main()
