"""Benchmark of the per-layer routed-expert step (decode, batch 1) on B200.

Workload (default): gpt-oss-120b-shaped decode -- 36 layers x 128 routed
experts, top-4, d = 2880, SwiGLU F = 2880, NVFP4 expert records (13.997 MB
each, 64.5 GB pool in page-locked host memory), router weights bf16, AR(1)
bf16 hidden states (rho = 0.9), 512 tokens at batch 1, HBM cache of 40% of the
pool (1843 slots), cold at the start of the timed region.

A step is one token through all 36 layers: router + top-k + LRU lookup, miss
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
DISTINCT_RECORDS = 32  # generated records; the rest of the pool repeats them (same bytes moved)


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=512)
    ap.add_argument("--warmup", type=int, default=8)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default="gpt-oss-120b-shaped", choices=list(synth.SHAPES))
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-kernel-timing", action="store_true")
    ap.add_argument("--layers", type=int, default=0, help="override L (small profiling cases)")
    ap.add_argument("--slots", type=int, default=0, help="override the HBM cache slots")
    ap.add_argument("--pool-records", type=int, default=0, help="override the host pool records")
    ap.add_argument("--warm", action="store_true",
                    help="warm up on the timed inputs and keep the cache (all-hit runs)")
    return ap.parse_args()


def dist_setup(n):
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local = int(os.environ.get("LOCAL_RANK", 0))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=600),
                                             device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(v: float, world: int) -> float:
    if world == 1:
        return v
    t = torch.tensor([v], dtype=torch.float64, device="cuda")
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(v: float, world: int) -> float:
    if world == 1:
        return v
    t = torch.tensor([v], dtype=torch.float64, device="cuda")
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


def make_inputs(shape, T, stream0):
    return sp.decode_inputs(shape, T, 1, stream0=stream0)


def run_tokens(stack, x, y, L, host=False):
    for t in range(x.shape[0]):
        for l in range(L):
            if host:
                stack.forward_host(l, x[t, l], y[t, l])
            else:
                stack.forward(l, x[t, l], y[t, l])


def timed(stack, x, y, L, world, host=False):
    barrier(world)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stack.compute)
    run_tokens(stack, x, y, L, host)
    e1.record(stack.compute)
    torch.cuda.synchronize()
    barrier(world)
    return e0.elapsed_time(e1) * 1e-3


def cpu_baseline(shape, pool_np, P, Wr, shared, x, budget_s=12.0):
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
    rb = synth.record_bytes(shape.d, shape.F)
    while True:
        for l in range(L):
            sh = None if shared is None else shared[l * rb:(l + 1) * rb]
            idx, _, _ = oracle.moe_layer(pool_np, P, l, E, shape.d, shape.F, shape.k, Wr[l], sh,
                                         x[tokens % x.shape[0], l])
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
    """The oracle timed on the host cores; each step = one layer of one token."""
    rank = int(os.environ.get("RANK", 0))
    if rank != 0:
        return
    import oracle
    rb = synth.record_bytes(shape.d, shape.F)
    P = min(shape.L * shape.E, DISTINCT_RECORDS)
    pool = np.concatenate([synth.expert_record(i // shape.E, i % shape.E, shape.d, shape.F)
                           for i in range(P)])
    Wr = sp.router_weights(shape)
    shared = sp.shared_records(shape)
    x = make_inputs(shape, max(1, (args.steps + args.warmup) // shape.L + 1), 0)

    def step(i):
        l, t = i % shape.L, i // shape.L
        sh = None if shared is None else shared[l * rb:(l + 1) * rb]
        oracle.moe_layer(pool, P, l, shape.E, shape.d, shape.F, shape.k, Wr[l], sh, x[t, l])

    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        step(args.warmup + i)
    el = time.perf_counter() - t0
    per_layer = el / args.steps
    tok_s = 1.0 / (per_layer * shape.L)
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count()))
    line = {"impl": "reference", "metric": METRIC, "value": tok_s, "unit": "tok/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": per_layer * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "warm_cache": bool(args.warm),
            "config": {"workload": shape.name, "step": "one layer of one token (oracle)"},
            "cpu_baseline": {"value": tok_s, "unit": "tok/s", "cores": cores, "kind": "oracle",
                             "sample": f"{args.steps} layer evaluations (1 token-layer each); "
                                       f"tok/s = 1 / (mean layer time x {shape.L} layers)"},
            "e2e": {"value": tok_s, "unit": "tok/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


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
    from expert_offload_caching_b200 import abi
    from expert_offload_caching_b200.runtime import LayerStack

    L, E, k, d, F = shape.L, shape.E, shape.k, shape.d, shape.F
    rb = synth.record_bytes(d, F)
    # one replica per rank; with several ranks on one host the pools alias so
    # that the host RAM holds about one full pool in total
    P = shape.L * shape.E if world == 1 else max(DISTINCT_RECORDS, (shape.L * shape.E) // world)
    if args.pool_records:
        P = min(args.pool_records, shape.L * shape.E)
    pool = sp.RegisteredPool(shape, P, distinct=DISTINCT_RECORDS)
    Wr = sp.router_weights(shape)
    shared = sp.shared_records(shape)
    dims = abi.make_dims(L, E, k, d, F, shape.shared, True, 1, 0 if P == L * E else P)
    stack = LayerStack(dims, pool.tensor, sp.to_device(Wr), sp.to_device(shared),
                       shape.cache_slots)

    # H2D bandwidth of this machine, measured now (the roofline's PCIe term)
    nb = 1 << 30
    hbuf = torch.empty(nb, dtype=torch.uint8, pin_memory=True)
    dbuf = torch.empty(nb, dtype=torch.uint8, device="cuda")
    h2d = abi.moe_measure_h2d(dbuf, hbuf, nb, 0, 10, stack.copy)
    h2d_rec = abi.moe_measure_h2d(dbuf, hbuf, (nb // rb) * rb, rb, 5, stack.copy)
    del dbuf, hbuf

    x_warm = torch.from_numpy(make_inputs(shape, max(args.warmup, 1), 1000 + rank)).cuda()
    x = torch.from_numpy(make_inputs(shape, args.steps, rank)).cuda()
    y = torch.empty((args.steps, L, 1, d), dtype=torch.float32, device="cuda")
    yw = torch.empty((x_warm.shape[0], L, 1, d), dtype=torch.float32, device="cuda")
    torch.cuda.synchronize()

    # warm-up on other inputs, then a cold cache
    if args.warm:
        run_tokens(stack, x, y, L)
        stack.synchronize()
        abi.moe_get_stats(stack.ctx)
        base = abi.moe_get_stats(stack.ctx)
    else:
        run_tokens(stack, x_warm[:args.warmup], yw, L)
        stack.synchronize()
        stack.reset()
    clocks = ClockSampler(local if world > 1 else 0)
    clocks.start()
    el = timed(stack, x, y, L, world)
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
        timed(stack, x, y, L, world)
        kst = abi.moe_get_stats(stack.ctx)
        abi.moe_set_timing(stack.ctx, False)
        for i in range(abi.MOE_K_COUNT):
            kst.kernel_launches[i] -= before.kernel_launches[i]
            kst.kernel_ms[i] -= before.kernel_ms[i]
            kst.kernel_bytes[i] -= before.kernel_bytes[i]
    el_max = max_over_ranks(el, world)
    tokens_total = sum_over_ranks(float(args.steps), world)
    value = tokens_total / el_max

    # roofline of the step (the benchmark spec): max(hit bytes / HBM BW, miss bytes / H2D BW)
    hbm_peak, peak_kind = measured_peaks()
    hit_bytes = (st.hits + (st.forward_calls if shape.shared else 0)) * rb
    miss_bytes = st.misses * rb
    t_roof = max(hit_bytes / (hbm_peak * 1e9), miss_bytes / (h2d * 1e9))
    t_roof_8tb = max(hit_bytes / 8000e9, miss_bytes / (h2d * 1e9))

    # dominant kernel by device time (from the timed pass with per-kernel events)
    roof, kernels = None, {}
    if kst is not None:
        ms = list(kst.kernel_ms)
        dom = int(np.argmax(ms))
        if kst.kernel_launches[dom] > 0 and ms[dom] > 0:
            achieved = kst.kernel_bytes[dom] / (ms[dom] * 1e-3) / 1e9
            roof = {"kernel": abi.KERNEL_NAMES[dom], "bound": "hbm", "achieved": achieved,
                    "peak": hbm_peak, "unit": "GB/s", "frac": achieved / hbm_peak,
                    "peak_kind": f"{peak_kind} hbm_gbs", "traffic": None,
                    "launches": int(kst.kernel_launches[dom]),
                    "avg_launch_us": ms[dom] * 1e3 / kst.kernel_launches[dom],
                    "bytes_per_launch": kst.kernel_bytes[dom] / kst.kernel_launches[dom]}
        kernels = {abi.KERNEL_NAMES[i]: {"launches": int(kst.kernel_launches[i]),
                                         "ms": round(kst.kernel_ms[i], 3),
                                         "GBps": (kst.kernel_bytes[i] / (kst.kernel_ms[i] * 1e-3) / 1e9
                                                  if kst.kernel_ms[i] > 0 else None)}
                   for i in range(abi.MOE_K_COUNT) if kst.kernel_launches[i]}
    route_phases = {n: round(v / max(st.forward_calls, 1), 3)
                    for n, v in zip(abi.ROUTE_PHASES, st.route_phase_us)}
    launches = int(st.forward_calls * 3 + 2 * st.misses)  # route, hit gate/up, hit down; 2 per miss

    # end to end: host buffers through moe_layer_forward_host
    e2e = None
    if not args.no_e2e:
        stack.reset()
        xh = x.cpu().pin_memory()
        yh = torch.empty((args.steps, L, 1, d), dtype=torch.float32).pin_memory()
        el2 = timed(stack, xh, yh, L, world, host=True)
        e2e = {"value": tokens_total / max_over_ranks(el2, world), "unit": "tok/s",
               "h2d_bytes_per_step": L * d * 2, "d2h_bytes_per_step": L * d * 4}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(shape, pool.array, P, Wr, shared, x.cpu().numpy())

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tok/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": el_max / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "nvfp4 x bf16 -> f32 (w4a16)", "data": "synthetic",
            "warm_cache": bool(args.warm),
            "config": {"workload": f"{shape.name} decode: {L} layers x {E} experts, top-{k}, "
                                   f"d={d}, F={F}, NVFP4 records of {rb} B, batch 1, "
                                   f"{args.steps} tokens, HBM cache {shape.cache_slots} slots "
                                   f"({shape.cache_slots / (L * E):.0%} of the pool), pool "
                                   f"{P * rb / 1e9:.1f} GB pinned host",
                       "l2": "inputs larger than L2 (each step reads "
                             f"{k * L * rb / 1e9:.2f} GB of expert records)",
                       "cold_cache": True, "parallelism": f"replicas x{world}",
                       "pool_distinct_records": DISTINCT_RECORDS},
            "miss_rate": st.misses / max(st.lookups, 1),
            "h2d_gbs": h2d, "h2d_record_gbs": h2d_rec,
            "layer_roofline": {"t_roof_s": t_roof, "t_measured_s": el,
                               "frac": t_roof / el, "frac_at_8tbs": t_roof_8tb / el,
                               "hbm_term_s": hit_bytes / (hbm_peak * 1e9),
                               "h2d_term_s": miss_bytes / (h2d * 1e9),
                               "bw_hbm_gbs": hbm_peak, "bw_h2d_gbs": h2d,
                               "hit_bytes": hit_bytes, "miss_bytes": miss_bytes},
            "roofline": roof, "kernels": kernels, "route_phase_us_per_call": route_phases,
            "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": launches, "clocks": clk,
        }
        print(json.dumps(line), flush=True)
    stack.close()
    pool.close()
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
