"""Decode path on the GPU against the CPU oracle, through the C ABI.

Bit-exact: expert indices, the cache event sequence (hit/miss, slot,
evicted key), the table (map, owners, stamps, clock) and slot contents.
Within 1e-3 relative L2: the layer outputs."""
import numpy as np
import pytest
import torch

import oracle
import synth
from synth import problem as sp
from expert_offload_caching_b200 import abi
from tests.gpu_problem import REL_L2_MAX, DecodeProblem, rel_l2

pytestmark = pytest.mark.gpu

# Several GEMV tiles, ragged K tails (d = 960: 15 chunks of 64; F = 320: 5 chunks),
# E not a multiple of 32, shared expert, 3 layers.
MID = synth.LayerShape("mid", L=3, E=40, k=5, d=960, F=320, shared=True, tokens=24, cache_slots=12)


def _check_run(pb: DecodeProblem, run, samples=None):
    idx, gates = pb.oracle_routing()
    want_events, lru = pb.oracle_trace(idx)
    assert len(run.events) == len(want_events)
    for g, w in zip(run.events, want_events):
        assert g == w, (g, w)
    m, o, s, c = lru.state()
    np.testing.assert_array_equal(run.table[0], m)
    np.testing.assert_array_equal(run.table[1], o)
    np.testing.assert_array_equal(run.table[2], s)
    assert run.table[3] == c
    if run.idx is not None:
        np.testing.assert_array_equal(run.idx, idx)
        np.testing.assert_allclose(run.gates, gates, rtol=2e-5, atol=1e-7)
    pairs = [(t, l) for t in range(pb.T) for l in range(pb.shape.L)] if samples is None else samples
    y = run.y.cpu().numpy()
    worst = 0.0
    for t, l in pairs:
        e = rel_l2(y[t, l], pb.oracle_y(t, l))
        worst = max(worst, e)
        assert e <= REL_L2_MAX, (t, l, e)
    hits = sum(ev[4] for ev in run.events)
    assert run.stats.lookups == len(run.events) and run.stats.hits == hits
    assert run.stats.misses == len(run.events) - hits
    return worst


def test_tiny_decode_full_parity():
    pb = DecodeProblem(synth.TINY, T=64)
    run = pb.run(routing=True)
    worst = _check_run(pb, run)
    assert worst < 1e-5
    pb.check_slots(pb._last_stack, run.table[1])
    assert 0 < run.stats.misses < run.stats.lookups


def test_mid_shape_multi_layer_shared_expert():
    pb = DecodeProblem(MID, T=24)
    run = pb.run(routing=True)
    assert _check_run(pb, run) < 1e-5
    pb.check_slots(pb._last_stack, run.table[1])


@pytest.mark.parametrize("S", [2, 5, 16])
def test_batched_decode_rows(S):
    C = min(S * MID.k, MID.E) + 6
    pb = DecodeProblem(MID, T=8, streams=S, C=C, stream0=100)
    run = pb.run(routing=True)
    assert _check_run(pb, run) < 1e-5
    pb.check_slots(pb._last_stack, run.table[1])


def test_all_resident_cache_has_no_misses_after_first_use():
    pb = DecodeProblem(synth.TINY, T=40, C=synth.TINY.E)
    run = pb.run()
    _check_run(pb, run)
    firsts = {}
    for ev in run.events:
        key = ev[2]
        if key in firsts:
            assert ev[4] == 1  # resident forever once loaded
        else:
            firsts[key] = ev
            assert ev[4] == 0 and ev[5] == -1
    assert run.stats.evictions == 0


def test_topk_equal_to_E_and_top1():
    for k in (1, 16):
        sh = synth.LayerShape(f"tiny-k{k}", L=2, E=16, k=k, d=256, F=512, shared=False,
                              tokens=6, cache_slots=16)
        pb = DecodeProblem(sh, T=6)
        run = pb.run(routing=True)
        _check_run(pb, run)


def test_host_io_path_matches_device_path():
    pb = DecodeProblem(MID, T=6)
    a = pb.run()
    b = pb.run(host_io=True)
    assert a.events == b.events
    assert torch.equal(a.y, b.y)


def test_cache_persists_across_calls_and_reset_clears_it():
    pb = DecodeProblem(synth.TINY, T=20)
    st = pb.stack()
    r1 = pb.run(stack=st)
    st.reset()
    r2 = pb.run(stack=st)
    assert r1.events == r2.events  # reset = cold start again
    assert r2.stats.lookups == len(r2.events)  # counters restart at the reset


@pytest.mark.parametrize("name,T,samples", [
    ("gpt-oss-120b-shaped", 512, 6),
    ("qwen3.8-flash-next-shaped", 256, 6),
    ("deepseek-v4-flash-shaped", 256, 4),
])
def test_full_size_decode_trace_and_sampled_outputs(name, T, samples):
    """The bench's configurations at full size and full token count: the whole
    routing and cache trace bit-exact, outputs on sampled (token, layer) pairs.
    The host pool holds 97 distinct records; expert (l, e) reads record
    (l*E + e) mod 97 (the C ABI's pool aliasing)."""
    sh = synth.SHAPES[name]
    pb = DecodeProblem(sh, T=T, P=97)
    run = pb.run()
    rng = np.random.default_rng(1)
    pairs = [(int(rng.integers(T)), int(rng.integers(sh.L))) for _ in range(samples)]
    pairs.append((T - 1, sh.L - 1))
    _check_run(pb, run, samples=pairs)
    pb.check_slots(pb._last_stack, run.table[1], sample=24)
    miss_rate = run.stats.misses / run.stats.lookups
    assert 0.0 < miss_rate < 1.0


def test_errors_capacity_and_unpinned_pool():
    sh = synth.TINY
    pb = DecodeProblem(sh, T=2)
    st = pb.stack()
    with pytest.raises(abi.MoeError) as ei:
        abi.cache_configure(st.ctx, 1, st.arena, st.arena.numel(), abi.MOE_CACHE_RESET)
    assert ei.value.status == abi.MOE_ERR_CAPACITY
    with pytest.raises(abi.MoeError) as ei:  # prefetch needs two layers' worth of slots
        abi.cache_configure(st.ctx, 4, st.arena, st.arena.numel(),
                            abi.MOE_CACHE_RESET | abi.MOE_CACHE_PREFETCH_NEXT)
    assert ei.value.status == abi.MOE_ERR_CAPACITY
    pageable = np.zeros(pb.pool.numel(), dtype=np.uint8)
    with pytest.raises(abi.MoeError) as ei:
        abi.moe_layer_init(pb.dims(), pageable, pageable.size, st.router_w, None, st.ws,
                           st.ws.numel(), st.compute, st.copy)
    assert ei.value.status == abi.MOE_ERR_NOT_PINNED
    with pytest.raises(abi.MoeError) as ei:
        st.forward(1, torch.zeros((1, sh.d), dtype=torch.uint16, device="cuda"),
                   torch.zeros((1, sh.d), device="cuda"))
    assert ei.value.status == abi.MOE_ERR_ARG


def test_injected_timeout_then_reset_recovers():
    pb = DecodeProblem(synth.TINY, T=10)
    st = pb.stack()
    abi.moe_set_wait_limit(st.ctx, 0.2)
    abi.moe_debug_inject(st.ctx, 2, 1)  # the next lookup does not publish its miss list
    x = torch.from_numpy(pb.x[0, 0]).cuda()
    y = torch.zeros((1, pb.shape.d), device="cuda")
    torch.cuda.synchronize()
    with pytest.raises(abi.MoeError) as ei:
        st.forward(0, x, y)
    assert ei.value.status == abi.MOE_ERR_TIMEOUT
    with pytest.raises(abi.MoeError) as ei:
        st.forward(0, x, y)
    assert ei.value.status == abi.MOE_ERR_STATE
    st.reset()
    abi.moe_set_wait_limit(st.ctx, 60.0)
    run = pb.run(stack=st)
    _check_run(pb, run)


def test_injected_copy_failure_then_reset_recovers():
    pb = DecodeProblem(synth.TINY, T=10)
    st = pb.stack()
    abi.moe_debug_inject(st.ctx, 1, 3)  # the third H2D copy issue fails
    x = torch.from_numpy(pb.x[:, 0]).cuda()
    y = torch.zeros((10, 1, pb.shape.d), device="cuda")
    torch.cuda.synchronize()
    failed = None
    for t in range(10):
        try:
            st.forward(0, x[t], y[t])
        except abi.MoeError as e:
            failed = e
            break
    assert failed is not None and failed.status == abi.MOE_ERR_CUDA
    with pytest.raises(abi.MoeError) as ei:
        st.forward(0, x[0], y[0])
    assert ei.value.status == abi.MOE_ERR_STATE
    st.reset()
    _check_run(pb, pb.run(stack=st))


def test_h2d_measurement():
    n = 256 << 20
    h = torch.empty(n, dtype=torch.uint8, pin_memory=True)
    d = torch.empty(n, dtype=torch.uint8, device="cuda")
    s = torch.cuda.Stream()
    gbs = abi.moe_measure_h2d(d, h, n, 0, 3, s)
    gbs_rec = abi.moe_measure_h2d(d, h, n, synth.record_bytes(2880, 2880), 3, s)
    assert 5.0 < gbs < 200.0 and 5.0 < gbs_rec < 200.0
    with pytest.raises(abi.MoeError) as ei:
        abi.moe_measure_h2d(d, np.zeros(16, np.uint8), 16, 0, 1, s)
    assert ei.value.status == abi.MOE_ERR_NOT_PINNED


def test_h2d_sm_measurement_copies_the_bytes():
    n = 64 << 20
    h = torch.randint(0, 256, (n,), dtype=torch.uint8).pin_memory()
    d = torch.zeros(n, dtype=torch.uint8, device="cuda")
    s = torch.cuda.Stream()
    torch.cuda.synchronize()
    gbs = abi.moe_measure_h2d_sm(d, h, n, 0, 1, s)
    s.synchronize()
    assert torch.equal(d.cpu(), h)
    d.zero_()
    torch.cuda.synchronize()
    gbs_rec = abi.moe_measure_h2d_sm(d, h, n - 4096, synth.record_bytes(2048, 768), 1, s)
    s.synchronize()
    assert torch.equal(d[:n - 4096].cpu(), h[:n - 4096]) and int(d[n - 4096:].sum()) == 0
    assert 1.0 < gbs < 200.0 and 1.0 < gbs_rec < 200.0
    with pytest.raises(abi.MoeError) as ei:
        abi.moe_measure_h2d_sm(d, h, 24, 0, 1, s)  # not a multiple of 16
    assert ei.value.status == abi.MOE_ERR_ARG


@pytest.mark.parametrize("S", [1, 5])
def test_static_split_policy_trace_and_outputs(S):
    """The static per-layer split: fixed resident experts per layer, misses into
    scratch slots; events bit-exact against the oracle's simulator, the resident
    slots hold their records, outputs within the bar."""
    from oracle.workloads import static_split_trace
    from expert_offload_caching_b200.runtime import LayerStack
    R = min(S * MID.k, MID.E)
    C = 3 * MID.L + R + 2  # 3 resident experts per layer (2 slots left over)
    pb = DecodeProblem(MID, T=6, streams=S, C=C, stream0=200)
    st = LayerStack(pb.dims(), pb.pool, sp.to_device(pb.Wr), sp.to_device(pb.shared), C,
                    static_split=True)
    run = pb.run(stack=st, routing=True)
    idx, gates = pb.oracle_routing()
    np.testing.assert_array_equal(run.idx, idx)
    assert run.events == static_split_trace(idx, MID.L, MID.E, C, R)
    m, o = run.table[0], run.table[1]
    for l in range(MID.L):
        for e in range(MID.E):
            assert m[l * MID.E + e] == (l * 3 + e if e < 3 else -1)
    assert all(o[s] == (s // 3) * MID.E + s % 3 for s in range(3 * MID.L))
    assert all(o[s] == -1 for s in range(3 * MID.L, C))
    pb.check_slots(st, o)
    y = run.y.cpu().numpy()
    for t in range(pb.T):
        for l in range(MID.L):
            assert rel_l2(y[t, l], pb.oracle_y(t, l)) <= REL_L2_MAX
    hits = sum(ev[4] for ev in run.events)
    assert run.stats.hits == hits and run.stats.misses == len(run.events) - hits > 0
    assert run.stats.evictions == 0
    with pytest.raises(abi.MoeError) as ei:  # no next-layer prefetch with the static split
        abi.cache_configure(st.ctx, C, st.arena, st.arena.numel(),
                            abi.MOE_CACHE_RESET | abi.MOE_CACHE_STATIC_SPLIT | abi.MOE_CACHE_PREFETCH_NEXT)
    assert ei.value.status == abi.MOE_ERR_ARG
    st.close()


def test_host_io_unaligned_buffers_take_the_copy_path():
    """Decode with host buffers: aligned pinned buffers are read and written in
    place (mapped), unaligned ones go through staging copies; same results."""
    pb = DecodeProblem(MID, T=3)
    a = pb.run()
    st = pb.stack()
    sh = MID
    n = pb.T * sh.L * sh.d
    xh = torch.empty(n + 8, dtype=torch.int16).pin_memory()
    yh = torch.empty(pb.T * sh.L * sh.d + 4, dtype=torch.float32).pin_memory()
    xv = xh[1:1 + n].view(pb.T, sh.L, 1, sh.d)  # 2 bytes off the allocation's alignment
    yv = yh[1:1 + pb.T * sh.L * sh.d].view(pb.T, sh.L, 1, sh.d)
    xv.copy_(torch.from_numpy(pb.x.view(np.int16)))
    for t in range(pb.T):
        for l in range(sh.L):
            st.forward_host(l, xv[t, l], yv[t, l])
    st.synchronize()
    assert torch.equal(yv.cuda(), a.y)
    st.close()


def test_non_finite_rows_select_valid_experts_like_the_oracle():
    """Rows holding -inf, NaN and +inf through the whole decode step: the
    selection rule (NaN logits as -inf, ties to the lower id) gives valid ids,
    equal to the oracle's; the cache trace and table follow the oracle's LRU;
    finite rows keep their outputs, non-finite rows give non-finite outputs
    (no fault, no out-of-range index)."""
    pb = DecodeProblem(MID, T=4)
    bad = {(1, 0, 3): -np.inf, (2, 1, 5): np.nan, (3, 2, 0): np.inf}
    for (t, l, c), v in bad.items():
        pb.x[t, l, 0, c] = synth.to_bf16(np.array([v], np.float32))[0]
    run = pb.run(routing=True)
    idx, gates = pb.oracle_routing()
    np.testing.assert_array_equal(run.idx, idx)
    assert run.idx.min() >= 0 and run.idx.max() < MID.E
    np.testing.assert_allclose(run.gates, gates, rtol=2e-5, atol=1e-7)  # NaN where the oracle has NaN
    want_events, lru = pb.oracle_trace(idx)
    assert run.events == want_events
    m, o, s, c = lru.state()
    np.testing.assert_array_equal(run.table[0], m)
    np.testing.assert_array_equal(run.table[1], o)
    np.testing.assert_array_equal(run.table[2], s)
    y = run.y.cpu().numpy()
    for t in range(pb.T):
        for l in range(MID.L):
            if (t, l) in {(k[0], k[1]) for k in bad}:
                assert not np.isfinite(y[t, l]).all()
            else:
                assert rel_l2(y[t, l], pb.oracle_y(t, l)) <= REL_L2_MAX


def test_forward_rejects_unaligned_activations_before_launching():
    pb = DecodeProblem(synth.TINY, T=1)
    st = pb.stack()
    d = synth.TINY.d
    xs = torch.zeros(d + 8, dtype=torch.uint16, device="cuda")
    ys = torch.zeros(d + 4, dtype=torch.float32, device="cuda")
    for xv, yv in [(xs[1:1 + d], ys[:d]), (xs[:d], ys.view(torch.uint8)[1:1 + 4 * d])]:
        with pytest.raises(abi.MoeError) as ei:
            abi.moe_layer_forward(st.ctx, 0, xv, 1, yv, None)
        assert ei.value.status == abi.MOE_ERR_ARG
    # nothing ran: the context is usable and the cache still cold
    run = pb.run(stack=st)
    assert run.stats.lookups == len(run.events) > 0
    st.close()


def test_layer_kernel_path_matches_the_oracle():
    """The persistent layer kernel (one launch per layer, misses gated by copy
    flags) instead of the default launches: same trace, table, slots and
    outputs; then back to the default on the same cache."""
    pb = DecodeProblem(MID, T=12)
    st = pb.stack()
    abi.moe_debug_inject(st.ctx, 3, 1)
    run = pb.run(stack=st, routing=True)
    assert _check_run(pb, run) < 1e-5
    pb.check_slots(st, run.table[1])
    abi.moe_debug_inject(st.ctx, 3, 0)
    st.close()


@pytest.mark.parametrize("T", [1, 5])
def test_split_k_per_miss_kernels_match_the_oracle(T):
    """The per-miss path with the split-K expert kernels (expert_gemv.cu)
    instead of the streaming ones: same trace, table, slots and outputs."""
    pb = DecodeProblem(MID, T=12, streams=T, C=min(T * MID.k, MID.E) + 6)
    st = pb.stack()
    abi.moe_debug_inject(st.ctx, 7, 0)
    run = pb.run(stack=st, routing=True)
    assert _check_run(pb, run) < 1e-5
    pb.check_slots(st, run.table[1])
    st.close()


@pytest.mark.parametrize("path", [1, 0], ids=["layer-kernel", "per-miss"])
def test_two_copy_streams_match_the_oracle(path):
    """Misses alternating between the caller's copy stream and the library's
    second one, on both decode paths: same trace, table, slots and outputs.
    Several misses per call (12 rows, cold cache), so both streams carry copies
    in the same call; the cache then persists across calls."""
    pb = DecodeProblem(MID, T=12)
    st = pb.stack()
    abi.moe_debug_inject(st.ctx, 3, path)
    abi.moe_debug_inject(st.ctx, 6, 2)
    run = pb.run(stack=st, routing=True)
    assert _check_run(pb, run) < 1e-5
    pb.check_slots(st, run.table[1])
    assert run.stats.misses >= 2 * pb.T // 3  # the calls held several misses each
    st.close()


def _launches(st):
    ks = abi.moe_get_stats(st.ctx)
    return {n: int(ks.kernel_launches[i]) for i, n in enumerate(abi.KERNEL_NAMES)}


def test_one_launch_per_miss_by_default():
    """Default path: one hit launch per call and one launch per miss (its whole
    record copied, then gate/up and down in the same launch, the down tiles
    waiting for the gate/up tiles inside it; the last one combines): outputs,
    trace, table and slots match the oracle."""
    pb = DecodeProblem(MID, T=12)
    st = pb.stack()
    abi.moe_set_timing(st.ctx, True)
    run = pb.run(stack=st, routing=True)
    assert _check_run(pb, run) < 1e-5
    pb.check_slots(st, run.table[1])
    n = _launches(st)
    calls = pb.T * MID.L
    assert n["expert_hits"] == calls and n["route_lookup"] == calls
    assert n["expert_miss"] == run.stats.misses > calls // 2
    assert n["gate_up"] == n["down"] == 0
    st.close()


# d = 4096: a gate/up tile is 36 KB (NVFP4) or 34 KB (MXFP4), so only 5 stages fit
# (five groups of three warps, one stage each)
WIDE = synth.LayerShape("wide", L=2, E=16, k=4, d=4096, F=256, shared=True, tokens=6, cache_slots=10)


@pytest.mark.parametrize("fmt", [sp.FMT_NVFP4, sp.FMT_MXFP4], ids=["nvfp4", "mxfp4"])
@pytest.mark.parametrize("S", [1, 3])
def test_large_tiles_match_the_oracle(fmt, S):
    """Large tiles (one stage per consumer group; 1 row with activations in
    shared memory, 3 rows from global memory), the hit launch and every miss
    launch: trace, table, slots and outputs match the oracle."""
    pb = DecodeProblem(WIDE, T=6, streams=S, fmt=fmt, C=min(S * WIDE.k, WIDE.E) + 4)
    st = pb.stack()
    run = pb.run(stack=st, routing=True)
    assert _check_run(pb, run) < 1e-5
    pb.check_slots(st, run.table[1])
    assert 0 < run.stats.misses < run.stats.lookups
    st.close()


def test_split_record_copies_match_the_oracle():
    """Each missed record as two copies (the gate/up prefix, then W2, each with
    its event) and a gate/up and a down launch instead of one of each: same
    trace, table, slots and outputs."""
    pb = DecodeProblem(MID, T=12)
    st = pb.stack()
    abi.moe_debug_inject(st.ctx, 11, 1)
    abi.moe_set_timing(st.ctx, True)
    run = pb.run(stack=st, routing=True)
    assert _check_run(pb, run) < 1e-5
    pb.check_slots(st, run.table[1])
    n = _launches(st)
    assert n["gate_up"] == n["down"] == run.stats.misses > 0 and n["expert_miss"] == 0
    st.close()


@pytest.mark.parametrize("frac", [0.1, 0.9], ids=["head-in-gate-up", "head-past-gate-up"])
def test_sm_head_copy_of_the_first_miss_matches_the_oracle(frac):
    """The hit launch's SMs copy the head of each layer's first miss from the
    page-locked pool (through its device address) and the copy engine the rest:
    the slots are bit-exact and the outputs match the oracle, with the head
    ending inside the gate/up prefix and past it."""
    pb = DecodeProblem(MID, T=12)
    st = pb.stack()
    rb = synth.record_bytes(MID.d, MID.F)
    head = int(frac * rb) // 16 * 16
    abi.moe_debug_inject(st.ctx, 10, head)
    run = pb.run(stack=st, routing=True)
    assert _check_run(pb, run) < 1e-5
    pb.check_slots(st, run.table[1])
    assert run.stats.misses > 0
    st.close()


def test_streaming_kernel_wait_runs_out_then_reset_recovers():
    """CTA 0 of the next streaming launches issues no copies for its first work
    item: the consumer's bounded wait on that stage runs out (limit 0.3 s), the
    CTA records the failed check in the mapped page, lets its other copies land
    and returns -- nothing hangs, the context stays usable.  The next call
    reports it (MOE_ERR_CUDA, device check 42-44), a reset brings the context
    back, and a full run matches the oracle."""
    import time
    pb = DecodeProblem(synth.TINY, T=8)
    st = pb.stack()
    abi.moe_set_wait_limit(st.ctx, 0.3)
    abi.moe_debug_inject(st.ctx, 8, 3)  # the next three streaming launches
    x = torch.from_numpy(pb.x[:, 0]).cuda()
    y = torch.zeros((pb.T, 1, pb.shape.d), device="cuda")
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    st.forward(0, x[0], y[0])
    st.synchronize()
    assert time.perf_counter() - t0 < 10.0
    with pytest.raises(abi.MoeError) as ei:
        st.forward(0, x[1], y[1])
    assert ei.value.status == abi.MOE_ERR_CUDA
    msg = abi.moe_last_error(st.ctx)
    assert any(f"device check {c}" in msg for c in (42, 43, 44)), msg
    abi.moe_debug_inject(st.ctx, 0, 0)
    st.reset()
    abi.moe_set_wait_limit(st.ctx, 60.0)
    _check_run(pb, pb.run(stack=st))
    st.close()


def test_layer_kernel_flag_wait_runs_out_then_reset_recovers():
    """A miss whose copy flags are never written: the layer kernel's bounded wait
    runs out (limit 0.3 s), the kernel records the failed check in the mapped
    page and returns; the next call reports it (MOE_ERR_CUDA, device check 40 or
    41), a reset brings the context back, and a full run matches the oracle."""
    import time
    pb = DecodeProblem(synth.TINY, T=8)
    st = pb.stack()
    abi.moe_debug_inject(st.ctx, 3, 1)  # the layer kernel
    abi.moe_set_wait_limit(st.ctx, 0.3)
    abi.moe_debug_inject(st.ctx, 4, 1)  # the next miss: copies issued, flags not written
    x = torch.from_numpy(pb.x[:, 0]).cuda()
    y = torch.zeros((pb.T, 1, pb.shape.d), device="cuda")
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    st.forward(0, x[0], y[0])  # cold cache: every selected expert misses
    st.synchronize()
    assert time.perf_counter() - t0 < 10.0
    with pytest.raises(abi.MoeError) as ei:
        st.forward(0, x[1], y[1])
    assert ei.value.status == abi.MOE_ERR_CUDA
    msg = abi.moe_last_error(st.ctx)
    assert "device check 40" in msg or "device check 41" in msg, msg
    st.reset()
    abi.moe_set_wait_limit(st.ctx, 60.0)
    _check_run(pb, pb.run(stack=st))
    st.close()
