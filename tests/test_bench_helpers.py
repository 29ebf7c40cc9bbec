"""bench.py's host-side arithmetic without a GPU: the roofline object of the
dominant kernel class, per-kernel tables, counter deltas and host times per
call, on hand-built moe_stats records whose answers are worked out here."""
import pytest

import bench
from expert_offload_caching_b200 import abi


def _stats(**kw):
    s = abi.moe_stats()
    for k, v in kw.items():
        if isinstance(v, (list, tuple)):
            arr = getattr(s, k)
            for i, x in enumerate(v):
                arr[i] = x
        else:
            setattr(s, k, v)
    return s


def _per_class(values):
    out = [0] * abi.MOE_K_COUNT
    for i, v in values.items():
        out[i] = v
    return out


def test_roofline_object_of_the_dominant_kernel_uses_device_spans():
    # gate/up: 10 launches, 2 ms of span time (5 ms of event time), 13 GB moved
    # down: 10 launches, 1 ms span; route: 10 launches, events only (0.5 ms)
    st = _stats(kernel_launches=_per_class({abi.MOE_K_ROUTE: 10, abi.MOE_K_GATEUP: 10, abi.MOE_K_DOWN: 10}),
                kernel_ms=_per_class({abi.MOE_K_ROUTE: 0.5, abi.MOE_K_GATEUP: 5.0, abi.MOE_K_DOWN: 4.0}),
                kernel_span_ms=_per_class({abi.MOE_K_GATEUP: 2.0, abi.MOE_K_DOWN: 1.0}),
                kernel_bytes=_per_class({abi.MOE_K_ROUTE: 1e6, abi.MOE_K_GATEUP: 13e9, abi.MOE_K_DOWN: 4e9}))
    r = bench.hbm_roofline(st, 6500.0, "measured")
    assert r["kernel"] == abi.KERNEL_NAMES[abi.MOE_K_GATEUP]
    assert r["achieved"] == pytest.approx(13e9 / 2e-3 / 1e9)  # 6500 GB/s
    assert r["frac"] == pytest.approx(1.0)
    assert r["timing"] == "device span" and r["launches"] == 10
    assert r["avg_launch_us"] == pytest.approx(200.0)
    assert r["bytes_per_launch"] == pytest.approx(1.3e9)
    tab = bench.kernel_table(st)
    assert set(tab) == {abi.KERNEL_NAMES[i] for i in (abi.MOE_K_ROUTE, abi.MOE_K_GATEUP, abi.MOE_K_DOWN)}
    route = tab[abi.KERNEL_NAMES[abi.MOE_K_ROUTE]]
    assert route["timing"] == "events" and route["ms"] == 0.5
    assert route["GBps"] == pytest.approx(1e6 / 0.5e-3 / 1e9)


def test_roofline_object_is_none_without_launches():
    assert bench.hbm_roofline(_stats(), 6500.0, "measured") is None


def test_stats_delta_and_host_times_per_call():
    before = _stats(lookups=10, hits=7, misses=3, forward_calls=2, host_us=[100.0, 80.0, 10.0],
                    kernel_ms=_per_class({abi.MOE_K_GATEUP: 1.5}))
    after = _stats(lookups=30, hits=20, misses=10, forward_calls=6, host_us=[500.0, 380.0, 50.0],
                   kernel_ms=_per_class({abi.MOE_K_GATEUP: 4.0}))
    d = bench.stats_delta(after, before)
    assert (d.lookups, d.hits, d.misses, d.forward_calls) == (20, 13, 7, 4)
    assert d.kernel_ms[abi.MOE_K_GATEUP] == pytest.approx(2.5)
    assert bench.host_us_per_call(d) == {"in_call": 100.0, "wait_miss_list": 75.0,
                                         "issue_after_list": 10.0}
    s = bench.stats_combine(before, before, 1)
    assert s.lookups == 20 and s.host_us[0] == 200.0


def test_replica_pool_records():
    L, E = 36, 128
    assert bench.replica_pool_records(L, E, 1) == L * E
    assert bench.replica_pool_records(L, E, 8) == L * E // 8
    assert bench.replica_pool_records(1, 16, 8) == bench.DISTINCT_RECORDS  # never below the distinct records


def test_gpu_launches_count_the_hit_launch_unless_the_layer_kernel_ran():
    """Default decode path: route + hit launch per call and one launch per miss
    are all launches of their own; with the layer kernel the hit-phase class is
    a part of its launches and is not counted again."""
    default = _stats(kernel_launches=_per_class({abi.MOE_K_ROUTE: 48, abi.MOE_K_LAYER_HITS: 48,
                                                 abi.MOE_K_MISS: 126}))
    assert bench.launch_count(default, None) == 48 + 48 + 126
    layer = _stats(kernel_launches=_per_class({abi.MOE_K_ROUTE: 48, abi.MOE_K_LAYER: 48,
                                               abi.MOE_K_LAYER_HITS: 48}))
    assert bench.launch_count(layer, None) == 96
    split = _stats(kernel_launches=_per_class({abi.MOE_K_ROUTE: 48, abi.MOE_K_LAYER_HITS: 48,
                                               abi.MOE_K_GATEUP: 126, abi.MOE_K_DOWN: 126}))
    assert bench.launch_count(split, None) == 48 + 48 + 252
    # without the timing pass: the default path's structure from the counters
    st = abi.moe_stats()
    st.forward_calls, st.misses = 48, 126
    assert bench.launch_count(None, st) == 2 * 48 + 126


def test_kernel_names_cover_every_class():
    assert len(abi.KERNEL_NAMES) == abi.MOE_K_COUNT
    assert abi.KERNEL_NAMES[abi.MOE_K_MISS] == "expert_miss"
    assert abi.KERNEL_NAMES[abi.MOE_K_LAYER_HITS] == "expert_hits"
