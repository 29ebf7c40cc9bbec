"""The C ABI without a GPU: the library loads, exports every declared symbol,
and its pure host functions (layout, sizes, planner, argument checks) agree
with the oracle and the golden cases."""
import math
import os
import re

import numpy as np
import pytest

import oracle
import synth
from expert_offload_caching_b200 import abi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
GOLDEN = os.path.join(ROOT, "tests", "golden")


def _declared():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            names += re.findall(r"^MOE_API\s+[\w\s\*]+?\b(\w+)\s*\(", text, flags=re.M)
    return names


def test_library_exports_every_declared_symbol():
    names = _declared()
    assert len(names) >= 18
    L = abi.lib()
    for n in names:
        assert hasattr(L, n), n
    assert set(abi.EXPORTS) <= set(names)


@pytest.mark.parametrize("shape", list(synth.SHAPES.values()), ids=lambda s: s.name)
def test_record_layout_matches_oracle(shape):
    d = abi.make_dims(shape.L, shape.E, shape.k, shape.d, shape.F, shape.shared)
    assert abi.moe_record_layout(d) == oracle.record_layout(shape.d, shape.F)
    assert abi.moe_record_bytes(d) == synth.record_bytes(shape.d, shape.F)
    assert abi.moe_workspace_bytes(d) > 0
    a1, a2 = abi.moe_arena_bytes(d, 10), abi.moe_arena_bytes(d, 20)
    assert a2 - a1 >= 10 * abi.moe_record_bytes(d)


def _golden_rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]


def test_plan_split_golden_and_oracle():
    for m, bp, bh, thr, mode, q in _golden_rows("planner_cases.txt"):
        r = abi.plan_split(int(m), float(bp), float(bh), float(thr))
        assert (r.mode, r.q, r.cpu) == (int(mode), int(q), int(m) - int(q))
    rng = np.random.default_rng(0)
    for _ in range(300):
        m = int(rng.integers(0, 300))
        bp = float(rng.uniform(1, 80))
        bh = float(rng.uniform(0, 300))
        eb = float(rng.uniform(1e5, 2e7))
        r = abi.plan_split(m, bp, bh, 2.0, eb)
        o = oracle.plan_split(m, bp, bh, 2.0, eb)
        assert (r.q, r.cpu, r.mode) == (o["q"], o["cpu"], o["mode"])
        assert r.q_real == pytest.approx(o["q_real"], rel=1e-15)
        assert r.t_finish == pytest.approx(o["t_finish"], rel=1e-12)
        if bh > bp:  # equal finish at the real-valued split
            assert r.q_real / bp == pytest.approx((m - r.q_real) / (bh - bp), rel=1e-12, abs=1e-12)


def test_plan_split_rejects_bad_arguments():
    for args in [(-1, 10.0, 20.0), (3, 0.0, 20.0), (3, 10.0, -1.0), (3, float("nan"), 1.0)]:
        with pytest.raises(abi.MoeError) as ei:
            abi.plan_split(*args)
        assert ei.value.status == abi.MOE_ERR_ARG
    with pytest.raises(abi.MoeError):
        abi.plan_split(3, 10.0, 20.0, 2.0, 0.0)


def test_init_argument_checks_without_device():
    good = abi.make_dims(2, 16, 2, 256, 512, max_rows=1)
    fake = 0x1000  # never dereferenced: argument checks come first
    with pytest.raises(abi.MoeError) as ei:
        abi.moe_layer_init(good, None, 1 << 30, fake, None, fake, 1 << 30, fake, fake)
    assert ei.value.status == abi.MOE_ERR_ARG
    bad_shape = abi.make_dims(2, 16, 2, 250, 512, max_rows=1)  # d not a multiple of 64
    with pytest.raises(abi.MoeError) as ei:
        abi.moe_layer_init(bad_shape, fake, 1 << 30, fake, None, fake, 1 << 30, fake, fake)
    assert ei.value.status == abi.MOE_ERR_UNSUPPORTED
    too_many_k = abi.make_dims(2, 64, 33, 256, 512, max_rows=1)
    with pytest.raises(abi.MoeError) as ei:
        abi.moe_layer_init(too_many_k, fake, 1 << 30, fake, None, fake, 1 << 30, fake, fake)
    assert ei.value.status == abi.MOE_ERR_UNSUPPORTED
    narrow_prefill = abi.make_dims(2, 16, 2, 192, 512, max_rows=64)  # prefill needs d, F >= 256
    with pytest.raises(abi.MoeError) as ei:
        abi.moe_layer_init(narrow_prefill, fake, 1 << 30, fake, None, fake, 1 << 30, fake, fake)
    assert ei.value.status == abi.MOE_ERR_UNSUPPORTED
    narrow_decode = abi.make_dims(2, 16, 2, 192, 512, max_rows=32)  # decode only: accepted shape
    with pytest.raises(abi.MoeError) as ei:  # ... and then the unpinned fake pool is refused
        abi.moe_layer_init(narrow_decode, fake, 1 << 30, fake, None, fake, 1 << 40, fake, fake)
    assert ei.value.status != abi.MOE_ERR_UNSUPPORTED
    shared_missing = abi.make_dims(2, 16, 2, 256, 512, has_shared=True, max_rows=1)
    with pytest.raises(abi.MoeError) as ei:
        abi.moe_layer_init(shared_missing, fake, 1 << 30, fake, None, fake, 1 << 30, fake, fake)
    assert ei.value.status == abi.MOE_ERR_ARG
    assert abi.moe_record_bytes(abi.make_dims(0, 16, 2, 256, 512)) == 0
    assert abi.moe_status_str(abi.MOE_ERR_TIMEOUT) == "timed out waiting for the device"


@pytest.mark.parametrize("shape", list(synth.SHAPES.values()), ids=lambda s: s.name)
def test_mxfp4_and_bf16_record_layouts(shape):
    """MXFP4 routed records and BF16 shared records: the ABI's offsets and sizes
    agree with the oracle's and the generator's layouts."""
    d = abi.make_dims(shape.L, shape.E, shape.k, shape.d, shape.F, True,
                      weight_format=abi.MOE_FMT_MXFP4)
    off = oracle.mx_record_layout(shape.d, shape.F)
    assert synth.mx_record_layout(shape.d, shape.F) == off
    assert abi.moe_record_layout(d) == (off[0], off[1], off[2], off[3], -1, off[4])
    assert abi.moe_record_bytes(d) == off[4]
    assert abi.moe_shared_record_bytes(d) == off[4]  # shared format = routed format
    for wf in (abi.MOE_FMT_NVFP4, abi.MOE_FMT_MXFP4):
        db = abi.make_dims(shape.L, shape.E, shape.k, shape.d, shape.F, True,
                           weight_format=wf, shared_format=abi.MOE_FMT_BF16)
        assert abi.moe_shared_record_bytes(db) == 2 * 3 * shape.d * shape.F
        assert synth.expert_record_bf16(0, 0, shape.d, shape.F).nbytes == 6 * shape.d * shape.F
    nv = abi.make_dims(shape.L, shape.E, shape.k, shape.d, shape.F, True)
    assert abi.moe_shared_record_bytes(nv) == abi.moe_record_bytes(nv)


def test_format_argument_checks_without_device():
    fake = 0x1000
    bad = [abi.make_dims(2, 16, 2, 256, 512, weight_format=abi.MOE_FMT_BF16),  # BF16 routed
           abi.make_dims(2, 16, 2, 256, 512, weight_format=7),
           abi.make_dims(2, 16, 2, 256, 512, True, weight_format=abi.MOE_FMT_MXFP4,
                         shared_format=abi.MOE_FMT_NVFP4)]  # shared neither routed nor BF16
    for d in bad:
        assert abi.moe_record_bytes(d) == 0 and abi.moe_shared_record_bytes(d) == 0
        with pytest.raises(abi.MoeError) as ei:
            abi.moe_layer_init(d, fake, 1 << 30, fake, fake, fake, 1 << 30, fake, fake)
        assert ei.value.status == abi.MOE_ERR_ARG
    # no shared expert: the shared format is not looked at
    ok = abi.make_dims(2, 16, 2, 256, 512, False, weight_format=abi.MOE_FMT_MXFP4,
                       shared_format=abi.MOE_FMT_NVFP4)
    assert abi.moe_record_bytes(ok) == oracle.mx_record_layout(256, 512)[4]
    # MXFP4 and BF16 records run on the decode and the prefill paths
    for wf, sf in ((abi.MOE_FMT_MXFP4, None), (abi.MOE_FMT_NVFP4, abi.MOE_FMT_BF16),
                   (abi.MOE_FMT_MXFP4, abi.MOE_FMT_BF16)):
        for rows in (32, 64):
            dims = abi.make_dims(2, 16, 2, 256, 512, True, max_rows=rows, weight_format=wf,
                                 shared_format=sf)
            with pytest.raises(abi.MoeError) as ei:  # accepted shape; then the fake pool is refused
                abi.moe_layer_init(dims, fake, 1 << 30, fake, fake, fake, 1 << 40, fake, fake)
            assert ei.value.status == abi.MOE_ERR_NOT_PINNED


def test_size_queries_and_init_checks_over_random_dims():
    """Random dims, valid and not: the size queries return 0 exactly for
    invalid dims, grow with the slot count, and cover the layout; init with
    fake pointers answers ARG, UNSUPPORTED or NOT_PINNED (never touching them)."""
    rng = np.random.default_rng(51)
    fake = 0x1000
    seen = set()
    for _ in range(400):
        L = int(rng.choice([0, 1, 2, 48, 64]))
        E = int(rng.choice([0, 1, 16, 256, 512, 1024, 2048]))
        k = int(rng.choice([0, 1, 4, 10, 32, 33]))
        d = int(rng.choice([0, 64, 192, 250, 2048, 2880, 4096, 8192]))
        F = int(rng.choice([0, 64, 768, 2880, 4096, 5000]))
        rows = int(rng.choice([0, 1, 32, 33, 4096, 5000]))
        wf = int(rng.choice([0, 1, 2, 3]))
        sf = int(rng.choice([0, 1, 2]))
        sh = bool(rng.integers(2))
        dims = abi.make_dims(L, E, k, d, F, sh, True, rows, 0, weight_format=wf, shared_format=sf)
        valid = (L > 0 and E > 0 and 0 < k <= E and d > 0 and F > 0 and rows > 0 and wf in (0, 1)
                 and (not sh or sf in (wf, 2)))
        rb = abi.moe_record_bytes(dims)
        assert (rb > 0) == valid
        if not valid:
            assert abi.moe_workspace_bytes(dims) == 0 and abi.moe_arena_bytes(dims, 8) == 0
            with pytest.raises(abi.MoeError) as ei:
                abi.moe_layer_init(dims, fake, 1 << 40, fake, fake, fake, 1 << 40, fake, fake)
            assert ei.value.status == abi.MOE_ERR_ARG
            seen.add("arg")
            continue
        off = abi.moe_record_layout(dims)
        assert off[5] == rb and max(off[:5]) < rb
        assert abi.moe_workspace_bytes(dims) > 0
        a8, a16 = abi.moe_arena_bytes(dims, 8), abi.moe_arena_bytes(dims, 16)
        assert a16 - a8 >= 8 * rb
        with pytest.raises(abi.MoeError) as ei:
            abi.moe_layer_init(dims, fake, 1 << 50, fake, fake, fake, 1 << 50, fake, fake)
        assert ei.value.status in (abi.MOE_ERR_UNSUPPORTED, abi.MOE_ERR_NOT_PINNED)
        seen.add(ei.value.status)
    assert seen >= {"arg", abi.MOE_ERR_UNSUPPORTED, abi.MOE_ERR_NOT_PINNED}
