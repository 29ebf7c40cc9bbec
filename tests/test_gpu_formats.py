"""Decode path with MXFP4 routed records and BF16 (or MXFP4) shared records,
on the GPU against the CPU oracle, through the C ABI.

Same bar as the NVFP4 decode tests: expert indices, cache events and the
table bit-exact; slot contents byte for byte; layer outputs within 1e-3
relative L2 (the kernels multiply exactly and accumulate in fp32, so the
error is at the 1e-6 level)."""
import numpy as np
import pytest

import synth
from synth import problem as sp
from tests.gpu_problem import DecodeProblem
from tests.test_gpu_decode import MID, _check_run

pytestmark = pytest.mark.gpu

MX, BF, NV = sp.FMT_MXFP4, sp.FMT_BF16, sp.FMT_NVFP4


@pytest.mark.parametrize("fmt,shared_fmt", [(MX, MX), (MX, BF), (NV, BF)],
                         ids=["mxfp4", "mxfp4+bf16-shared", "nvfp4+bf16-shared"])
def test_mid_shape_formats_full_parity(fmt, shared_fmt):
    # 3 layers, ragged K tails (d = 960, F = 320), E = 40 with 12 slots: hits,
    # misses and evictions; one row per call (the single-row mma columns)
    pb = DecodeProblem(MID, T=16, fmt=fmt, shared_fmt=shared_fmt)
    run = pb.run(routing=True)
    assert _check_run(pb, run) < 1e-5
    pb.check_slots(pb._last_stack, run.table[1])
    assert 0 < run.stats.misses < run.stats.lookups


@pytest.mark.parametrize("S", [5, 12])
def test_batched_rows_mxfp4_bf16_shared(S):
    # several rows per call: the two-group mma path of the routed GEMV, and
    # two passes (8 + 4 rows) of the BF16 shared expert at S = 12
    C = min(S * MID.k, MID.E) + 6
    pb = DecodeProblem(MID, T=4, streams=S, C=C, stream0=200, fmt=MX, shared_fmt=BF)
    run = pb.run(routing=True)
    assert _check_run(pb, run) < 1e-5


def test_host_io_path_with_formats():
    pb = DecodeProblem(MID, T=4, fmt=MX, shared_fmt=BF)
    a = pb.run()
    b = pb.run(host_io=True)
    assert a.events == b.events
    assert bool((a.y == b.y).all())


def test_gpt_oss_shaped_mxfp4_sampled():
    # the gpt-oss-shaped layer (d = F = 2880, E = 128, k = 4) with MXFP4
    # records, as its checkpoints ship them; 16 distinct records repeat over
    # the pool (same bytes, same transfers)
    sh = synth.SHAPES["gpt-oss-120b-shaped"]
    sh2 = synth.LayerShape("gpt-oss-mx", L=2, E=sh.E, k=sh.k, d=sh.d, F=sh.F, shared=False,
                           tokens=6, cache_slots=24)
    pb = DecodeProblem(sh2, T=6, distinct=16, fmt=MX)
    run = pb.run(routing=True)
    rng = np.random.default_rng(3)
    samples = [(int(t), int(l)) for t, l in zip(rng.integers(0, 6, 3), rng.integers(0, 2, 3))]
    assert _check_run(pb, run, samples=samples) < 1e-4
