"""The decode path at its largest row count (T = 32 rows per call: the union
lookup of 32 x k selections, four 8-row passes of the GEMV's mma columns,
four 8-row passes of the BF16 shared expert) against the oracle."""
import pytest

from synth import problem as sp
from tests.gpu_problem import DecodeProblem
from tests.test_gpu_decode import MID, _check_run

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("fmt,shared_fmt", [(sp.FMT_NVFP4, None), (sp.FMT_MXFP4, sp.FMT_BF16)],
                         ids=["nvfp4", "mxfp4+bf16-shared"])
def test_decode_at_32_rows(fmt, shared_fmt):
    S = 32
    C = MID.L * MID.E  # every expert stays once loaded: misses on the first call, hits after
    pb = DecodeProblem(MID, T=3, streams=S, C=C, stream0=300, fmt=fmt, shared_fmt=shared_fmt)
    run = pb.run(routing=True)
    assert _check_run(pb, run) < 1e-5
    assert 0 < run.stats.hits < run.stats.lookups
    pb.check_slots(pb._last_stack, run.table[1])
