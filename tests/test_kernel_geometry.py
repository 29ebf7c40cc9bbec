"""CPU mirror of the GEMV kernel's staging arithmetic: for every workload shape,
each CTA's two copies (tile codes, tile scales) and its down-projection L2
prefetch range lie inside the expert record, start on 16-byte boundaries and
have sizes that are multiples of 16; shared-memory use fits the launch."""
import pytest

import synth
from expert_offload_caching_b200 import abi

SHAPES = list(synth.SHAPES.values()) + [
    synth.LayerShape("mid", L=3, E=40, k=5, d=960, F=320, shared=True, tokens=24, cache_slots=12)]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: s.name)
def test_tile_copies_inside_record_and_aligned(shape):
    dims = abi.make_dims(shape.L, shape.E, shape.k, shape.d, shape.F, shape.shared)
    off = abi.moe_record_layout(dims)
    rb = off[5]
    assert rb % 256 == 0 and all(o % 256 == 0 for o in off)
    for mode, K, tiles, codes0, scales0, end in (
            ("gate_up", shape.d, shape.F // 8, off[0], off[1], off[2]),
            ("down", shape.F, shape.d // 16, off[2], off[3], off[5])):
        code_bytes, scale_bytes = 16 * (K // 2), K
        assert code_bytes % 16 == 0 and scale_bytes % 16 == 0
        assert code_bytes + scale_bytes <= 96 * 1024  # dynamic shared memory limit set at launch
        for t in range(tiles):
            c0, s0 = codes0 + t * code_bytes, scales0 + t * scale_bytes
            assert c0 % 16 == 0 and s0 % 16 == 0
            assert c0 + code_bytes <= scales0, (mode, t)
            assert s0 + scale_bytes <= end, (mode, t)
        # shared-memory destinations: codes at 0, scales right after (16-byte multiple)
        assert code_bytes % 16 == 0
    assert off[4] == 0 and off[0] >= 12  # tensor scales at the head: W13 + scales form a prefix
    # down-projection prefetch ranges issued by the gate/up CTAs
    total = off[5] - off[2]
    grid = shape.F // 8
    per = ((total // grid) + 127) & ~127
    covered = 0
    for b in range(grid):
        o = per * b
        if o < total:
            n = min(per, total - o)
            assert off[2] + o + n <= off[5]
            covered += n
    assert covered == total


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: s.name)
def test_router_rows_fit_the_register_tile(shape):
    nvec = shape.d // 8
    nv = (nvec + 31) // 32
    assert nv <= 16  # route kernel templates: 1, 2, 4, 8, 12, 16 vectors per lane
    total = shape.E * shape.d * 2
    grid = (shape.E + 7) // 8
    per = ((total // grid) + 127) & ~127
    assert per * (grid - 1) < total
