"""MXFP4 scale edge cases on the GPU against the oracle: E8M0 codes spread
far apart inside one K-step (the GEMV factors out each step's largest code),
blocks far below their step's largest (their contribution falls under fp16),
and a NaN scale (code 255), which the OCP definition propagates to every
output of the expert."""
import numpy as np
import pytest

import synth
from synth import problem as sp
from tests.gpu_problem import REL_L2_MAX, DecodeProblem, rel_l2
from tests.test_gpu_decode import _check_run

pytestmark = pytest.mark.gpu

# ragged K tails on both projections (d = 320: 5 chunks of 64; F = 192: 3),
# 2 layers, a shared expert, fewer slots than experts
SHAPE = synth.LayerShape("mx-range", L=2, E=12, k=3, d=320, F=192, shared=True, tokens=8,
                         cache_slots=8)


def _scale_sections(d, F):
    off = synth.mx_record_layout(d, F)
    return [(off[1], 2 * F * d // 32), (off[3], d * F // 32)]


def _respread(buf: np.ndarray, nrec: int, rb: int, d: int, F: int, rng) -> None:
    """Overwrite every scale byte of nrec records in buf: codes drawn from
    [99, 124] (2^-28 .. 2^-3: a spread of 25 inside one K-step, with the
    largest blocks keeping the outputs at the generator's magnitudes), one block
    in 50 at codes 20..40 (more than 35 below its step's largest)."""
    for r in range(nrec):
        for start, n in _scale_sections(d, F):
            codes = rng.integers(99, 125, n)
            tiny = rng.random(n) < 0.02
            codes[tiny] = rng.integers(20, 41, int(tiny.sum()))
            buf[r * rb + start:r * rb + start + n] = codes.astype(np.uint8)


def _problem(rng):
    pb = DecodeProblem(SHAPE, T=8, fmt=sp.FMT_MXFP4, shared_fmt=sp.FMT_MXFP4)
    _respread(pb.pool_np, pb.P, pb.rb, SHAPE.d, SHAPE.F, rng)
    _respread(pb.shared, SHAPE.L, pb.srb, SHAPE.d, SHAPE.F, rng)
    return pb


def test_wide_scale_spread_within_a_step():
    pb = _problem(np.random.default_rng(21))
    run = pb.run(routing=True)
    assert _check_run(pb, run) < 1e-4


def test_nan_scale_propagates_to_the_rows_that_use_the_expert():
    pb = _problem(np.random.default_rng(22))
    idx, _ = pb.oracle_routing()
    e_nan = int(idx[0, 0, 0, 0])  # an expert token 0 uses at layer 0
    w13_scales = synth.mx_record_layout(SHAPE.d, SHAPE.F)[1]
    pb.pool_np[e_nan * pb.rb + w13_scales + 3] = 255  # record (0, e_nan): one W13 block
    run = pb.run(routing=True)
    _check_run(pb, run, samples=[])  # indices, events, table: unchanged by the weights
    y = run.y.cpu().numpy()
    n_nan = 0
    for t in range(pb.T):
        for l in range(SHAPE.L):
            want, got = pb.oracle_y(t, l), y[t, l].astype(np.float64)
            uses = l == 0 and e_nan in idx[t, l, 0]
            assert np.isnan(want).all() == uses
            if uses:
                assert np.isnan(got).all(), (t, l)
                n_nan += 1
            else:
                assert np.isfinite(got).all() and rel_l2(got, want) <= REL_L2_MAX, (t, l)
    assert n_nan >= 1
