"""Pins of the CPU oracle against things other than itself: hand-worked values
(tests/golden, each cited), library routines (torch float8, scipy), closed
forms, invariants and brute force.  No GPU needed."""
import itertools
import math
import os
from collections import OrderedDict
from fractions import Fraction

import numpy as np
import pytest
import torch
from scipy.special import expit

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]


def _bf16_bits(a):
    return synth.to_bf16(np.asarray(a, dtype=np.float32))


def _bf16_val(b):
    return synth.bf16_to_f32(np.asarray(b, dtype=np.uint16)).astype(np.float64)


# Independent decode used by the tests: E2M1 from the golden table, E4M3 from torch.
E2M1_GOLDEN = {int(c, 16): float(v) for c, v in _rows("e2m1_table.txt")}


def _e4m3_torch(b):
    return torch.tensor(np.asarray(b, dtype=np.uint8)).view(torch.float8_e4m3fn).double().numpy()


def _dequant_independent(codes, scales, rows, K, ts):
    codes = np.asarray(codes, dtype=np.uint8).reshape(rows, K // 2)
    lo, hi = codes & 0xF, codes >> 4
    nib = np.empty((rows, K), dtype=np.uint8)
    nib[:, 0::2], nib[:, 1::2] = lo, hi
    vals = np.vectorize(E2M1_GOLDEN.get)(nib).astype(np.float64)
    sc = _e4m3_torch(np.asarray(scales).reshape(rows, K // 16))
    return vals * np.repeat(sc, 16, axis=1) * ts


def _matrices_independent(rec, d, F):
    off = synth.record_layout(d, F)  # the generator's layout: written separately from the oracle's
    ts = np.frombuffer(rec[off[4]:off[4] + 12].tobytes(), dtype=np.float32).astype(np.float64)
    w13c, w13s = rec[off[0]:off[0] + F * d], rec[off[1]:off[1] + F * d // 8]
    W13 = _dequant_independent(w13c, w13s, 2 * F, d, 1.0)
    W1, W3 = W13[0::2] * ts[0], W13[1::2] * ts[1]
    W2 = _dequant_independent(rec[off[2]:off[2] + d * F // 2], rec[off[3]:off[3] + d * F // 16],
                              d, F, ts[2])
    return W1, W3, W2


# ------------------------------------------------------------ formats --
def test_e2m1_matches_hand_table():
    for code, val in E2M1_GOLDEN.items():
        got = oracle.e2m1(code)
        assert got == val and math.copysign(1, got) == math.copysign(1, val), code


def test_e4m3_hand_points():
    for b, v in _rows("e4m3_points.txt"):
        assert oracle.e4m3(int(b, 16)) == float(v), b


def test_e4m3_exhaustive_vs_torch():
    ref = _e4m3_torch(np.arange(256))
    for b in range(256):
        got = oracle.e4m3(b)
        if math.isnan(ref[b]):
            assert math.isnan(got), b
        else:
            assert got == ref[b], (b, got, ref[b])


def test_nvfp4_worked_example():
    (cb, sb, ts, ev, od), = _rows("nvfp4_worked_example.txt")
    d, F = 64, 64
    off = oracle.record_layout(d, F)
    rec = np.zeros(off[5], dtype=np.uint8)
    # element (row 2j=gate_j, K) with j = 3, K = 2i = 20 -> byte 10 of W13 row 6
    j, i = 3, 10
    rec[off[0] + (2 * j) * (d // 2) + i] = int(cb, 16)
    rec[off[1] + (2 * j) * (d // 16) + (2 * i) // 16] = int(sb, 16)
    rec[off[4]:off[4] + 12] = np.frombuffer(np.array([float(ts)] * 3, np.float32).tobytes(),
                                            np.uint8)
    W1 = oracle.dequant_matrix(rec, d, F, 0)
    assert W1[j, 2 * i] == float(ev) and W1[j, 2 * i + 1] == float(od)
    assert np.count_nonzero(W1) == 2 and np.count_nonzero(oracle.dequant_matrix(rec, d, F, 1)) == 0


def test_record_bytes_golden():
    for d, F, nb in _rows("record_bytes.txt"):
        assert oracle.record_layout(int(d), int(F))[5] == int(nb)
        assert synth.record_bytes(int(d), int(F)) == int(nb)


def test_dequant_layout_random_record():
    rng = np.random.default_rng(1)
    d, F = 128, 192
    off = oracle.record_layout(d, F)
    rec = rng.integers(0, 256, off[5], dtype=np.uint8)
    for o, n in ((off[1], 2 * F * d // 16), (off[3], d * F // 16)):  # finite scales only
        s = rec[o:o + n]
        s[(s & 0x7F) == 0x7F] = 0x38
    rec[off[4]:off[4] + 12] = np.frombuffer(np.array([0.5, 0.25, 2.0], np.float32).tobytes(),
                                            np.uint8)
    W1, W3, W2 = _matrices_independent(rec, d, F)
    np.testing.assert_array_equal(oracle.dequant_matrix(rec, d, F, 0), W1)
    np.testing.assert_array_equal(oracle.dequant_matrix(rec, d, F, 1), W3)
    np.testing.assert_array_equal(oracle.dequant_matrix(rec, d, F, 2), W2)


# ------------------------------------------------------------ routing --
def test_logits_exact_rational():
    rng = np.random.default_rng(2)
    E, d = 5, 32
    Wr = _bf16_bits(rng.normal(0, 0.5, (E, d)))
    x = _bf16_bits(rng.normal(0, 1, (1, d)))
    _, _, z, _ = oracle.route(Wr, x, 2)
    for e in range(E):
        exact = sum(Fraction(float(a)) * Fraction(float(b))
                    for a, b in zip(_bf16_val(Wr[e]), _bf16_val(x[0])))
        assert abs(z[0, e] - float(exact)) <= 1e-15 * max(1.0, abs(float(exact)))


@pytest.mark.parametrize("k", [1, 2, 3, 4])
def test_topk_bruteforce_subsets(k):
    rng = np.random.default_rng(10 + k)
    E, d, T = 16, 64, 24
    Wr = _bf16_bits(rng.normal(0, 0.1, (E, d)))
    x = _bf16_bits(rng.normal(0, 1, (T, d)))
    idx, gates, z, gap = oracle.route(Wr, x, k)
    for t in range(T):
        best = max(itertools.combinations(range(E), k), key=lambda s: sum(z[t, list(s)]))
        assert tuple(idx[t]) == tuple(sorted(best))
        assert abs(gates[t].sum() - 1.0) < 1e-12
        # closed form of the renormalised gates: ratios are exp of logit differences
        for a, b in itertools.combinations(range(k), 2):
            assert gates[t, a] / gates[t, b] == pytest.approx(
                math.exp(z[t, idx[t, a]] - z[t, idx[t, b]]), rel=1e-12)
        zs = np.sort(z[t])[::-1]
        if k < E:
            assert gap[t] == zs[k - 1] - zs[k]


def test_gates_without_renorm_are_softmax_probabilities():
    rng = np.random.default_rng(3)
    E, d = 16, 64
    Wr = _bf16_bits(rng.normal(0, 0.1, (E, d)))
    x = _bf16_bits(rng.normal(0, 1, (3, d)))
    idx, p, z, _ = oracle.route(Wr, x, E, renorm=False)  # k = E: every probability
    np.testing.assert_array_equal(idx, np.tile(np.arange(E), (3, 1)))
    np.testing.assert_allclose(p.sum(1), 1.0, rtol=1e-13)
    np.testing.assert_allclose(p, torch.softmax(torch.tensor(z), dim=1).numpy(), rtol=1e-12)


def test_topk_ties_go_to_lower_id():
    d = 32
    row = _bf16_bits(np.linspace(-1, 1, d))
    Wr = np.stack([row * 0, row, row, row, row * 0])  # experts 1,2,3 tie
    x = _bf16_bits(np.linspace(-1, 1, d)[None])
    idx, _, _, gap = oracle.route(Wr, x, 2)
    assert tuple(idx[0]) == (1, 2) and gap[0] == 0.0


def test_non_finite_logits_rank_as_minus_infinity():
    """Hand-worked selections with non-finite inputs: NaN logits rank as -inf,
    equal values go to the lower id, and k distinct ids in [0, E) come out."""
    E, d = 8, 16
    Wr = np.zeros((E, d), dtype=np.float32)
    Wr[:, 1:] = 0.25
    Wr[:, 0] = [1, 1, -1, 1, 0, -1, 1, 1]  # x_0 = -inf: experts 2 and 5 go to +inf, 4 to NaN
    x = np.ones((3, d), dtype=np.float32)
    x[0, 0] = -np.inf
    x[1, 0] = np.nan                       # every logit NaN
    x[2, 0] = np.inf                       # +inf except 2, 5 (-inf) and 4 (NaN)
    idx, gates, z, _ = oracle.route(_bf16_bits(Wr), _bf16_bits(x), 3)
    assert tuple(idx[0]) == (0, 2, 5)      # the two +inf, then the lowest -inf
    assert tuple(idx[1]) == (0, 1, 2)      # all -inf: the lowest ids
    assert tuple(idx[2]) == (0, 1, 3)      # five +inf: the lowest three
    assert z[0, 4] == -np.inf and np.all(z[1] == -np.inf)
    assert np.all(np.isnan(gates))         # inf - inf in every softmax
    # a finite row beside them is untouched
    x2 = np.ones((1, d), dtype=np.float32)
    i2, g2, z2, _ = oracle.route(_bf16_bits(Wr), _bf16_bits(x2), 3)
    assert np.all(np.isfinite(g2)) and abs(g2.sum() - 1.0) < 1e-12


# --------------------------------------------------------- expert FFN --
def test_expert_one_hot_input_closed_form():
    d, F = 128, 256
    rec = synth.expert_record(0, 5, d, F)
    W1, W3, W2 = _matrices_independent(rec, d, F)
    K = 37
    x = np.zeros(d, dtype=np.uint16)
    x[K] = _bf16_bits([1.0])[0]
    y, h = oracle.expert_w4a16(rec, d, F, x)
    g, u = W1[:, K], W3[:, K]
    h_ref = g * expit(g) * u
    np.testing.assert_allclose(h, h_ref, rtol=1e-13, atol=1e-300)
    np.testing.assert_allclose(y, W2 @ h_ref, rtol=1e-10, atol=1e-14)


def test_expert_dense_reference():
    d, F = 256, 512
    rec = synth.expert_record(0, 1, d, F)
    W1, W3, W2 = _matrices_independent(rec, d, F)
    x = _bf16_bits(np.random.default_rng(4).normal(0, 1, d))
    xv = _bf16_val(x)
    y, h = oracle.expert_w4a16(rec, d, F, x)
    g, u = W1 @ xv, W3 @ xv
    np.testing.assert_allclose(h, g * expit(g) * u, rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(y, W2 @ (g * expit(g) * u), rtol=1e-9, atol=1e-12)


def test_silu_special_values():
    d, F = 64, 64
    off = oracle.record_layout(d, F)
    rec = np.zeros(off[5], dtype=np.uint8)
    rec[off[4]:off[4] + 12] = np.frombuffer(np.array([1, 1, 1], np.float32).tobytes(), np.uint8)
    x = _bf16_bits(np.ones(d))
    y, h = oracle.expert_w4a16(rec, d, F, x)  # all-zero codes: silu(0) * 0 = 0
    assert not h.any() and not y.any()


def test_layer_combine_special_cases():
    s = synth.TINY
    P = s.L * s.E
    rb = synth.record_bytes(s.d, s.F)
    pool = np.concatenate([synth.expert_record(0, e, s.d, s.F) for e in range(s.E)])
    Wr = synth.router_bf16(0, s.E, s.d)
    shared = synth.expert_record(0, 0, s.d, s.F, shared=True)
    x = _bf16_bits(np.random.default_rng(5).normal(0, 1, (3, s.d)))
    # top-1 with renormalisation: gate 1, y = E_e(x)
    idx, g, y = oracle.moe_layer(pool, P, 0, s.E, s.d, s.F, 1, Wr, None, x)
    np.testing.assert_array_equal(g, 1.0)
    for t in range(3):
        e = idx[t, 0]
        np.testing.assert_array_equal(y[t], oracle.expert_w4a16(pool[e * rb:(e + 1) * rb],
                                                                s.d, s.F, x[t])[0])
    # the shared expert adds with unit weight
    _, _, y0 = oracle.moe_layer(pool, P, 0, s.E, s.d, s.F, 2, Wr, None, x)
    _, _, y1 = oracle.moe_layer(pool, P, 0, s.E, s.d, s.F, 2, Wr, shared, x)
    for t in range(3):
        np.testing.assert_allclose(y1[t] - y0[t], oracle.expert_w4a16(shared, s.d, s.F, x[t])[0],
                                   rtol=1e-9, atol=1e-12)
    # pool aliasing: record of (layer, e) is (layer*E + e) mod P
    _, _, ya = oracle.moe_layer(pool[:5 * rb], 5, 0, s.E, s.d, s.F, 1, Wr, None, x)
    for t in range(3):
        e = idx[t, 0] % 5
        np.testing.assert_array_equal(ya[t], oracle.expert_w4a16(pool[e * rb:(e + 1) * rb],
                                                                 s.d, s.F, x[t])[0])


# ------------------------------------------------------------ LRU ------
def test_lru_hand_trace():
    rows = _rows("lru_hand_trace.txt")
    lru = oracle.LRU(1, 16, 4)
    hits = misses = 0
    for r in rows:
        if r[0] == "final":
            assert list(lru.state()[1]) == [int(v) for v in r[1].split(",")]
            continue
        req = [int(v) for v in r[1].split(",")]
        want = [tuple(int(v) for v in ev.split(":")) for ev in r[2:]]
        got = lru.batch(0, req)
        assert got == want, (r, got)
        hits += sum(g[2] for g in got)
        misses += sum(1 - g[2] for g in got)
    assert (misses, hits) == (7, 5)


def test_static_split_hand_trace():
    """The static per-layer split against the hand-worked trace (golden)."""
    from oracle.workloads import static_split_trace
    rows = _rows("static_split_hand_trace.txt")
    idx = np.zeros((2, 2, 2, 2), dtype=np.int32)
    want = []
    for r in rows:
        t, l = int(r[0]), int(r[1])
        idx[t, l] = [[int(v) for v in row.split(",")] for row in r[2].split("|")]
        want += [(t, l) + tuple(int(v) for v in ev.split(":")) + (-1,) for ev in r[4:]]
    assert static_split_trace(idx, 2, 8, 8, 4) == want


def test_static_split_miss_rate_closed_form():
    """Every expert of every layer used once per step: the hits are exactly the s
    resident experts per layer, so the miss rate is 1 - s/E; no slot outside
    [0, C) and no resident slot is ever given to a miss."""
    from oracle.workloads import static_split_trace
    L, E, C, R = 3, 40, 50, 10
    s = (C - R) // L  # 13
    idx = np.tile(np.arange(E, dtype=np.int32), (2, L, 1, 1))  # [T=2, L, rows=1, k=E]
    ev = static_split_trace(idx, L, E, C, R + E)  # scratch for a whole-E batch
    s2 = min((C - (R + E)) // L, E)
    assert s2 == 0 and all(h == 0 for *_, h, _v in ev)
    ev = static_split_trace(idx, L, E, C + E, R + E)
    s3 = (C + E - R - E) // L
    assert s3 == s
    hits = sum(e[4] for e in ev)
    assert hits == 2 * L * s and len(ev) == 2 * L * E
    assert all(0 <= e[3] < C + E for e in ev)
    assert all(e[3] >= L * s for e in ev if not e[4])
    assert abs((1 - hits / len(ev)) - (1 - s / E)) < 1e-12


class _DictLRU:
    """Brute-force LRU for the cross-check: an ordered dict of resident keys."""

    def __init__(self, C):
        self.C, self.od, self.free = C, OrderedDict(), list(range(C))

    def batch(self, layer, E, experts):
        out, keys = [], [layer * E + e for e in experts]
        for key in keys:
            if key in self.od:
                self.od.move_to_end(key)
        for e, key in zip(experts, keys):
            if key in self.od:
                out.append((e, self.od[key], 1, -1))
                continue
            if self.free:
                slot, ev = self.free.pop(0), -1
            else:
                ev, slot = self.od.popitem(last=False)
            self.od[key] = slot
            out.append((e, slot, 0, ev))
        return out


@pytest.mark.parametrize("L,E,C,k", [(1, 16, 4, 2), (3, 8, 5, 3), (4, 32, 40, 4), (2, 64, 64, 10)])
def test_lru_matches_bruteforce_and_invariants(L, E, C, k):
    rng = np.random.default_rng(L * 100 + C)
    lru, ref = oracle.LRU(L, E, C), _DictLRU(C)
    n_lookups = n_hits = 0
    for step in range(300):
        layer = int(rng.integers(L))
        req = np.sort(rng.choice(E, size=min(k, C, E), replace=False)).astype(np.int32)
        got = lru.batch(layer, req)
        assert got == ref.batch(layer, E, [int(v) for v in req])
        n_lookups += len(got)
        n_hits += sum(g[2] for g in got)
        m, owner, stamp, clock = lru.state()
        res = np.nonzero(owner >= 0)[0]
        assert len(res) <= C
        for s in res:
            assert m[owner[s]] == s  # map/owner bijection
        assert np.count_nonzero(m >= 0) == len(res)
        assert clock == n_lookups  # one stamp per lookup
    assert 0 < n_hits < n_lookups


def test_lru_rejects_bad_batches():
    lru = oracle.LRU(2, 8, 3)
    for bad in ([3, 1], [1, 1], [9], [0, 1, 2, 3]):
        with pytest.raises(ValueError):
            lru.batch(0, bad)
    with pytest.raises(ValueError):
        lru.batch(2, [0])


# ----------------------------------------------------------- planner --
def test_planner_golden_cases():
    for m, bp, bh, thr, mode, q in _rows("planner_cases.txt"):
        r = oracle.plan_split(int(m), float(bp), float(bh), float(thr))
        assert (r["mode"], r["q"], r["cpu"]) == (int(mode), int(q), int(m) - int(q))


def test_planner_equal_finish_invariant():
    rng = np.random.default_rng(6)
    for _ in range(200):
        m = int(rng.integers(1, 200))
        bp = float(rng.uniform(5, 60))
        bh = bp * float(rng.uniform(1.01, 8))
        r = oracle.plan_split(m, bp, bh, 2.0)
        qr = r["q_real"]
        assert qr / bp == pytest.approx((m - qr) / (bh - bp), rel=1e-12)
        assert qr / bp == pytest.approx(m / bh, rel=1e-12)
        if bh / bp > 2.0:
            assert r["q"] == math.floor(qr + 0.5) and r["mode"] == 1
        else:
            assert r["q"] == m and r["mode"] == 0


# --------------------------------------------------------- quantizer --
def test_e4m3_rne_vs_torch_including_ties():
    pos = np.array([oracle.e4m3(b) for b in range(0x7F)])
    mids = (pos[:-1] + pos[1:]) / 2
    rng = np.random.default_rng(7)
    samples = np.concatenate([pos, mids, rng.uniform(0, 448, 4000), rng.uniform(0, 0.02, 2000),
                              [447.9, 448.0]]).astype(np.float32)
    ref = torch.tensor(samples).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_rne(float(v)) for v in samples])
    np.testing.assert_array_equal(got, ref)
    assert oracle.e4m3_rne(1e6) == 0x7E and oracle.e4m3_rne(449.0) == 0x7E


def test_e2m1_rne_midpoints_and_saturation():
    # midpoint -> value: ties go to the even mantissa
    for v, want in [(0.25, 0.0), (0.75, 1.0), (1.25, 1.0), (1.75, 2.0), (2.5, 2.0), (3.5, 4.0),
                    (5.0, 4.0), (7.0, 6.0), (1e9, 6.0), (0.2, 0.0), (0.26, 0.5), (5.01, 6.0)]:
        assert E2M1_GOLDEN[oracle.e2m1_rne(v)] == want, v
        assert E2M1_GOLDEN[oracle.e2m1_rne(-v)] == -want, v
    for c, val in E2M1_GOLDEN.items():  # every representable value maps back to itself
        assert E2M1_GOLDEN[oracle.e2m1_rne(val)] == val


def test_quantizer_round_trip_of_representable_blocks():
    rng = np.random.default_rng(8)
    nblk = 64
    s_t = np.float32(2.0 ** -10)
    codes = rng.integers(0, 16, (nblk, 16))
    scales = rng.integers(1, 0x7F, nblk)
    scales[0] = 0x7E
    for b in range(nblk):  # every block holds a +-6 so its amax is 6 * scale * s_t
        codes[b, rng.integers(16)] = 7 if rng.random() < 0.5 else 15
    x = np.array([[E2M1_GOLDEN[c] * oracle.e4m3(s) * s_t for c in row]
                  for row, s in zip(codes, scales)], dtype=np.float32).ravel()
    assert oracle.tensor_scale(x) == s_t
    qc, qs = oracle.nvfp4_quantize(x, s_t)
    np.testing.assert_array_equal(qs, scales)
    lo, hi = qc & 0xF, qc >> 4
    got = np.empty(x.size, dtype=np.int64)
    got[0::2], got[1::2] = lo, hi
    want = codes.ravel().copy()
    want[np.array([E2M1_GOLDEN[c] for c in want]) == 0.0] = got[
        np.array([E2M1_GOLDEN[c] for c in want]) == 0.0]  # +-0 may carry either sign
    np.testing.assert_array_equal(got, want)


def test_w4a4_one_hot_row():
    d, F = 128, 256
    rec = synth.expert_record(0, 9, d, F)
    W1, W3, W2 = _matrices_independent(rec, d, F)
    K = 5
    x = np.zeros(d, dtype=np.uint16)
    x[K] = _bf16_bits([1.0])[0]
    y = oracle.expert_w4a4(rec, d, F, x)
    s = np.float32(1.0) / np.float32(2688.0)  # one-hot row: quantized x_K = 6 * 448 * s
    xk = 6.0 * 448.0 * float(s)
    g, u = W1[:, K] * xk, W3[:, K] * xk
    h = (g * expit(g) * u).astype(np.float32)
    sh = oracle.tensor_scale(h)
    hc, hs = oracle.nvfp4_quantize(h, sh)
    nib = np.empty(F, dtype=np.int64)
    nib[0::2], nib[1::2] = hc & 0xF, hc >> 4
    hq = np.array([E2M1_GOLDEN[c] for c in nib]) * np.repeat(_e4m3_torch(hs), 16) * float(sh)
    np.testing.assert_allclose(y, W2 @ hq, rtol=1e-9, atol=1e-12)
    # and the quantized h is within NVFP4's error of h
    assert np.linalg.norm(hq - h) / np.linalg.norm(h) < 0.15


def _e2m1_rne_independent(v):
    """E2M1 code of fp32 values by nearest grid point, ties to the even
    mantissa (even index), |v| > 6 saturating; sign bit from the sign."""
    grid = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    a = np.abs(np.asarray(v, dtype=np.float64))
    dist = np.abs(a[:, None] - grid[None, :])
    best = dist.min(axis=1, keepdims=True)
    cand = dist == best
    even = cand & (np.arange(8) % 2 == 0)[None, :]
    m = np.where(even.any(axis=1), even.argmax(axis=1), cand.argmax(axis=1))
    return np.where(np.signbit(np.asarray(v, dtype=np.float32)), 8, 0) | m


def _nvfp4_act_dequant_independent(v):
    """Per-row NVFP4 activation quantization written from the definition, in
    fp32 with RNE: s_t = amax / 2688, per 16 values the E4M3 scale of
    amax_b / (6 s_t) (torch's RNE cast), codes E2M1(v / (scale s_t)); returns
    the dequantised values in fp64."""
    v = np.asarray(v, dtype=np.float32)
    amax = np.float32(np.abs(v).max())
    s_t = np.float32(amax / np.float32(2688.0)) if amax > 0 else np.float32(1.0)
    out = np.empty(v.size, dtype=np.float64)
    for b in range(v.size // 16):
        blk = v[16 * b:16 * b + 16]
        r = np.float32(np.abs(blk).max() / np.float32(np.float32(6.0) * s_t))
        sb = torch.tensor([min(float(r), 448.0)], dtype=torch.float32).to(torch.float8_e4m3fn)
        sval = np.float32(sb.double().item())
        if sval == 0:
            out[16 * b:16 * b + 16] = 0.0
            continue
        denom = np.float32(sval * s_t)
        codes = _e2m1_rne_independent((blk / denom).astype(np.float32))
        out[16 * b:16 * b + 16] = np.array([E2M1_GOLDEN[int(c)] for c in codes]) * float(sval) * float(s_t)
    return out


def test_w4a4_expert_matches_its_steps_in_numpy():
    """The NVFP4 prefill expert on dense rows: x quantized per block of 16 with
    one fp32 row scale, fp64 products against independently decoded weights, h
    rounded to fp32 and quantized the same way, then the down projection.
    Block magnitudes spread over several decades, so every block has its own
    scale and a wrong block size or an unquantized operand moves the result
    far beyond the tolerance."""
    d, F = 256, 128
    rec = synth.expert_record(1, 7, d, F)
    W1, W3, W2 = _matrices_independent(rec, d, F)
    rng = np.random.default_rng(44)
    for trial in range(3):
        spread = np.repeat(10.0 ** rng.uniform(-3, 1, d // 16), 16)
        x = _bf16_bits(rng.normal(0, 1, d) * spread)
        xq = _nvfp4_act_dequant_independent(_bf16_val(x).astype(np.float32))
        g, u = W1 @ xq, W3 @ xq
        h = (g * expit(g) * u).astype(np.float32)
        want = W2 @ _nvfp4_act_dequant_independent(h)
        got = oracle.expert_w4a4(rec, d, F, x)
        np.testing.assert_allclose(got, want, rtol=1e-11, atol=1e-14 * np.abs(want).max())
        exact = oracle.expert_w4a16(rec, d, F, x)[0]
        assert 1e-4 < np.linalg.norm(got - exact) / np.linalg.norm(exact) < 0.3


# ----------------------------------------------------- generator sanity --
def test_generator_weights_dequantize_near_draws():
    d, F = 256, 512
    rec = synth.expert_record(0, 2, d, F)
    for m in range(3):
        W = oracle.dequant_matrix(rec, d, F, m)
        M = synth.expert_matrix_f32(0, 2, m, d, F).astype(np.float64)
        assert np.linalg.norm(W - M) / np.linalg.norm(M) < 0.12
        assert abs(M.std() - 0.02) < 0.001


def test_ar1_statistics():
    x, _ = synth.decode_hidden_bf16(0, 0, 400, 256)
    xv = _bf16_val(x)
    assert abs(xv.var() - 1.0) < 0.1
    c = np.mean([np.corrcoef(xv[:-1, i], xv[1:, i])[0, 1] for i in range(256)])
    assert abs(c - 0.9) < 0.03


def test_layer_record_index_uses_layer_and_expert():
    s = synth.TINY
    L, P = 3, 3 * s.E - 5  # P < L*E: records alias modulo P
    rb = synth.record_bytes(s.d, s.F)
    pool = np.concatenate([synth.expert_record(i // s.E, i % s.E, s.d, s.F) for i in range(P)])
    Wr = synth.router_bf16(2, s.E, s.d)
    x = _bf16_bits(np.random.default_rng(9).normal(0, 1, (4, s.d)))
    idx, _, y = oracle.moe_layer(pool, P, 2, s.E, s.d, s.F, 1, Wr, None, x)
    for t in range(4):
        r = (2 * s.E + idx[t, 0]) % P
        np.testing.assert_array_equal(y[t], oracle.expert_w4a16(pool[r * rb:(r + 1) * rb],
                                                                s.d, s.F, x[t])[0])


# ------------------------------------------------- MXFP4 and BF16 records --
def test_e8m0_golden_points():
    for c, v in _rows("e8m0_points.txt"):
        got = oracle.e8m0(int(c, 16))
        if v == "nan":
            assert math.isnan(got)
        else:
            assert got == float(v), (c, got, v)


def _mx_tiny_record(codes_row, scale):
    """An MXFP4 record of d = 32, F = 32 whose gate row 0 holds the given 32 codes."""
    d, F = 32, 32
    off = oracle.mx_record_layout(d, F)
    rec = np.zeros(off[4], dtype=np.uint8)
    packed = [codes_row[2 * i] | (codes_row[2 * i + 1] << 4) for i in range(16)]
    rec[off[0]:off[0] + 16] = packed  # W13 row 0 (gate_0)
    rec[off[1]] = scale               # its one scale byte
    return rec, d, F


def test_mxfp4_worked_block_decodes_by_hand():
    rows = _rows("mxfp4_worked_block.txt")
    scale = int(rows[0][1], 16)
    codes = [0] * 32
    want = np.zeros(32)
    for r in rows[1:]:
        codes[int(r[0])] = int(r[2], 16)
        want[int(r[0])] = float(r[3])
    rec, d, F = _mx_tiny_record(codes, scale)
    got = oracle.dequant_matrix_mx(rec, d, F, 0)[0]
    np.testing.assert_array_equal(got, want)


def test_mxfp4_encoder_reproduces_the_worked_block():
    """The input generator's MXFP4 encoder gives the hand-derived codes and scale."""
    rows = _rows("mxfp4_worked_block.txt")
    x = np.zeros(32, dtype=np.float32)
    want = np.zeros(32, dtype=np.int64)
    for r in rows[1:]:
        x[int(r[0])] = float(r[1])
        want[int(r[0])] = int(r[2], 16)
    codes, scales = synth.mx_encode(x)
    got = np.empty(32, dtype=np.int64)
    got[0::2], got[1::2] = codes[0] & 0xF, codes[0] >> 4
    np.testing.assert_array_equal(got, want)
    assert scales[0, 0] == int(rows[0][1], 16)


def test_mxfp4_records_decode_like_an_independent_numpy_decode():
    d, F = 256, 128
    rec = synth.expert_record_mx(1, 7, d, F)
    off = oracle.mx_record_layout(d, F)
    assert off == synth.mx_record_layout(d, F)
    tab = np.array([E2M1_GOLDEN[c] for c in range(16)])

    def decode(codes, scales, rows, K):
        c = codes.reshape(rows, K // 2)
        v = np.empty((rows, K))
        v[:, 0::2] = tab[c & 0xF]
        v[:, 1::2] = tab[c >> 4]
        sc = 2.0 ** (scales.reshape(rows, K // 32).astype(np.float64) - 127)
        return v * np.repeat(sc, 32, axis=1)

    w13 = decode(rec[off[0]:off[0] + F * d], rec[off[1]:off[1] + F * d // 16], 2 * F, d)
    w2 = decode(rec[off[2]:off[2] + d * F // 2], rec[off[3]:off[3] + d * F // 32], d, F)
    np.testing.assert_array_equal(oracle.dequant_matrix_mx(rec, d, F, 0), w13[0::2])
    np.testing.assert_array_equal(oracle.dequant_matrix_mx(rec, d, F, 1), w13[1::2])
    np.testing.assert_array_equal(oracle.dequant_matrix_mx(rec, d, F, 2), w2)
    # the encoding error bound of the scale rule: X = 2^e <= amax/4 per block; an element
    # within 6X is off by at most X (half the widest E2M1 gap), a clamped one by < 2X
    for m, W in ((0, w13[0::2]), (1, w13[1::2]), (2, w2)):
        w = synth.expert_matrix_f32(1, 7, m, d, F).astype(np.float64)
        blocks = np.abs(w).reshape(-1, 32)
        X = 2.0 ** (np.floor(np.log2(blocks.max(axis=1))) - 2)
        err = np.abs(W - w).reshape(-1, 32)
        assert np.all(err <= 2 * X[:, None] + 1e-12)
        inside = blocks <= 6 * X[:, None]
        assert np.all(err[inside] <= np.broadcast_to(X[:, None], err.shape)[inside] + 1e-12)


def test_mxfp4_and_bf16_experts_match_dense_numpy():
    d, F = 256, 128
    x = _bf16_bits(np.random.default_rng(5).standard_normal(d))
    xv = _bf16_val(x)
    silu = lambda v: v * expit(v)  # noqa: E731
    rec = synth.expert_record_mx(2, 3, d, F)
    g, u = oracle.dequant_matrix_mx(rec, d, F, 0) @ xv, oracle.dequant_matrix_mx(rec, d, F, 1) @ xv
    want = oracle.dequant_matrix_mx(rec, d, F, 2) @ (silu(g) * u)
    np.testing.assert_allclose(oracle.expert_mx_w4a16(rec, d, F, x), want, rtol=1e-12, atol=1e-15)
    b = synth.expert_record_bf16(2, 0, d, F)
    w13 = _bf16_val(b[:2 * F * d]).reshape(2 * F, d)
    w2 = _bf16_val(b[2 * F * d:]).reshape(d, F)
    h = silu(w13[0::2] @ xv) * (w13[1::2] @ xv)
    np.testing.assert_allclose(oracle.expert_bf16(b, d, F, x), w2 @ h, rtol=1e-12, atol=1e-15)
    # the BF16 record holds the same draws as the NVFP4 shared record, rounded to bf16
    gate = synth.expert_matrix_f32(2, 0, 0, d, F, shared=True)
    np.testing.assert_array_equal(b[:2 * F * d].reshape(2 * F, d)[0::2], _bf16_bits(gate))


def test_layer_with_mxfp4_records_and_bf16_shared_matches_numpy():
    """The layer over MXFP4 routed records (pool indexed by MXFP4 record size)
    and an MXFP4 or BF16 shared record, against a numpy composition that
    decodes the records itself."""
    d, F, E, k, L = 256, 128, 6, 2, 2
    tab = np.array([E2M1_GOLDEN[c] for c in range(16)])
    off = synth.mx_record_layout(d, F)

    def mx(rec, which):
        lo, hi = (off[0], off[1]) if which < 2 else (off[2], off[3])
        rows, K = (2 * F, d) if which < 2 else (d, F)
        c = rec[lo:lo + rows * K // 2].reshape(rows, K // 2)
        v = np.empty((rows, K))
        v[:, 0::2], v[:, 1::2] = tab[c & 0xF], tab[c >> 4]
        v *= np.repeat(2.0 ** (rec[hi:hi + rows * K // 32].reshape(rows, K // 32) - 127.0), 32, axis=1)
        return v if which == 2 else v[which::2]

    silu = lambda v: v * expit(v)  # noqa: E731

    def expert_mx(rec, xv):
        return mx(rec, 2) @ (silu(mx(rec, 0) @ xv) * (mx(rec, 1) @ xv))

    def expert_bf(b, xv):
        w13 = _bf16_val(b[:2 * F * d]).reshape(2 * F, d)
        return _bf16_val(b[2 * F * d:]).reshape(d, F) @ (silu(w13[0::2] @ xv) * (w13[1::2] @ xv))

    pool = np.concatenate([synth.expert_record_mx(l, e, d, F) for l in range(L) for e in range(E)])
    rb = off[4]
    Wr = synth.router_bf16(1, E, d)
    x = _bf16_bits(np.random.default_rng(11).normal(0, 1, (3, d)))
    shared_mx = synth.expert_record_mx(1, 0, d, F, shared=True)
    shared_bf = synth.expert_record_bf16(1, 0, d, F)
    for P in (L * E, 5):  # record of (layer, e) is (layer*E + e) mod P
        for srec, sfmt, sfun in ((None, None, None), (shared_mx, oracle.FMT_MXFP4, expert_mx),
                                 (shared_bf, oracle.FMT_BF16, expert_bf)):
            idx, g, y = oracle.moe_layer(pool[:P * rb], P, 1, E, d, F, k, Wr, srec, x,
                                         fmt=oracle.FMT_MXFP4, shared_fmt=sfmt)
            i2, g2, _, _ = oracle.route(Wr, x, k)
            np.testing.assert_array_equal(idx, i2)
            for t in range(3):
                xv = _bf16_val(x[t])
                want = sum(g[t, j] * expert_mx(pool[((E + idx[t, j]) % P) * rb:][:rb], xv) for j in range(k))
                if srec is not None:
                    want = want + sfun(srec, xv)
                np.testing.assert_allclose(y[t], want, rtol=1e-11, atol=1e-14)
    with pytest.raises(ValueError):  # a shared record neither in the routed format nor BF16
        oracle.moe_layer(pool, L * E, 1, E, d, F, k, Wr, shared_mx, x, fmt=oracle.FMT_MXFP4,
                         shared_fmt=oracle.FMT_NVFP4)
    # the prefill path (W4A4): MXFP4 activations for MXFP4 records, a BF16 shared
    # expert unquantized
    for srec, sfmt, sfun in ((shared_mx, oracle.FMT_MXFP4, oracle.expert_mx_w4a4),
                             (shared_bf, oracle.FMT_BF16, oracle.expert_bf16)):
        idx, g, y = oracle.moe_layer(pool, L * E, 1, E, d, F, k, Wr, srec, x, w4a4=True,
                                     fmt=oracle.FMT_MXFP4, shared_fmt=sfmt)
        for t in range(3):
            want = sum(g[t, j] * oracle.expert_mx_w4a4(pool[(E + idx[t, j]) * rb:][:rb], d, F, x[t])
                       for j in range(k))
            np.testing.assert_allclose(y[t], want + sfun(srec, d, F, x[t]), rtol=1e-11, atol=1e-14)


# ------------------------------------------- MXFP4 activations (prefill) --
def test_mx_quantizer_reproduces_the_worked_block():
    """The oracle's MXFP4 activation quantizer gives the hand-derived codes and scale."""
    rows = _rows("mxfp4_worked_block.txt")
    x = np.zeros(32, dtype=np.float32)
    want = np.zeros(32, dtype=np.int64)
    for r in rows[1:]:
        x[int(r[0])] = float(r[1])
        want[int(r[0])] = int(r[2], 16)
    codes, scales = oracle.mx_quantize(x)
    got = np.empty(32, dtype=np.int64)
    got[0::2], got[1::2] = codes & 0xF, codes >> 4
    np.testing.assert_array_equal(got, want)
    assert scales[0] == int(rows[0][1], 16)


def test_mx_quantizer_matches_the_generators_encoder():
    """Two implementations of the OCP rule (the oracle's and the input
    generator's, no shared code) agree bit for bit, including zero blocks,
    -0, fp32 subnormals, huge values and exact E2M1 midpoints."""
    rng = np.random.default_rng(31)
    x = (rng.standard_normal((64, 256)) * np.exp(rng.uniform(-30, 30, (64, 1)))).astype(np.float32)
    x[0, :32] = 0.0
    x[1, :32] = -0.0
    x[2, :32] = np.float32(1e-42) * rng.integers(1, 100, 32)
    x[3, :32] = np.float32(3e38) * rng.uniform(-1, 1, 32)
    x[4, :32] = np.array([4.0, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0] * 4, dtype=np.float32)
    codes, scales = oracle.mx_quantize(x)
    c2, s2 = synth.mx_encode(x)
    np.testing.assert_array_equal(codes, c2.ravel())
    np.testing.assert_array_equal(scales, s2.ravel())


def test_mx_quantizer_round_trip_of_representable_blocks():
    """A block of E2M1 values times 2^e whose largest magnitude is 4 or 6 times
    2^e quantizes to itself (codes and scale 127 + e)."""
    rng = np.random.default_rng(32)
    for e in (-127, -60, -3, 0, 5, 120):
        for top in (6, 7):  # a 4 or a 6 in the block: amax in [4, 8) * 2^e
            codes = rng.integers(0, 16, 32)
            codes[rng.integers(32)] = top
            vals = np.array([E2M1_GOLDEN[c] for c in codes]) * 2.0 ** e
            q, s = oracle.mx_quantize(vals.astype(np.float32))
            got = np.empty(32, dtype=np.int64)
            got[0::2], got[1::2] = q & 0xF, q >> 4
            assert s[0] == 127 + e
            np.testing.assert_array_equal(np.array([E2M1_GOLDEN[c] for c in got]),
                                          np.array([E2M1_GOLDEN[c] for c in codes]))


def test_mx_w4a4_expert_matches_its_steps_in_numpy():
    """The MXFP4 prefill expert: x quantized per block of 32, fp64 products,
    h rounded to fp32 and quantized, then the down projection."""
    d, F = 256, 128
    rec = synth.expert_record_mx(3, 5, d, F)
    x = _bf16_bits(np.random.default_rng(33).normal(0, 1, d))
    tab = np.array([E2M1_GOLDEN[c] for c in range(16)])

    def deq(codes, scales):
        v = np.empty(codes.size * 2)
        v[0::2], v[1::2] = tab[codes & 0xF], tab[codes >> 4]
        return v * np.repeat(2.0 ** (scales.astype(np.float64) - 127), 32)

    silu = lambda v: v * expit(v)  # noqa: E731
    xv = deq(*oracle.mx_quantize(_bf16_val(x).astype(np.float32)))
    g = oracle.dequant_matrix_mx(rec, d, F, 0) @ xv
    u = oracle.dequant_matrix_mx(rec, d, F, 1) @ xv
    hv = deq(*oracle.mx_quantize((silu(g) * u).astype(np.float32)))
    want = oracle.dequant_matrix_mx(rec, d, F, 2) @ hv
    np.testing.assert_allclose(oracle.expert_mx_w4a4(rec, d, F, x), want, rtol=1e-11, atol=1e-14)
    # and the quantization costs what 4-bit activations cost, no more
    exact = oracle.expert_mx_w4a16(rec, d, F, x)
    assert 0 < np.linalg.norm(want - exact) / np.linalg.norm(exact) < 0.3
