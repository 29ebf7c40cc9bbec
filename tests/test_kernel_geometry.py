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
        nsteps = (K // 64 + 3) // 4
        warps = (nsteps + (2 if nsteps >= 8 else 1) - 1) // (2 if nsteps >= 8 else 1)
        smem = 3 * (code_bytes + scale_bytes) + 2 * warps * 2 * 512  # ring + two partials buffers (NG 2)
        assert smem <= 160 * 1024  # dynamic shared memory limit set at launch
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


@pytest.mark.parametrize("nitems,G", [(1440, 296), (720, 296), (360, 296), (5, 296), (296, 296),
                                      (4 * 2560, 148), (1, 1), (7, 3)])
def test_persistent_gemv_items_cover_each_item_once(nitems, G):
    """CTA b takes items b, b + G, ...: its count is (nitems - 1 - b) // G + 1 when b < nitems."""
    seen = []
    for b in range(min(G, nitems)):
        n_my = (nitems - 1 - b) // G + 1 if b < nitems else 0
        seen += [b + j * G for j in range(n_my)]
    assert sorted(seen) == list(range(nitems))


@pytest.mark.parametrize("nvalid,tiles", [(4, 360), (4, 180), (11, 96), (1, 360), (138, 128)])
def test_combine_ticket_reaches_the_count_once_per_tile(nvalid, tiles):
    """Expert-major items: each tile receives one ticket per valid expert, so the
    count nvalid - 1 is reached exactly once per tile, after all its partials."""
    tickets = [0] * tiles
    combined = []
    for item in range(nvalid * tiles):  # any completion order gives the same counts
        t = item % tiles
        if tickets[t] == nvalid - 1:
            combined.append(t)
        tickets[t] += 1
    assert sorted(combined) == list(range(tiles))


PREFILL = [s for s in SHAPES if s.d >= 256 and s.F >= 256]


@pytest.mark.parametrize("shape", PREFILL, ids=lambda s: s.name)
def test_grouped_gemm_boxes_and_scale_words_inside_their_tensors(shape):
    """The tcgen05 grouped GEMM: TMA boxes of 128 bytes x 128 rows start on
    16-byte x coordinates inside each operand's row; the scale words a CTA loads
    lie inside the record's scale section (weights) or the grouped rows
    (activations); tensor-memory columns and shared memory fit."""
    dims = abi.make_dims(shape.L, shape.E, shape.k, shape.d, shape.F, shape.shared)
    off = abi.moe_record_layout(dims)
    assert 128 + 3 * 4 * 8 <= 256  # accumulator + scale-factor columns of one CTA
    smem = 2 * 3 * 128 * 128 + 2 * 3 * 4 * 512 + 128 + 1024
    assert smem <= 113 * 1024  # two CTAs per SM
    for K, rows_w, sf0, sf_end in ((shape.d, 2 * shape.F, off[1], off[2]),
                                   (shape.F, shape.d, off[3], off[5])):
        ksteps, nkb = K // 64, (K // 64 + 3) // 4
        m_tiles = (rows_w + 127) // 128
        assert (K // 2) % 16 == 0 and K // 2 >= 128
        for it in range(nkb):
            x = it * 128
            assert x % 16 == 0 and x < K // 2  # box start inside the row (the tail is zero-filled)
        pitch = K // 16
        assert pitch % 4 == 0
        last_word = (rows_w - 1) * pitch + 4 * (ksteps - 1) + 4
        assert sf0 + last_word <= sf_end
        assert m_tiles * 128 >= rows_w


@pytest.mark.parametrize("seed", range(20))
def test_grouped_gemm_pair_capacity_bounds_the_tile_plan(seed):
    """sum over jobs of ceil(rows / 128), plus the shared expert's tiles, never
    exceeds the capacity the host sizes the grid and buffers with."""
    import numpy as np
    rng = np.random.default_rng(seed)
    T, k = int(rng.integers(33, 4097)), int(rng.integers(1, 33))
    E = int(rng.integers(k, 1025))
    sel = np.stack([rng.choice(E, k, replace=False) for _ in range(min(T, 64))])
    sel = np.concatenate([sel] * (T // len(sel)) + [sel[:T % len(sel)]])
    counts = np.bincount(sel.ravel(), minlength=E)
    jobs = counts[counts > 0]
    for shared in (0, 1):
        need = int(np.sum((jobs + 127) // 128)) + (shared * ((T + 127) // 128))
        cap = len(jobs) + (T * k + 127) // 128 + (shared * ((T + 127) // 128))
        assert need <= cap


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: s.name)
def test_mxfp4_tile_copies_and_scale_reads(shape):
    """The GEMV's MXFP4 instantiation: a 16-row tile stages 16 * K/2 code bytes
    and 16 * K/32 = K/2 scale bytes; both copies lie inside their record
    sections on 16-byte boundaries; a thread's two E8M0 bytes of chunk c of
    tile row r (a 16-bit read at r * K/32 + 2c) are aligned and inside the
    staged scales; shared memory fits."""
    dims = abi.make_dims(shape.L, shape.E, shape.k, shape.d, shape.F, shape.shared,
                         weight_format=abi.MOE_FMT_MXFP4)
    off = abi.moe_record_layout(dims)
    assert off[4] == -1 and all(o % 256 == 0 for i, o in enumerate(off) if i != 4)
    for K, tiles, codes0, scales0, end in ((shape.d, shape.F // 8, off[0], off[1], off[2]),
                                           (shape.F, shape.d // 16, off[2], off[3], off[5])):
        code_bytes, scale_bytes = 16 * (K // 2), K // 2
        assert code_bytes % 16 == 0 and scale_bytes % 16 == 0
        nsteps = (K // 64 + 3) // 4
        spw = 2 if nsteps >= 8 else 1
        warps = (nsteps + spw - 1) // spw
        assert 3 * (code_bytes + scale_bytes) + 2 * warps * 2 * 512 <= 160 * 1024
        for t in (0, tiles - 1):
            assert (codes0 + t * code_bytes) % 16 == 0 and (scales0 + t * scale_bytes) % 16 == 0
            assert codes0 + (t + 1) * code_bytes <= scales0
            assert scales0 + (t + 1) * scale_bytes <= end
        nch = K // 64
        for r in (0, 7, 8, 15):
            for c in (0, nch - 1):
                o = r * (K // 32) + 2 * c
                assert o % 2 == 0 and o + 2 <= scale_bytes


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: s.name)
def test_bf16_shared_reads_inside_record(shape):
    """The BF16 shared-expert GEMV: warp j of gate/up reads W13 rows 2j, 2j+1 in
    16-byte chunks, warp i of down reads W2 rows 2i, 2i+1; all inside the 6dF
    bytes of the record and 16-byte aligned (the record's pitch keeps them)."""
    d, F = shape.d, shape.F
    dims = abi.make_dims(shape.L, shape.E, shape.k, d, F, True, shared_format=abi.MOE_FMT_BF16)
    rb = abi.moe_shared_record_bytes(dims)
    assert rb == 6 * d * F and rb % 16 == 0
    for K, rows, base in ((d, 2 * F, 0), (F, d, 4 * F * d)):
        nch = K // 8
        last_row = base + (rows - 1) * K * 2
        assert base % 16 == 0 and (K * 2) % 16 == 0
        assert last_row + 16 * (nch - 1) + 16 <= (4 * F * d if base == 0 else rb)


def test_mxfp4_step_factoring_keeps_products_exact():
    """(Imports the oracle: test infrastructure.)  A numpy model of the MXFP4 GEMV's arithmetic (per 256-value K-step and
    row: the largest E8M0 code c_max factored out, weights e2m1 * 2^(c - c_max
    + 12) rounded to fp16, activations as fp16 (hi, lo), fp32 step sums scaled
    by 2^(c_max - 139)) against the oracle's fp64 expert, on scales spread by
    25 codes inside a step with some blocks 80+ codes below: the products stay
    exact, so only fp32 summation separates the two."""
    import numpy as np
    import oracle
    import synth

    d, F = 320, 192
    rng = np.random.default_rng(41)
    rec = synth.expert_record_mx(0, 3, d, F).copy()
    off = synth.mx_record_layout(d, F)
    for start, n in ((off[1], 2 * F * d // 32), (off[3], d * F // 32)):
        c = rng.integers(99, 125, n)
        tiny = rng.random(n) < 0.02
        c[tiny] = rng.integers(20, 41, int(tiny.sum()))
        rec[start:start + n] = c.astype(np.uint8)
    tab = np.array([0, .5, 1, 1.5, 2, 3, 4, 6, 0, -.5, -1, -1.5, -2, -3, -4, -6])

    def gemv(codes, scales, K, act):
        v = np.empty((codes.shape[0], K))
        v[:, 0::2], v[:, 1::2] = tab[codes & 0xF], tab[codes >> 4]
        hi = act.astype(np.float16)
        lo = (act - hi.astype(np.float32)).astype(np.float16)
        out = np.zeros(codes.shape[0], np.float32)
        for k0 in range(0, K, 256):
            k1 = min(K, k0 + 256)
            sc = scales[:, k0 // 32:(k1 + 31) // 32].astype(np.int64)
            cmax = sc.max(axis=1)
            w = (v[:, k0:k1] * np.exp2(np.repeat(sc - cmax[:, None], 32, axis=1)[:, :k1 - k0] + 12.0))
            w16 = w.astype(np.float16).astype(np.float64)
            assert np.array_equal(w16[np.abs(w) >= 2.0 ** -24], w[np.abs(w) >= 2.0 ** -24])  # exact
            stp = (w16 @ hi[k0:k1].astype(np.float64) + w16 @ lo[k0:k1].astype(np.float64)).astype(np.float32)
            out = out + stp * np.exp2(cmax - 139.0).astype(np.float32)
        return out

    x = synth.to_bf16(rng.normal(0, 1, d).astype(np.float32))
    xf = synth.bf16_to_f32(x).astype(np.float32)
    c13 = rec[off[0]:off[0] + F * d].reshape(2 * F, d // 2)
    s13 = rec[off[1]:off[1] + 2 * F * d // 32].reshape(2 * F, d // 32)
    gu = gemv(c13, s13, d, xf)
    g, u = gu[0::2], gu[1::2]
    h = (g / (1 + np.exp(-g)) * u).astype(np.float32)
    y = gemv(rec[off[2]:off[2] + d * F // 2].reshape(d, F // 2),
             rec[off[3]:off[3] + d * F // 32].reshape(d, F // 32), F, h)
    want = oracle.expert_mx_w4a16(rec, d, F, x)
    assert np.linalg.norm(y - want) / np.linalg.norm(want) < 1e-6


# ------------------------------------------------------- decode layer kernel --
def _layer_decode(i, H, M, nA, nB):
    """Mirror of the layer kernel's queue decode: (expert slot, gate_up, tile, miss)."""
    per = nA + nB
    if i < H * nA:
        return (i // nA, 1, i % nA, -1)
    if i < H * per:
        j = i - H * nA
        return (j // nB, 0, j % nB, -1)
    j = i - H * per
    m, r = divmod(j, per)
    return (H + m, 1 if r < nA else 0, r if r < nA else r - nA, m)


@pytest.mark.parametrize("H,M", [(1, 0), (0, 3), (7, 0), (4, 2), (11, 10), (1, 32)])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: s.name)
def test_layer_queue_covers_every_tile_once_in_dependency_order(shape, H, M):
    """Every (expert, phase, tile) once; each down tile after all gate/up tiles of
    its expert (so a waiting CTA only waits on tiles held by running CTAs); the
    misses in the order the host copies them, each miss's gate/up before its down."""
    nA, nB = shape.F // 8, shape.d // 16
    total = (H + M) * (nA + nB)
    seen = {}
    for i in range(total):
        key = _layer_decode(i, H, M, nA, nB)
        assert key[:3] not in seen
        seen[key[:3]] = i
    assert len(seen) == total
    for (x, gu, t), i in seen.items():
        if not gu:
            assert all(seen[(x, 1, a)] < i for a in range(nA))
    firsts = [min(i for (x, gu, t), i in seen.items() if x == H + m) for m in range(M)]
    assert firsts == sorted(firsts)
    assert all(_layer_decode(i, H, M, nA, nB)[3] == -1 for i in range(H * (nA + nB)))


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: s.name)
@pytest.mark.parametrize("mx", [False, True])
def test_layer_kernel_ring_fits_and_keeps_two_ctas_per_sm_where_it_can(shape, mx):
    """The launcher's choice: a 3-tile ring when two CTAs still fit an SM (227 KB of
    shared memory, ~5 KB static per CTA), else 2; the ring covers the longer K."""
    Kmax = max(shape.d, shape.F)
    nsteps = (Kmax // 64 + 3) // 4
    spw = 2 if nsteps >= 8 else 1
    warps = (nsteps + spw - 1) // spw
    buf = 16 * (Kmax // 2) + (Kmax // 2 if mx else Kmax)
    for ng in (1, 2):
        red = 2 * warps * ng * 4 * 32 * 4
        smem3 = 3 * buf + red
        S = 3 if 2 * (smem3 + 6 * 1024) <= 227 * 1024 else 2
        smem = S * buf + red
        assert smem <= 200 * 1024
        assert buf % 16 == 0  # every stage starts on a cp.async boundary
        if S == 2:
            assert smem + 6 * 1024 <= 227 * 1024  # one CTA fits with room for the static part


# ------------------------------------------------ streaming expert kernel --
def _stream_launch(d, F, T, k, max_exp, mx, sms=148):
    """launch_stream's sizing, restated: stage bytes, tiles per item (gate/up,
    down), stages, consumer groups, metadata, row-ref and x offsets, grid.  A
    stage holds an item's codes and scales, 16 bytes of tensor scales and, with
    activations in shared memory (T <= 2), a down item's h rows."""
    sa = T <= 2
    xbytes = T * 4 * d if sa else 0
    hbytes = T * 4 * F if sa else 0
    tA = 8 * d + (d // 2 if mx else d)
    tB = 8 * F + (F // 2 if mx else F)
    sb = max(tA + 16, tB + 16 + hbytes, 16 * 1024)
    sb = (sb + 127) & ~127
    nA, nB = F // 8, d // 16
    want = 3 * sms

    def per_item(room, tile_bytes, tiles_per_exp):
        tp = room // tile_bytes
        tiles = tiles_per_exp * max_exp
        while tp > 1 and tiles // tp < want:
            tp -= 1
        return max(tp, 1)

    tpa, tpb = per_item(sb - 16, tA, nA), per_item(sb - 16 - hbytes, tB, nB)
    meta = (max_exp * 40 + 15) & ~15
    rr = (T * k * 4 + 15) & ~15
    budget = 200 * 1024
    assert meta + rr + xbytes + 2 * sb <= budget
    ns = min((budget - meta - rr - xbytes) // sb, 8)
    nc = ns // 2 if ns >= 6 else min(ns, 5)
    if nc > 4 and ns >= 6:
        nc = 4
    ns = (2 if ns >= 2 * nc else 1) * nc
    return dict(sb=sb, tpa=tpa, tpb=tpb, ns=ns, nc=nc, meta_off=ns * sb, rr_off=ns * sb + meta,
                x_off=ns * sb + meta + rr, xbytes=xbytes, hbytes=hbytes,
                smem=ns * sb + meta + rr + xbytes, nA=nA, nB=nB, cbA=8 * d, sbA=d // 2 if mx else d,
                cbB=8 * F, sbB=F // 2 if mx else F)


def _stream_items(L, nexp, phase):
    """st_item over a launch: (expert, gate_up, tile0, nt) in global item order."""
    iA = -(-L["nA"] // L["tpa"])
    iB = -(-L["nB"] // L["tpb"])
    total = nexp * ((iA if phase & 1 else 0) + (iB if phase & 2 else 0))
    gA = nexp * iA if phase & 1 else 0
    out = []
    for g in range(total):
        if g < gA:
            e, j = divmod(g, iA)
            t0 = j * L["tpa"]
            out.append((e, 1, t0, min(L["tpa"], L["nA"] - t0)))
        else:
            e, j = divmod(g - gA, iB)
            t0 = j * L["tpb"]
            out.append((e, 0, t0, min(L["tpb"], L["nB"] - t0)))
    return out


@pytest.mark.parametrize("mx", [False, True], ids=["nvfp4", "mxfp4"])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: s.name)
def test_stream_items_fit_their_stage_and_stay_in_the_record(shape, mx):
    fmt = abi.MOE_FMT_MXFP4 if mx else abi.MOE_FMT_NVFP4
    dims = abi.make_dims(shape.L, shape.E, shape.k, shape.d, shape.F, shape.shared, weight_format=fmt)
    off = abi.moe_record_layout(dims)  # w13 codes, w13 scales, w2 codes, w2 scales, tensor scales, bytes
    # the hit launch (every selected expert + the shared one), and a miss's own
    # launch (one expert: its gate/up, then its down tiles)
    for T, max_exp in [(T, m) for T in (1, 4, 16, 32) for m in (min(T * shape.k, shape.E) + 1, 1)]:
        L = _stream_launch(shape.d, shape.F, T, shape.k, max_exp, mx)
        assert 2 <= L["ns"] <= 8 and 2 <= L["nc"] <= 7
        # each stage serves one consumer warp: the uses of a stage are waited on in order
        assert L["ns"] % L["nc"] == 0
        for l in range(64):
            assert (l % L["ns"]) % L["nc"] == l % L["nc"]
        assert L["smem"] <= 200 * 1024 and L["meta_off"] % 128 == 0 and L["rr_off"] % 8 == 0
        assert L["x_off"] % 16 == 0 and L["xbytes"] % 16 == 0 and (4 * shape.F) % 16 == 0
        for phase in (1, 2, 3):
            nexp = min(max_exp, 3)
            items = _stream_items(L, nexp, phase)
            seen = set()
            first_down = None
            for n, (e, gu, t0, nt) in enumerate(items):
                assert nt >= 1
                cb, sb = (L["cbA"], L["sbA"]) if gu else (L["cbB"], L["sbB"])
                codes0, scales0, end = (off[0], off[1], off[2]) if gu else (off[2], off[3], off[5])
                # the stage: codes of nt tiles, their scales, 16 bytes of tensor
                # scales, then (down items, T <= 2) the expert's h rows
                assert nt * (cb + sb) + 16 + (0 if gu else L["hbytes"]) <= L["sb"]
                assert (nt * (cb + sb)) % 16 == 0
                assert (nt * cb) % 16 == 0 and (nt * sb) % 16 == 0
                # the two bulk copies: 16-byte aligned, inside their record section
                c0, s0 = codes0 + t0 * cb, scales0 + t0 * sb
                assert c0 % 16 == 0 and s0 % 16 == 0
                assert c0 + nt * cb <= scales0 and s0 + nt * sb <= end
                for t in range(t0, t0 + nt):
                    assert (e, gu, t) not in seen
                    seen.add((e, gu, t))
                if not gu and first_down is None:
                    first_down = n
                if gu:  # gate/up items precede every down item (phase 3's dependency order)
                    assert first_down is None
            want = set()
            for e in range(nexp):
                if phase & 1:
                    want |= {(e, 1, t) for t in range(L["nA"])}
                if phase & 2:
                    want |= {(e, 0, t) for t in range(L["nB"])}
            assert seen == want


def test_stream_k_step_reads_stay_inside_the_tile():
    """The K-step's shared-memory reads (rows rA/rB <= 15, chunk c < K/64, 32 code
    bytes and 4 (NVFP4) or 2 (MXFP4) scale bytes per row and chunk) end at the
    tile's code and scale sizes exactly."""
    for K in (256, 320, 768, 960, 2048, 2880, 4096):
        nch = K // 64
        assert 15 * (K // 2) + 32 * (nch - 1) + 32 == 8 * K
        assert 15 * (K // 16) + 4 * (nch - 1) + 4 == K
        assert 15 * (K // 32) + 2 * (nch - 1) + 2 == K // 2


def test_topk_order_key_preserves_the_selection_order():
    """The route kernels' warp argmax compares order-preserving 32-bit keys of
    the logits (a max reduction, then the lowest id holding it): the key must be
    monotone in the value, give -0 and +0 the same key, keep -inf the smallest,
    and invert exactly."""
    import numpy as np

    def key(v):
        v = np.where(v == 0, np.float32(0), v).astype(np.float32)
        u = v.view(np.uint32)
        return np.where(u & np.uint32(0x80000000), ~u, u | np.uint32(0x80000000)).astype(np.uint32)

    def value(k):
        u = np.where(k & np.uint32(0x80000000), k & np.uint32(0x7fffffff), ~k).astype(np.uint32)
        return u.view(np.float32)

    rng = np.random.default_rng(7)
    vals = np.concatenate([
        np.array([-np.inf, -3.4e38, -1.0, -1e-45, -0.0, 0.0, 1e-45, 1.0, 3.4e38, np.inf], np.float32),
        rng.standard_normal(4000).astype(np.float32) * np.float32(50),
        (rng.standard_normal(500) * 1e-40).astype(np.float32)])  # subnormals
    k = key(vals)
    order_v = np.argsort(vals, kind="stable")
    assert np.all(np.diff(k[order_v].astype(np.int64)) >= 0)          # monotone
    assert key(np.array([-0.0], np.float32))[0] == key(np.array([0.0], np.float32))[0]
    finite_or_inf = vals[vals == vals]
    assert key(np.array([-np.inf], np.float32))[0] == key(finite_or_inf).min()
    back = value(k)
    same = np.where(vals == 0, np.float32(0), vals)
    assert np.array_equal(back.view(np.uint32), same.view(np.uint32))  # exact inverse



def _route_split(E, d, sms=148, warps=8):
    """launch_route_lookup's choice, restated: warps per router row (1, 2, 4 or
    8) while the grid stays within one CTA per SM, the row's 16-byte vectors
    divide evenly and every lane keeps at least one of its segment."""
    nvec = d // 8
    split = 1
    while split < 8 and E * 2 * split <= warps * sms and nvec % (2 * split) == 0 and nvec // (2 * split) >= 32:
        split *= 2
    grid = -(-E // (warps // split))
    nv = -(-(nvec // split) // 32)
    return split, grid, nv


@pytest.mark.parametrize("E", [1, 2, 8, 40, 100, 128, 256, 512, 1000, 1024])
@pytest.mark.parametrize("d", [64, 192, 256, 960, 2048, 2880, 4096])
def test_route_row_split_covers_every_row_and_vector_once(E, d):
    """Every (row, 16-byte vector) of the router is loaded by exactly one lane
    of one warp, segments of a row are consecutive warps of one CTA (their
    partial sums meet in that CTA's shared memory, slots warp .. warp + S - 1),
    the grid fits one CTA per SM once split, and NV covers a segment."""
    split, grid, nv = _route_split(E, d)
    assert split in (1, 2, 4, 8) and nv in range(1, 17)
    assert split == 1 or grid <= 148
    nvec = d // 8
    assert nvec % split == 0
    segv = nvec // split
    assert nv * 32 >= segv
    seen = {}
    for b in range(grid):
        for warp in range(8):
            seg, row = warp % split, b * (8 // split) + warp // split
            if row >= E:
                continue
            assert warp - seg + split <= 8  # the row's warps (its partial-sum slots) lie in the CTA
            for lane in range(32):
                for i in range(nv):
                    v = lane + 32 * i
                    if v < segv:
                        key = (row, seg * segv + v)
                        assert key not in seen
                        seen[key] = (b, warp, lane)
    assert len(seen) == E * nvec
