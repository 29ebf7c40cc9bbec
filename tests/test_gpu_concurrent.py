"""Concurrent decode at the Qwen3.8-Flash-Next shape (512 routed experts, top-10
+ shared, d 2048, F 768): a 4096-row prefill chunk, then steps of 16 rows
(16 independent AR(1) streams, batch 16) on the same cache, each step's lookup
batch the union of the 16 rows' selections (about 138 distinct experts per
layer).  Against the oracle: expert ids, the whole event trace (prefill and
decode), the table and sampled slot bytes bit for bit, outputs of sampled
(step, layer) pairs within 1e-3 relative L2 per row.

Two caches: the bench's 6144 slots with next-layer prefetch (every expert of
these few layers stays resident: the decode steps are all hits), and 700
slots without prefetch, so the prefill chunk evicts and the decode steps miss
and evict too."""
import numpy as np
import pytest
import torch

import oracle
import synth
from oracle.workloads import conditioned_decode, decode_trace
from expert_offload_caching_b200 import abi
from expert_offload_caching_b200.runtime import new_trace, trace_events
from tests.gpu_problem import REL_L2_MAX, rel_l2
from tests.test_gpu_prefill import PrefillProblem, _check

pytestmark = pytest.mark.gpu

QW = synth.QWEN38
S = 16  # concurrent streams


@pytest.mark.parametrize("L,C,prefetch,steps", [(3, QW.cache_slots, True, 4), (3, 700, False, 6)],
                         ids=["6144-slots-prefetch", "700-slots-evicting"])
def test_qwen_shaped_chunk_then_16_streams(L, C, prefetch, steps):
    sh = synth.LayerShape(QW.name, L=L, E=QW.E, k=QW.k, d=QW.d, F=QW.F, shared=True, tokens=0,
                          cache_slots=C)
    pb = PrefillProblem(sh, T=4096, P=97, C=C)
    st = pb.stack(prefetch)
    events, idx, gates, y = pb.run(st)
    rows = np.sort(np.random.default_rng(5).choice(4096, 8, replace=False))
    lru = _check(pb, st, events, idx, gates, y, prefetch, rows=rows)

    xdec = np.empty((steps, L, S, sh.d), np.uint16)
    for s in range(S):
        for l in range(L):
            xdec[:, l, s] = conditioned_decode(pb.Wr[l], sh.k, 400 + s, l, steps)[0]
    xd = torch.from_numpy(xdec).cuda()
    yd = torch.zeros((steps, L, S, sh.d), device="cuda")
    torch.cuda.synchronize()
    tr, arr = new_trace(2 * sh.E + 8)
    got, union = [], []
    gidx = np.empty((steps, L, S, sh.k), np.int32)
    for t in range(steps):
        for l in range(L):
            st.forward(l, xd[t, l], yd[t, l], tr)
            ev = trace_events(tr, arr)
            union.append(len(ev))
            got += [(t, l, e[1], e[2], e[3], e[4]) for e in ev]
            gates_t = np.empty((S, sh.k), np.float32)
            abi.moe_get_routing(st.ctx, gidx[t, l], gates_t, S)
    st.synchronize()
    didx = np.stack([[oracle.route(pb.Wr[l], xdec[t, l], sh.k)[0] for l in range(L)]
                     for t in range(steps)])
    np.testing.assert_array_equal(gidx, didx)
    want, lru = decode_trace(didx, L, sh.E, C, lru=lru)
    assert len(got) == len(want)
    for g, w in zip(got, want):
        assert g == w, (g, w)
    assert 100 < np.mean(union) < 180  # the union of 16 rows' top-10 of 512
    hits = sum(e[4] for e in got)
    if prefetch:
        assert hits == len(got)
    else:
        assert 0 < hits < len(got) and any(e[5] >= 0 for e in got)

    m = np.empty(L * sh.E, np.int32)
    o = np.empty(C, np.int32)
    s_ = np.empty(C, np.uint64)
    clock = abi.moe_cache_export(st.ctx, m, o, s_)
    wm, wo, ws, wc = lru.state()
    np.testing.assert_array_equal(m, wm)
    np.testing.assert_array_equal(o, wo)
    np.testing.assert_array_equal(s_, ws)
    assert clock == wc
    slots = np.random.default_rng(6).choice(np.nonzero(o >= 0)[0], 24, replace=False)
    for sl in slots:
        r = int(o[sl]) % pb.P
        want_b = pb.pool[r * pb.rb:(r + 1) * pb.rb].cuda()
        assert torch.equal(st.arena[int(sl) * pb.rb:(int(sl) + 1) * pb.rb], want_b), sl

    ydn = yd.cpu().numpy()
    shared = [pb.shared[l * pb.rb:(l + 1) * pb.rb] for l in range(L)]
    for t, l in [(0, 0), (steps - 1, L - 1), (steps // 2, 1)]:
        want_y = oracle.moe_layer(pb.pool.numpy(), pb.P, l, sh.E, sh.d, sh.F, sh.k, pb.Wr[l],
                                  shared[l], xdec[t, l])[2]
        for r in range(S):
            assert rel_l2(ydn[t, l, r], want_y[r]) <= REL_L2_MAX, (t, l, r)
    st.close()
