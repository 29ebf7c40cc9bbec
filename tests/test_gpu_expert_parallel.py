"""Expert parallelism (moe_set_expert_shard): the layer split over G ranks by
expert id, e mod G.  On one GPU the G shard contexts run one after another --
no kernel of one waits on another -- and their partial outputs are summed
here, as an all-reduce would sum them across GPUs.  Against the oracle: each
rank's cache trace is the LRU over its own experts (bit-exact, with the
table), the sum of the partials is the whole layer (1e-3 relative L2 per
row), and a rank that owns none of a step's experts contributes zero."""
import numpy as np
import pytest
import torch

import synth
from oracle.workloads import decode_trace
from expert_offload_caching_b200 import abi
from expert_offload_caching_b200.runtime import LayerStack, new_trace, trace_events
from synth import problem as sp
from tests.gpu_problem import REL_L2_MAX, DecodeProblem, rel_l2
from tests.test_gpu_decode import MID

pytestmark = pytest.mark.gpu


def _shard_run(pb, rank, size):
    sh = pb.shape
    st = LayerStack(pb.dims(), pb.pool, sp.to_device(pb.Wr), sp.to_device(pb.shared), pb.C,
                    shard=(rank, size))
    xd = torch.from_numpy(pb.x).cuda()
    y = torch.zeros((pb.T, sh.L, pb.S, sh.d), device="cuda")
    torch.cuda.synchronize()
    tr, arr = new_trace(2 * sh.E + 8)
    events = []
    for t in range(pb.T):
        for l in range(sh.L):
            st.forward(l, xd[t, l], y[t, l], tr)
            events += [(t, l, e[1], e[2], e[3], e[4]) for e in trace_events(tr, arr)]
    st.synchronize()
    m = np.empty(sh.L * sh.E, np.int32)
    o = np.empty(pb.C, np.int32)
    s = np.empty(pb.C, np.uint64)
    clock = abi.moe_cache_export(st.ctx, m, o, s)
    stats = abi.moe_get_stats(st.ctx)
    return st, events, y, (m, o, s, clock), stats


@pytest.mark.parametrize("size,S", [(2, 1), (8, 1), (3, 5)])
def test_shards_sum_to_the_layer(size, S):
    pb = DecodeProblem(MID, T=10, streams=S, C=min(S * MID.k, MID.E) + 6, stream0=600)
    idx, _ = pb.oracle_routing()
    total = None
    empty_seen = False
    for rank in range(size):
        st, events, y, table, stats = _shard_run(pb, rank, size)
        want, lru = decode_trace(idx, MID.L, MID.E, pb.C, shard=(rank, size))
        assert events == want
        wm, wo, ws, wc = lru.state()
        np.testing.assert_array_equal(table[0], wm)
        np.testing.assert_array_equal(table[1], wo)
        np.testing.assert_array_equal(table[2], ws)
        assert table[3] == wc
        assert stats.lookups == len(events)
        pb.check_slots(st, table[1])
        yn = y.cpu().numpy()
        for t in range(pb.T):
            for l in range(MID.L):
                owned = [e for e in np.unique(idx[t, l]) if e % size == rank]
                if not owned and rank != 0:
                    assert not yn[t, l].any()  # nothing owned, no shared expert: zero
                    empty_seen = True
        total = yn if total is None else total + yn
        st.close()
    for t in range(pb.T):
        for l in range(MID.L):
            want_y = pb.oracle_y(t, l)
            for r in range(S):
                assert rel_l2(total[t, l, r], want_y[r]) <= REL_L2_MAX, (t, l, r)
    if size == 8:
        assert empty_seen  # 5 of 40 experts per step over 8 ranks: some rank owns none


def test_shard_argument_checks():
    pb = DecodeProblem(synth.TINY, T=1)
    st = pb.stack()
    for rank, size in ((0, 0), (2, 2), (-1, 2), (0, 17)):
        with pytest.raises(abi.MoeError) as ei:
            abi.moe_set_expert_shard(st.ctx, rank, size)
        assert ei.value.status == abi.MOE_ERR_ARG
    abi.moe_set_expert_shard(st.ctx, 1, 2)
    x = torch.zeros((1, synth.TINY.d), dtype=torch.uint16, device="cuda")
    y = torch.zeros((1, synth.TINY.d), device="cuda")
    with pytest.raises(abi.MoeError) as ei:  # a new shard needs a reset first
        st.forward(0, x, y)
    assert ei.value.status == abi.MOE_ERR_STATE
    st.reset()
    st.forward(0, x, y)
    st.synchronize()
    st.close()


@pytest.mark.parametrize("fmt,shared_fmt", [(sp.FMT_NVFP4, None), (sp.FMT_MXFP4, sp.FMT_BF16)],
                         ids=["nvfp4", "mxfp4+bf16-shared"])
def test_prefill_shards_sum_to_the_layer(fmt, shared_fmt):
    """A prefill chunk under expert parallelism (2 ranks, prefetch on): each
    rank's routed and prefetch batches hold its own experts only (trace and
    table equal the oracle's LRU over them), the grouped GEMMs run over its
    rows only, and the partials sum to the oracle's W4A4 layer row by row."""
    from oracle.workloads import prefill_trace
    from tests.test_gpu_prefill import PF, PrefillProblem
    import oracle
    pb = PrefillProblem(PF, T=200, fmt=fmt, shared_fmt=shared_fmt)
    total = None
    want_idx = np.stack([oracle.route(pb.Wr[l], pb.x[l], PF.k)[0] for l in range(PF.L)])
    for rank in range(2):
        sh = PF
        dims = abi.make_dims(sh.L, sh.E, sh.k, sh.d, sh.F, sh.shared, True, pb.T, 0, weight_format=fmt,
                             shared_format=pb.shared_fmt)
        st = LayerStack(dims, pb.pool, sp.to_device(pb.Wr), sp.to_device(pb.shared), pb.C, prefetch=True,
                        shard=(rank, 2))
        events, idx, gates, y = pb.run(st)
        np.testing.assert_array_equal(idx, want_idx)
        want_ev, lru = prefill_trace(want_idx, sh.L, sh.E, pb.C, prefetch=True, shard=(rank, 2))
        assert events == want_ev
        m = np.empty(sh.L * sh.E, np.int32)
        o = np.empty(pb.C, np.int32)
        s_ = np.empty(pb.C, np.uint64)
        clock = abi.moe_cache_export(st.ctx, m, o, s_)
        wm, wo, ws, wc = lru.state()
        np.testing.assert_array_equal(m, wm)
        np.testing.assert_array_equal(o, wo)
        assert clock == wc
        total = y if total is None else total + y
        st.close()
    for l in range(PF.L):
        want = pb.oracle_y(l, np.arange(pb.T))
        for r in range(pb.T):
            assert rel_l2(total[l][r], want[r]) <= REL_L2_MAX, (l, r)
