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
