"""moe_route_noalloc: routing with no workspace, for callers that cannot
allocate device memory when they run (a framework that owns the device memory
pool, a process whose memory is planned up front).  Its scratch lives in an
array inside the library.  Checked against the routing that moe_layer_forward
computes on the same rows, and against the oracle's routing, on calls in a row
(the shared scratch keeps the previous call's contents, which must not leak
into the next result).

This file is collected last on purpose."""
import numpy as np
import pytest
import torch

import oracle
import synth
from oracle.workloads import conditioned_prefill
from expert_offload_caching_b200 import abi
from tests.gpu_problem import DecodeProblem

pytestmark = pytest.mark.gpu

MID = synth.LayerShape("mid", L=3, E=40, k=5, d=960, F=320, shared=True, tokens=4, cache_slots=24)


def _noalloc(Wr_d, x_d, T, E, d, k, renorm, stream):
    """One call on `stream`.  The caller keeps Wr_d and x_d alive until the stream
    has synchronised: the kernel reads them there, after this returns, and the
    caching allocator may hand a freed block to the next allocation at once."""
    idx_d = torch.full((T, k), -1, dtype=torch.int32, device="cuda")
    gates_d = torch.full((T, k), -1.0, dtype=torch.float32, device="cuda")
    torch.cuda.synchronize()
    abi.moe_route_noalloc(Wr_d, x_d, T, E, d, k, renorm, idx_d, gates_d, stream)
    return idx_d, gates_d


def test_noalloc_routing_matches_layer_forward_on_two_calls():
    pb = DecodeProblem(MID, T=3, streams=3, C=24)
    st = pb.stack()
    S, k, E, d = pb.S, MID.k, MID.E, MID.d
    xd = torch.from_numpy(pb.x).cuda()
    y = torch.zeros((S, d), device="cuda")
    torch.cuda.synchronize()
    ref = {}
    for t, l in [(0, 1), (2, 2)]:  # routing from the existing entry point
        st.forward(l, xd[t, l], y)
        idx = np.empty((S, k), np.int32)
        gates = np.empty((S, k), np.float32)
        abi.moe_get_routing(st.ctx, idx, gates, S)
        ref[(t, l)] = (idx, gates)
    st.synchronize()

    stream = torch.cuda.Stream()
    outs = []
    for t, l in [(0, 1), (2, 2)]:  # two calls in a row through the C ABI
        idx_d, gates_d = _noalloc(st.router_w[l], xd[t, l], S, E, d, k, True, stream)
        outs.append(((t, l), idx_d, gates_d))
    stream.synchronize()
    for (t, l), idx_d, gates_d in outs:
        want_idx, want_g = ref[(t, l)]
        np.testing.assert_array_equal(idx_d.cpu().numpy(), want_idx)
        np.testing.assert_allclose(gates_d.cpu().numpy(), want_g, rtol=2e-5, atol=1e-7)


def test_noalloc_full_scratch_matches_the_oracle():
    """32 rows x 1024 experts fill the built-in logits array, k = 32, and the
    router has 128 CTAs, so the selection runs in the last CTA to finish.  Two
    calls in a row: renormalised gates, then the plain softmax probabilities,
    on other rows.  Ids bit-exact, gates within rtol 2e-5 of the oracle's."""
    E, d, k, T = 1024, 256, 32, 32
    Wr = synth.router_bf16(0, E, d)
    xa = conditioned_prefill(Wr, k, 0, T)[0]
    xb = conditioned_prefill(Wr, k, 1, T)[0]
    Wr_d = torch.from_numpy(Wr).cuda()
    xs_d = [torch.from_numpy(xa).cuda(), torch.from_numpy(xb).cuda()]
    stream = torch.cuda.Stream()
    got = []
    for x, x_d, renorm in [(xa, xs_d[0], True), (xb, xs_d[1], False)]:
        got.append((x, renorm) + _noalloc(Wr_d, x_d, T, E, d, k, renorm, stream))
    stream.synchronize()
    for x, renorm, idx_d, gates_d in got:
        want_idx, want_g, _, _ = oracle.route(Wr, x, k, renorm=renorm)
        np.testing.assert_array_equal(idx_d.cpu().numpy(), want_idx)
        np.testing.assert_allclose(gates_d.cpu().numpy(), want_g, rtol=2e-5, atol=1e-7)
        if not renorm:
            assert float(gates_d.sum(1).max()) < 1.0  # probabilities of 32 of 1024 experts


def test_noalloc_ragged_expert_count_after_a_larger_call():
    """E = 1000 (not a multiple of 8 or 32) right after a 1024-expert call: the
    previous call's logits are still in the array and must not leak."""
    stream = torch.cuda.Stream()
    Wbig = synth.router_bf16(2, 1024, 256)
    xbig = conditioned_prefill(Wbig, 32, 2, 32)[0]
    big_d = (torch.from_numpy(Wbig).cuda(), torch.from_numpy(xbig).cuda())
    _noalloc(big_d[0], big_d[1], 32, 1024, 256, 32, True, stream)
    E, d, k, T = 1000, 192, 7, 5
    Wr = synth.router_bf16(3, E, d)
    x = conditioned_prefill(Wr, k, 3, T)[0]
    small_d = (torch.from_numpy(Wr).cuda(), torch.from_numpy(x).cuda())
    idx_d, gates_d = _noalloc(small_d[0], small_d[1], T, E, d, k, True, stream)
    stream.synchronize()
    want_idx, want_g, _, _ = oracle.route(Wr, x, k)
    np.testing.assert_array_equal(idx_d.cpu().numpy(), want_idx)
    np.testing.assert_allclose(gates_d.cpu().numpy(), want_g, rtol=2e-5, atol=1e-7)


def test_noalloc_non_finite_rows_follow_the_selection_rule():
    """Rows holding -inf, NaN and +inf: NaN logits count as -inf and equal
    logits go to the lower id, so valid ids come out (the oracle's selection);
    the gates are NaN on both sides.  A finite row in the same call is exact."""
    E, d, k = 40, 192, 5
    Wr = synth.router_bf16(4, E, d)
    x = conditioned_prefill(Wr, k, 4, 4)[0]
    x[0, 3] = synth.to_bf16(np.array([-np.inf], np.float32))[0]
    x[1, 7] = synth.to_bf16(np.array([np.nan], np.float32))[0]
    x[2, 0] = synth.to_bf16(np.array([np.inf], np.float32))[0]
    stream = torch.cuda.Stream()
    in_d = (torch.from_numpy(Wr).cuda(), torch.from_numpy(x).cuda())
    idx_d, gates_d = _noalloc(in_d[0], in_d[1], 4, E, d, k, True, stream)
    stream.synchronize()
    want_idx, want_g, _, _ = oracle.route(Wr, x, k)
    got_idx = idx_d.cpu().numpy()
    np.testing.assert_array_equal(got_idx, want_idx)
    assert got_idx.min() >= 0 and got_idx.max() < E
    np.testing.assert_allclose(gates_d.cpu().numpy(), want_g, rtol=2e-5, atol=1e-7)  # NaN == NaN
    assert np.isnan(want_g[:3]).all() and np.isfinite(want_g[3]).all()


def test_noalloc_rejects_sizes_beyond_its_scratch():
    w = torch.zeros((8, 64), dtype=torch.uint16, device="cuda")
    x = torch.zeros((33, 64), dtype=torch.uint16, device="cuda")
    out_i = torch.zeros((33, 2), dtype=torch.int32, device="cuda")
    out_g = torch.zeros((33, 2), dtype=torch.float32, device="cuda")
    s = torch.cuda.Stream()
    with pytest.raises(abi.MoeError) as ei:  # 33 rows > 32
        abi.moe_route_noalloc(w, x, 33, 8, 64, 2, True, out_i, out_g, s)
    assert ei.value.status == abi.MOE_ERR_UNSUPPORTED
    with pytest.raises(abi.MoeError) as ei:  # k > E
        abi.moe_route_noalloc(w, x, 1, 8, 64, 9, True, out_i, out_g, s)
    assert ei.value.status == abi.MOE_ERR_ARG


def test_noalloc_rejects_unaligned_operands_before_launching():
    """Rows are read as 16-byte vectors: an operand 2 bytes off a 16-byte
    boundary is refused on the host (nothing is launched)."""
    w = torch.zeros((8 * 64 + 8,), dtype=torch.uint16, device="cuda")
    x = torch.zeros((2 * 64 + 8,), dtype=torch.uint16, device="cuda")
    out_i = torch.zeros((2, 2), dtype=torch.int32, device="cuda")
    out_g = torch.zeros((2, 2), dtype=torch.float32, device="cuda")
    s = torch.cuda.Stream()
    for wv, xv in [(w[1:1 + 8 * 64], x[:2 * 64]), (w[:8 * 64], x[1:1 + 2 * 64])]:
        with pytest.raises(abi.MoeError) as ei:
            abi.moe_route_noalloc(wv, xv, 2, 8, 64, 2, True, out_i, out_g, s)
        assert ei.value.status == abi.MOE_ERR_ARG
