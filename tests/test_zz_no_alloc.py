"""moe_route_noalloc: routing with no workspace, for callers that cannot
allocate device memory when they run (a framework that owns the device memory
pool, a process whose memory is planned up front).  Its scratch lives in an
array inside the library.  Checked against the routing that moe_layer_forward
computes on the same rows, on two calls in a row (the shared scratch keeps the
previous call's contents, which must not leak into the next result).

This file is collected last on purpose."""
import numpy as np
import pytest
import torch

import synth
from expert_offload_caching_b200 import abi
from tests.gpu_problem import DecodeProblem

pytestmark = pytest.mark.gpu

MID = synth.LayerShape("mid", L=3, E=40, k=5, d=960, F=320, shared=True, tokens=4, cache_slots=24)


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
        idx_d = torch.full((S, k), -1, dtype=torch.int32, device="cuda")
        gates_d = torch.full((S, k), -1.0, dtype=torch.float32, device="cuda")
        torch.cuda.synchronize()
        abi.moe_route_noalloc(st.router_w[l], xd[t, l], S, E, d, k, True, idx_d, gates_d, stream)
        outs.append(((t, l), idx_d, gates_d))
    stream.synchronize()
    for (t, l), idx_d, gates_d in outs:
        want_idx, want_g = ref[(t, l)]
        np.testing.assert_array_equal(idx_d.cpu().numpy(), want_idx)
        np.testing.assert_allclose(gates_d.cpu().numpy(), want_g, rtol=2e-5, atol=1e-7)


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
