"""The N > 1 path of bench.py on the CPU: two gloo ranks, replicas only.

Each rank is an independent replica (its own cache, pool share and input
streams); the process group carries only the barriers and the max/sum over
ranks of the timing, which is what these tests check."""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch
    import bench
    import synth
    try:
        r, w, _ = bench.dist_setup(world, backend="gloo")
        out = {"rank": r, "world": w}
        out["max"] = bench.max_over_ranks(1.0 + r, w)  # device time of the slowest rank
        out["sum"] = bench.sum_over_ranks(10.0 * (r + 1), w)  # units processed by all ranks
        bench.barrier(w)
        out["P"] = bench.replica_pool_records(36, 128, w)
        out["x"] = bench.make_inputs(synth.TINY, 3, r)  # this replica's decode stream
        # the reference arm runs on rank 0 only; the other ranks return at once
        if r != 0:
            out["ref"] = bench.reference_arm(None, synth.TINY)
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
        q.put(out)
    except Exception as e:  # report instead of hanging the parent
        q.put({"rank": rank, "error": repr(e)})


@pytest.fixture(scope="module")
def two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    outs = [q.get(timeout=180) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        if p.is_alive():
            p.kill()
    return sorted(outs, key=lambda o: o["rank"])


def test_reductions_over_two_ranks(two_ranks):
    for o in two_ranks:
        assert "error" not in o, o
        assert o["world"] == 2
        assert o["max"] == 2.0
        assert o["sum"] == 30.0


def test_replicas_split_the_host_pool_and_draw_their_own_inputs(two_ranks):
    assert all(o["P"] == 36 * 128 // 2 for o in two_ranks)
    x0, x1 = two_ranks[0]["x"], two_ranks[1]["x"]
    assert x0.shape == x1.shape
    assert not np.array_equal(x0, x1)


def test_reference_arm_only_on_rank_zero(two_ranks):
    assert two_ranks[1]["ref"] is None


# ------------------------------------------------- expert parallelism --
def _ep_worker(rank, world, port, q):
    """One rank of an expert-parallel layer on the CPU: the oracle's routing of
    the shared input, this rank's partial output -- its own experts (e % world
    == rank), gate-weighted, plus the shared expert on rank 0 -- then the
    bench's reduce over the ranks (gloo all-reduce)."""
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch
    import bench
    import oracle
    import synth
    from synth import problem as sp
    try:
        r, w, _ = bench.dist_setup(world, backend="gloo")
        sh = synth.LayerShape("ep", L=1, E=12, k=4, d=128, F=256, shared=True, tokens=2,
                              cache_slots=8)
        rb = synth.record_bytes(sh.d, sh.F)
        pool = np.concatenate([synth.expert_record(0, e, sh.d, sh.F) for e in range(sh.E)])
        Wr = sp.router_weights(sh)
        shared = sp.shared_records(sh)
        x = bench.make_inputs(sh, 3, 0)[:, 0, 0]  # the same rows on every rank
        part = np.zeros((x.shape[0], sh.d))
        owned_any = []
        for t in range(x.shape[0]):
            idx, gates, _, _ = oracle.route(Wr[0], x[t], sh.k)
            owned = [(e, g) for e, g in zip(idx[0], gates[0]) if bench.ep_owned(int(e), r, w)]
            owned_any.append(len(owned))
            for e, g in owned:
                part[t] += g * oracle.expert_w4a16(pool[e * rb:(e + 1) * rb], sh.d, sh.F, x[t])[0]
            if r == 0:
                part[t] += oracle.expert_w4a16(shared[:rb], sh.d, sh.F, x[t])[0]
        y = torch.from_numpy(part)
        bench.ep_reduce(y, w)
        full = oracle.moe_layer(pool, sh.E, 0, sh.E, sh.d, sh.F, sh.k, Wr[0], shared[:rb], x)[2]
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
        q.put({"rank": r, "y": y.numpy(), "full": full, "owned": owned_any})
    except Exception as e:
        q.put({"rank": rank, "error": repr(e)})


def test_expert_parallel_partials_sum_to_the_layer():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_ep_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    outs = sorted([q.get(timeout=180) for _ in procs], key=lambda o: o["rank"])
    for p in procs:
        p.join(timeout=60)
        if p.is_alive():
            p.kill()
    for o in outs:
        assert "error" not in o, o
        np.testing.assert_allclose(o["y"], o["full"], rtol=1e-12, atol=1e-14)
    # both ranks did part of the work
    assert sum(outs[0]["owned"]) > 0 and sum(outs[1]["owned"]) > 0
