"""The bench's multi-rank logic on CPU: two gloo processes take the same barrier
and max-over-ranks steps as the GPU ranks do, and split each shape group of the
benchmarked parameter set into disjoint owner batches that cover it (the
ownership sharding the bench drives at N > 1); the reference arm runs on rank 0
only."""

import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    from bit_muon_optimizer_b200 import workloads as WL
    import torch.distributed as dist
    w_, r_, _ = bench.init_dist(world)
    try:
        bench.barrier(w_)
        t = bench.max_over_ranks(1.5 * (r_ + 1), w_)
        from bit_muon_optimizer_b200 import sharding as S
        wl = WL.WORKLOADS[4]
        owned = []
        for gi, g in enumerate(wl.groups):
            ids = []
            S.ShardedStep([(g.m, g.n, g.count)], w_, r_, lambda m, n, i: ids.extend(i) or (lambda W, G: None),
                          first_index=wl.group_base(gi))
            owned.append(ids)
        ref = bench.run_reference(None, w_, r_) if r_ != 0 else None   # rank != 0: no work
        bench.barrier(w_)
        q.put((r_, w_, t, owned, ref))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_barrier_max_and_owner_split():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    out.sort()
    assert [o[0] for o in out] == [0, 1] and all(o[1] == 2 for o in out)
    assert all(o[2] == pytest.approx(3.0) for o in out)            # max over ranks of 1.5, 3.0
    assert out[1][4] is None
    from bit_muon_optimizer_b200 import workloads as WL
    wl = WL.WORKLOADS[4]
    for gi, g in enumerate(wl.groups):
        a, b = set(out[0][3][gi]), set(out[1][3][gi])
        assert not (a & b)
        assert a | b == set(range(wl.group_base(gi), wl.group_base(gi) + g.count))
        assert abs(len(a) - len(b)) <= 1                            # equal costs: balanced
