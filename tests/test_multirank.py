"""The bench's multi-rank logic on CPU: two gloo processes take the same barrier
and max-over-ranks steps as the GPU ranks do, and draw disjoint parameter sets
(weak scaling: no collective on the data path)."""

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
        wl = WL.WORKLOADS[2]
        bases = [(bench.matrix_base(wl, gi, r_), wl.groups[gi].count) for gi in range(len(wl.groups))]
        ref = bench.run_reference(None, w_, r_) if r_ != 0 else None   # rank != 0: no work
        bench.barrier(w_)
        q.put((r_, w_, t, bases, ref))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_barrier_max_and_disjoint_sets():
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
    sets = []
    for _, _, _, bases, _ in out:
        idx = set()
        for base, count in bases:
            idx.update(range(base, base + count))
        sets.append(idx)
    assert len(sets[0]) == len(sets[1]) == 84                      # 48 + 24 + 12 matrices per rank
    assert not (sets[0] & sets[1])
