"""Ownership sharding of one parameter set across ranks, on CPU.

The assignment is checked against a hand-worked LPT example and against the
textbook bound for LPT (Graham, 1969: makespan <= (4/3 - 1/(3w)) x optimum),
the optimum found by brute force. The exchange runs as gloo processes with a
stateful CPU stand-in for the per-matrix step: every rank must end with the
weights a single process computes, and every matrix must have one owner.
With the oracle's GRASP step as the per-matrix step (seeded by each matrix's
index in the set), weights and quantized states after two steps are the same
for 1, 2 and 3 ranks; seeded by the index inside each owner's batch instead,
they are not (the step-1 Rademacher start vectors move with the split).
"""

import itertools
import os
import random
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

from bit_muon_optimizer_b200 import sharding as S

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SHAPES = [(8, 16, 5), (16, 8, 3), (16, 16, 1), (8, 8, 4)]


def test_lpt_hand_worked_example():
    # 7 -> r0; 6 -> r1; 5 -> r1 (6 < 7); 4 -> r0 (7 < 11); 3 -> r0 (11 = 11, lower rank);
    # 2 -> r1 (11 < 14): loads 14 and 13
    assert S.lpt_owners([7, 6, 5, 4, 3, 2], 2) == [0, 1, 1, 0, 0, 1]
    assert S.lpt_owners([5.0], 3) == [0]
    assert S.lpt_owners([], 2) == []


@pytest.mark.parametrize("world", [2, 3])
def test_lpt_within_graham_bound(world):
    rnd = random.Random(world)
    for _ in range(20):
        costs = [rnd.randint(1, 50) for _ in range(rnd.randint(world, 8))]
        own = S.lpt_owners(costs, world)
        lpt = max(sum(c for c, o in zip(costs, own) if o == r) for r in range(world))
        best = min(max(sum(c for c, o in zip(costs, a) if o == r) for r in range(world))
                   for a in itertools.product(range(world), repeat=len(costs)))
        assert lpt <= (4 / 3 - 1 / (3 * world)) * best + 1e-9


class _StandIn:
    """Per-batch state: the number of steps taken; W -= 0.1 t G per matrix."""

    def __init__(self, m, n, ids):
        self.t = 0

    def __call__(self, W, G):
        self.t += 1
        W.sub_(0.1 * self.t * G)


class _StandInDir:
    """Per-batch state as _StandIn; the update direction O = 0.1 t G in bf16 (a
    non-finite G flags its matrix)."""

    def __init__(self, m, n, ids):
        self.t = 0

    def direction(self, G):
        self.t += 1
        flags = (~torch.isfinite(G).flatten(1).all(1)).to(torch.int32)
        return (0.1 * self.t * G).to(torch.bfloat16), flags


def _standin_update(W, Od, flags):
    keep = flags.bool()
    Wn = W - 0.5 * (Od.float() + 0.1 * W)
    W.copy_(torch.where(keep[:, None, None], W, Wn))


def _inputs(step):
    g = torch.Generator().manual_seed(100 + step)
    return [torch.randn((c, m, n), generator=g) for m, n, c in SHAPES]


def _run(world, rank, steps=2, exchange="weights"):
    if exchange == "weights":
        sh = S.ShardedStep(SHAPES, world, rank, _StandIn)
    else:
        sh = S.ShardedStep(SHAPES, world, rank, _StandInDir, update=_standin_update)
    W = [x.clone() for x in _inputs(0)]
    for t in range(1, steps + 1):
        G = _inputs(t)
        if exchange == "update" and t == 2:
            G[0][3, 1, 1] = float("nan")      # matrix 3 of group 0 is skipped in step 2
        sh(W, G)
    return sh, W


# the oracle's step on small shapes: k = 2, T = 2 NS steps
O_SHAPES = [(16, 32, 3), (32, 16, 2), (16, 16, 2)]
O_K, O_SEED = 2, 7


class _OracleStep:
    """The oracle's GRASP step for an owner batch; the Rademacher counter index b
    is each matrix's set index (``set_ids``) or its place in the batch.
    ``direction`` returns the oracle's O in bf16 instead of updating W."""

    def __init__(self, m, n, ids, set_ids=True):
        import oracle as O
        self.O = O
        self.m, self.n = m, n
        self.ids = list(ids) if set_ids else list(range(len(ids)))
        self.states = [O.zero_state(m, n, O_K) for _ in ids]

    def __call__(self, W, G):
        for i, b in enumerate(self.ids):
            r = self.O.grasp_step(self.states[i], W[i], G[i], mu=0.95, eta=0.02, seed=O_SEED, b=b,
                                  T=2)
            self.states[i] = r.state
            W[i] = r.W.float()

    def direction(self, G):
        Od = torch.empty((len(self.ids), self.m, self.n), dtype=torch.bfloat16)
        for i, b in enumerate(self.ids):
            r = self.O.grasp_step(self.states[i], torch.zeros(self.m, self.n), G[i], mu=0.95,
                                  eta=0.02, seed=O_SEED, b=b, T=2)
            self.states[i] = r.state
            Od[i] = r.O.to(torch.bfloat16)
        return Od, torch.zeros(len(self.ids), dtype=torch.int32)


def _oracle_update(W, Od, flags):
    W.sub_(0.02 * (Od.float() + 0.0 * W))


def _oracle_inputs(step):
    g = torch.Generator().manual_seed(300 + step)
    return [torch.randn((c, m, n), generator=g, dtype=torch.float64).float() * 1e-3
            for m, n, c in O_SHAPES]


def _run_oracle(world, rank, set_ids, exchange="weights"):
    steps = []

    def make(m, n, ids):
        st = _OracleStep(m, n, ids, set_ids)
        steps.append((m, n, ids, st))
        return st

    sh = S.ShardedStep(O_SHAPES, world, rank, make,
                       update=_oracle_update if exchange == "update" else None)
    W = [x.clone() * 20 for x in _oracle_inputs(0)]
    for t in (1, 2):
        sh(W, _oracle_inputs(t))
    codes = {(m, n, b): st.states[i].codes4 for m, n, ids, st in steps for i, b in enumerate(ids)}
    return W, codes


def _rank_main(rank, world, port, q, kind="standin", set_ids=True, exchange="weights"):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    torch.set_num_threads(1)
    import datetime

    import torch.distributed as dist
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        # plain arrays, pickled by value: a tensor would be shared through a file
        # descriptor that dies with this process if it exits before the parent reads
        if kind == "standin":
            sh, W = _run(world, rank, exchange=exchange)
            q.put((rank, sh.owner, [w.numpy() for w in W]))
        else:
            W, codes = _run_oracle(world, rank, set_ids, exchange)
            q.put((rank, [w.numpy() for w in W], {k: v.numpy() for k, v in codes.items()}))
    finally:
        dist.destroy_process_group()


def _spawn(world, kind="standin", set_ids=True, exchange="weights"):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q, kind, set_ids, exchange))
             for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=300) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    out = [(r, a, [torch.from_numpy(x) for x in b] if kind == "standin" else b) if kind == "standin"
           else (r, [torch.from_numpy(x) for x in a], {k: torch.from_numpy(v) for k, v in b.items()})
           for r, a, b in out]
    return sorted(out, key=lambda x: x[0])


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world", [2, 3])
def test_gloo_ranks_end_with_the_single_process_weights(world):
    _, W_ref = _run(1, 0)
    out = _spawn(world)
    owners = out[0][1]
    for rank, own, W in out:
        assert own == owners                                   # same assignment everywhere
        for a, b in zip(W, W_ref):
            assert torch.equal(a, b)
    # one owner per matrix; the 1-matrix group leaves some ranks without work in it
    assert [len(o) for o in owners] == [c for _, _, c in SHAPES]
    assert all(0 <= r < world for o in owners for r in o)
    assert len(set(owners[2])) == 1


def test_oracle_step_results_do_not_depend_on_the_world_size():
    """Two oracle GRASP steps of a small set on 1, 2 and 3 gloo ranks: every
    rank ends with the same weights, and each matrix's quantized state is the
    same whichever rank owns it, because the step is seeded by the matrix's
    index in the set. Seeded by its place in the owner's batch, the two-rank
    run departs from the one-rank run."""
    ref = _spawn(1, "oracle")[0]
    W1, codes1 = ref[1], ref[2]
    for world in (2, 3):
        out = _spawn(world, "oracle")
        codes = {}
        for _, W, c in out:
            for a, b in zip(W, W1):
                assert torch.equal(a, b)
            codes.update(c)
        assert codes.keys() == codes1.keys()
        for key in codes1:
            assert torch.equal(codes[key], codes1[key])
    local = _spawn(2, "oracle", set_ids=False)
    assert any(not torch.equal(a, b) for a, b in zip(local[0][1], W1))


@pytest.mark.parametrize("world", [2, 3])
def test_update_exchange_ranks_end_with_the_single_process_weights(world):
    """Exchanging the 16-bit update direction (with a per-matrix skip flag)
    instead of the weights: every rank ends with the weights one process
    computes, bit for bit, and the matrix whose gradient was non-finite in step
    2 kept its step-1 weights on every rank."""
    _, W_ref = _run(1, 0, exchange="update")
    _, W_one = _run(1, 0, steps=1, exchange="update")
    assert torch.equal(W_ref[0][3], W_one[0][3])
    assert not torch.equal(W_ref[0][2], W_one[0][2])
    for _, _, W in _spawn(world, exchange="update"):
        for a, b in zip(W, W_ref):
            assert torch.equal(a, b)


def test_update_exchange_oracle_results_do_not_depend_on_the_world_size():
    """The oracle's GRASP step with the bf16 O exchanged: weights and quantized
    states after two steps are the same on 1 and 2 ranks."""
    ref = _spawn(1, "oracle", exchange="update")[0]
    for _, W, c in _spawn(2, "oracle", exchange="update"):
        for a, b in zip(W, ref[1]):
            assert torch.equal(a, b)
        for key in c:
            assert torch.equal(c[key], ref[2][key])
