"""Ownership sharding of one parameter set across data-parallel ranks.

Muon needs each weight's whole gradient matrix, and every matrix's GRASP step
is independent of the others ("Achieving low-bit Muon through subspace
preservation and grid quantization": overall framework; its limitations
section describes quantizing per partition on top of distributed Muon). So a
set of 2-D weights splits by ownership: each matrix has one owner rank, which
alone keeps its quantized momentum and runs its step; the owners' updated
weights are then all-gathered so that every rank holds the whole set again.

Owners come from LPT greedy (longest processing time first) on a per-matrix
cost, by default the step's Newton-Schulz FLOP scaling m n min(m, n). Every
rank computes the same assignment from the same shapes, so no communication
decides it.

The per-matrix update is injected: ``make_step(m, n, ids)`` returns a callable
``step(W, G)`` that updates a contiguous [len(ids), m, n] fp32 weight batch in
place from a gradient batch of the same shape and keeps whatever state it
needs (the library's GRASP step on a GPU; any stand-in in tests). ``ids`` are
the batch's indices in the whole parameter set (groups in order, matrices in
order within a group): the step seeds its per-matrix random draws (the
Rademacher start vectors) from them, so a matrix's results do not depend on
the number of ranks or on which rank owns it. The exchange is one all-gather
per shape group through ``torch.distributed`` (NCCL on GPUs), each rank
sending its owned matrices padded to the largest owner's count.

Two things can be exchanged. By default the owners update their weights and
send the updated fp32 weights (4 B per element). Given an ``update`` callable,
the owners instead send the orthogonalized update O of worked step 6 in 16
bits (2 B per element, half the bytes) with one skip flag per matrix, and
every rank, owners included, applies W <- W - eta (O + wd W) to its own copy
through ``update(W, O, flags)``: all ranks apply the same O to the same W, so
they keep identical weights. The step object then provides
``direction(G) -> (O, flags)`` instead of updating W.

With ``peer=True`` (and an ``update``) the exchange is fused into the step: each
rank holds receive buffers for O and the flags of every shape group, mapped into
every other rank's address space through CUDA IPC, and the owners' last NS
product stores O straight into all of them (``orth_peers(G, peer_O, peer_flags,
dst_index)`` of the step object: gm_grasp_orth_peers), peers' over NVLink; a
stream synchronize and a barrier later every rank applies the update. Receive
buffers alternate between two sets from one call to the next, so a rank that
runs ahead never writes a buffer another rank may still be reading.
"""

from __future__ import annotations

from typing import Callable, Sequence

import torch
import torch.distributed as dist


def ns_cost(m: int, n: int) -> float:
    """NS FLOPs of one m x n matrix up to a constant factor: N^2 M' = m n min(m, n)."""
    return float(m) * n * min(m, n)


def lpt_owners(costs: Sequence[float], world: int) -> list[int]:
    """LPT greedy: items in order of decreasing cost (ties by index), each to
    the rank with the smallest load so far (ties to the lower rank). Returns the
    owner of every item."""
    if world < 1:
        raise ValueError("world must be >= 1")
    order = sorted(range(len(costs)), key=lambda i: (-costs[i], i))
    load = [0.0] * world
    owner = [0] * len(costs)
    for i in order:
        r = min(range(world), key=lambda q: (load[q], q))
        owner[i] = r
        load[r] += costs[i]
    return owner


class ShardedStep:
    """One optimizer step of a parameter set split by ownership.

    ``shapes`` lists the set's shape groups as (m, n, count), in order; the
    call takes, per group, the [count, m, n] weights (updated in place on
    every rank) and the matching gradients (every rank holds all of them, as
    after a data-parallel all-reduce). ``first_index`` is the set index of the
    first matrix (for a part of a larger set handled on its own)."""

    def __init__(self, shapes: Sequence[tuple[int, int, int]], world: int, rank: int,
                 make_step: Callable[[int, int, list], Callable], cost=ns_cost, group=None,
                 first_index: int = 0, update: Callable | None = None,
                 update_dtype: torch.dtype = torch.bfloat16, peer: bool = False):
        if not 0 <= rank < world:
            raise ValueError(f"rank {rank} outside world {world}")
        self.shapes = [tuple(s) for s in shapes]
        self.world, self.rank, self.group = world, rank, group
        self.update, self.update_dtype = update, update_dtype
        if peer and update is None:
            raise ValueError("the fused peer exchange delivers the update direction: give update")
        self.peer = peer
        self._bufs: dict = {}      # group -> two (O, flags) PeerBuffers sets
        self._idx: dict = {}       # group -> device int64 indices of this rank's matrices
        self._calls = 0
        costs = [cost(m, n) for m, n, count in self.shapes for _ in range(count)]
        flat = lpt_owners(costs, world)
        self.owner: list[list[int]] = []          # owner of matrix i of group g
        self.owned: list[list[list[int]]] = []    # owned[g][r]: indices rank r owns in g
        self.base: list[int] = []                 # set index of each group's first matrix
        pos = 0
        for m, n, count in self.shapes:
            own = flat[pos:pos + count]
            self.base.append(first_index + pos)
            pos += count
            self.owner.append(own)
            self.owned.append([[i for i in range(count) if own[i] == r] for r in range(world)])
        self.steps = [make_step(m, n, [base + i for i in o[rank]]) if o[rank] else None
                      for (m, n, _), o, base in zip(self.shapes, self.owned, self.base)]

    def loads(self, cost=ns_cost) -> list[float]:
        """Total cost each rank owns."""
        load = [0.0] * self.world
        for (m, n, _), own in zip(self.shapes, self.owner):
            for r in own:
                load[r] += cost(m, n)
        return load

    def __call__(self, Ws: Sequence[torch.Tensor], Gs: Sequence[torch.Tensor]) -> None:
        if len(Ws) != len(self.shapes) or len(Gs) != len(self.shapes):
            raise ValueError("one weight and one gradient tensor per shape group")
        self._call(Ws, Gs)
        self._calls += 1

    def _call(self, Ws, Gs) -> None:
        for g, ((m, n, count), W, G) in enumerate(zip(self.shapes, Ws, Gs)):
            if tuple(W.shape) != (count, m, n) or tuple(G.shape) != (count, m, n):
                raise ValueError(f"group {g}: expected [{count}, {m}, {n}] weights and gradients")
            mine = self.owned[g][self.rank]
            if self.peer:
                self._exchange_peer(g, m, n, count, W, G)
                continue
            if self.update is not None:
                self._exchange_update(g, m, n, count, W, G)
                continue
            Wb = None
            if mine:
                idx = torch.tensor(mine, device=W.device)
                Wb = W.index_select(0, idx)
                self.steps[g](Wb, G.index_select(0, idx))
            if self.world == 1:
                if Wb is not None:
                    W.index_copy_(0, idx, Wb)
                continue
            width = max(len(o) for o in self.owned[g])
            send = torch.zeros((width, m, n), dtype=W.dtype, device=W.device)
            if Wb is not None:
                send[:len(mine)] = Wb
            recv = [torch.empty_like(send) for _ in range(self.world)]
            dist.all_gather(recv, send, group=self.group)
            for r, own in enumerate(self.owned[g]):
                if own:
                    W.index_copy_(0, torch.tensor(own, device=W.device), recv[r][:len(own)])

    def _exchange_peer(self, g, m, n, count, W, G):
        """Owners' NS stores O and flags into every rank's receive buffers; after a
        barrier every rank applies all of them to its W."""
        if g not in self._bufs:
            mk = lambda shape, dt: PeerBuffers(shape, dt, W.device, self.world, self.rank,  # noqa: E731
                                                self.group)
            self._bufs[g] = [(mk((count, m, n), self.update_dtype), mk((count,), torch.int32))
                             for _ in range(2)]
            self._idx[g] = torch.tensor(self.owned[g][self.rank], dtype=torch.int64, device=W.device)
        Ob, Fb = self._bufs[g][self._calls & 1]
        mine = self.owned[g][self.rank]
        if mine:
            idx = self._idx[g]
            self.steps[g].orth_peers(G.index_select(0, idx), Ob.ptrs, Fb.ptrs, idx)
        if self.world > 1:
            torch.cuda.current_stream(W.device).synchronize()   # this rank's stores are done
            dist.barrier(group=self.group)                        # and every other rank's
        self.update(W, Ob.local, Fb.local)

    def close(self) -> None:
        """Unmaps the other ranks' receive buffers (every rank calls it)."""
        for sets in self._bufs.values():
            for Ob, Fb in sets:
                Ob.close()
                Fb.close()
        self._bufs.clear()

    def _exchange_update(self, g, m, n, count, W, G):
        """Owners send (O, flags); every rank applies all of them to its W."""
        mine = self.owned[g][self.rank]
        O = flags = None
        if mine:
            idx = torch.tensor(mine, device=W.device)
            O, flags = self.steps[g].direction(G.index_select(0, idx))
        if self.world == 1:
            self.update(W, O, flags)         # the one rank owns every matrix, in order
            return
        width = max(len(o) for o in self.owned[g])
        send = torch.zeros((width, m, n), dtype=self.update_dtype, device=W.device)
        sendf = torch.ones((width,), dtype=torch.int32, device=W.device)
        if mine:
            send[:len(mine)] = O
            sendf[:len(mine)] = flags
        recv = [torch.empty_like(send) for _ in range(self.world)]
        recvf = [torch.empty_like(sendf) for _ in range(self.world)]
        dist.all_gather(recv, send, group=self.group)
        dist.all_gather(recvf, sendf, group=self.group)
        O_all = torch.empty((count, m, n), dtype=self.update_dtype, device=W.device)
        f_all = torch.empty((count,), dtype=torch.int32, device=W.device)
        for r, own in enumerate(self.owned[g]):
            if own:
                t = torch.tensor(own, device=W.device)
                O_all.index_copy_(0, t, recv[r][:len(own)])
                f_all.index_copy_(0, t, recvf[r][:len(own)])
        self.update(W, O_all, f_all)


class PeerBuffers:
    """One zeroed device buffer per rank, and on every rank the addresses of all of
    them: its own, and the other ranks' mapped through CUDA IPC (gm_ipc_export /
    gm_ipc_open). Collective: every rank constructs it alike."""

    def __init__(self, shape, dtype, device, world: int, rank: int, group=None):
        from . import gmuon as gm
        self.local = torch.zeros(shape, dtype=dtype, device=device)
        self._opened: list[int] = []
        self.ptrs = [self.local.data_ptr()]
        if world > 1:
            handles: list = [None] * world
            dist.all_gather_object(handles, gm.ipc_export(self.local), group=group)
            self.ptrs = []
            for r, (h, off) in enumerate(handles):
                if r == rank:
                    self.ptrs.append(self.local.data_ptr())
                else:
                    base = gm.ipc_open(h)
                    self._opened.append(base)
                    self.ptrs.append(base + off)

    def close(self) -> None:
        from . import gmuon as gm
        for base in self._opened:
            gm.ipc_close(base)
        self._opened = []


def grasp_make_step(k: int, device=None, sub_batch_elements: float | None = None,
                    **params) -> Callable[[int, int, list], Callable]:
    """``make_step`` for the library's GRASP step: each owner batch gets its own
    step object and zero state (its quantized momentum lives on this rank only),
    with the batch's set indices as the step's matrix ids. A batch above
    ``sub_batch_elements`` (default: offload.SUB_BATCH_ELEMENTS) is stepped as
    several library calls on contiguous sub-batches sharing one workspace, the
    same results bit for bit; ``state`` then carries the first sub-batch's step
    count and the first non-zero sub-batch status after every call."""
    from . import gmuon as gm
    from .offload import SUB_BATCH_ELEMENTS, chunk_bounds, sub_batch_size

    limit = SUB_BATCH_ELEMENTS if sub_batch_elements is None else sub_batch_elements

    def make(m: int, n: int, ids: list):
        B = len(ids)
        state = gm.GraspState.zeros(B, m, n, k, device)
        bounds = chunk_bounds(B, sub_batch_size(B, m, n, limit))
        if len(bounds) == 1:
            step = gm.GraspStep(B, m, n, k, device=device, matrix_ids=ids, **params)

            def run(W: torch.Tensor, G: torch.Tensor) -> None:
                step(state, W, G)

            def direction(G: torch.Tensor):
                O = step.direction(state, G)
                return O, state.dev_status.expand(B).contiguous()

            def orth_peers(G: torch.Tensor, peer_O, peer_flags, dst_index) -> None:
                step.state_update(state, G)
                step.orth_peers(state, peer_O, peer_flags, dst_index)
        else:
            sizes = sorted({e - a for a, e in bounds})
            ns = params.get("ns", gm.GM_NS_STANDARD)
            ws = torch.empty(max(gm.workspace_bytes(gm.GM_OP_GRASP_STEP, c, m, n, k, ns) for c in sizes),
                             dtype=torch.uint8, device=device)
            steps = {c: gm.GraspStep(c, m, n, k, device=device, ws=ws, matrix_ids=ids[:c], **params)
                     for c in sizes}
            status = torch.zeros(len(bounds), dtype=torch.int32, device=device)
            subs = []
            for i, (a, e) in enumerate(bounds):
                st = gm.GraspState(state.codes4[a:e], state.rscale[a:e], state.cscale[a:e],
                                   state.P8[a:e], state.Pscale[a:e], state.R8[a:e], state.Rscale[a:e],
                                   torch.zeros(1, dtype=torch.int64, device=device), status[i:i + 1])
                subs.append((a, e, steps[e - a], st,
                             torch.tensor(ids[a:e], dtype=torch.int64, device=device)))
            counts = torch.tensor([e - a for a, e in bounds], device=device)

            def settle() -> None:
                """The batch's step count and first non-zero status into ``state``."""
                state.step.copy_(subs[0][3].step)
                first = (status != 0).to(torch.int32).argmax()   # 0 when all are clean
                state.dev_status.copy_(status.index_select(0, first.view(1)))

            def each(fn) -> None:
                for a, e, stp, st, sid in subs:
                    stp.ids.copy_(sid, non_blocking=True)
                    fn(a, e, stp, st)
                settle()

            def run(W: torch.Tensor, G: torch.Tensor) -> None:
                each(lambda a, e, stp, st: stp(st, W[a:e], G[a:e]))

            def direction(G: torch.Tensor):
                O = torch.empty((B, m, n), dtype=torch.bfloat16, device=device)
                each(lambda a, e, stp, st: stp.direction(st, G[a:e], out=O[a:e]))
                return O, status.repeat_interleave(counts, output_size=B)

            def orth_peers(G: torch.Tensor, peer_O, peer_flags, dst_index) -> None:
                def one(a, e, stp, st):
                    stp.state_update(st, G[a:e])
                    stp.orth_peers(st, peer_O, peer_flags, dst_index[a:e])
                each(one)

        run.state = state
        run.direction = direction
        run.orth_peers = orth_peers
        return run

    return make


def grasp_update(eta: float, wd: float = 0.0) -> Callable:
    """``update`` for ShardedStep: the library's weight update (gm_weight_update),
    each matrix skipped when its owner's step flagged a non-finite value."""
    from . import gmuon as gm

    def update(W: torch.Tensor, O: torch.Tensor, flags: torch.Tensor) -> None:
        gm.weight_update(W, O, eta, wd, skip=flags)

    return update
