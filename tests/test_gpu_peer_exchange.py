"""The exchange fused into the step (gm_grasp_orth_peers): the last NS product
stores O into several receive buffers at once.

* One process, two receive buffers standing in for two ranks' memory: both get
  the O of gm_grasp_orth (same NS, same rounding), bit for bit, at the permuted
  indices dst_index names, and the step's status in their flags; a non-finite
  gradient writes the flags only.
* sharding.ShardedStep(peer=True) on one rank equals the update exchange through
  the library's weight update.
* Two processes on this GPU (gloo for the host barrier and the handle exchange,
  CUDA IPC for the buffers): each rank's owners store into both ranks' buffers,
  and both ranks end with the weights one process computes, bit for bit. The
  kernels of the two ranks never wait for one another (the ranks meet on the
  host), so sharing one GPU is safe.
"""

import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

from bit_muon_optimizer_b200 import workloads as WL

pytestmark = pytest.mark.gpu

DEV = "cuda"
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _grad(B, m, n, seed):
    return WL.random_matrix((B, m, n), seed, std=1e-3).to(torch.bfloat16)


@pytest.mark.parametrize("ns", ["standard", "gram"])
def test_orth_peers_writes_every_receive_buffer(cuda_lib, ns):
    gm = cuda_lib
    B, m, n, k = 3, 256, 384, 8
    mode = gm.GM_NS_GRAM if ns == "gram" else gm.GM_NS_STANDARD
    G = _grad(B, m, n, 71).to(DEV)
    ref = gm.GraspStep(B, m, n, k, ns=mode, seed=2, device=DEV)
    sr = gm.GraspState.zeros(B, m, n, k, DEV)
    O_ref = ref.direction(sr, G, dtype=torch.bfloat16)
    step = gm.GraspStep(B, m, n, k, ns=mode, seed=2, device=DEV)
    st = gm.GraspState.zeros(B, m, n, k, DEV)
    step.state_update(st, G)
    count = 5
    bufs = [torch.full((count, m, n), 7.0, dtype=torch.bfloat16, device=DEV) for _ in range(2)]
    flags = [torch.full((count,), -1, dtype=torch.int32, device=DEV) for _ in range(2)]
    dst = torch.tensor([4, 0, 2], dtype=torch.int64, device=DEV)
    step.orth_peers(st, [b.data_ptr() for b in bufs], [f.data_ptr() for f in flags], dst)
    torch.cuda.synchronize()
    for b_, f_ in zip(bufs, flags):
        for i, j in enumerate(dst.tolist()):
            assert torch.equal(b_[j], O_ref[i])
        for j in (1, 3):                       # indices no matrix maps to stay untouched
            assert bool((b_[j] == 7.0).all()) and int(f_[j]) == -1
        assert [int(f_[j]) for j in dst.tolist()] == [0, 0, 0]
    # a non-finite gradient: the flags say so and no O is written
    G[1, 2, 3] = float("inf")
    st2 = gm.GraspState.zeros(B, m, n, k, DEV)
    step.state_update(st2, G)
    for b_ in bufs:
        b_.fill_(7.0)
    step.orth_peers(st2, [b.data_ptr() for b in bufs], [f.data_ptr() for f in flags], dst)
    torch.cuda.synchronize()
    for b_, f_ in zip(bufs, flags):
        assert bool((b_ == 7.0).all())
        assert [int(f_[j]) for j in dst.tolist()] == [gm.GM_E_NONFINITE] * 3


SHAPES = [(256, 384, 3), (384, 256, 2), (128, 128, 4)]
K, ETA, WD, SEED = 8, 0.02, 0.1, 5


def _run_sharded(world, rank, peer, steps=2):
    from bit_muon_optimizer_b200 import sharding as S
    make = S.grasp_make_step(K, torch.device(DEV), eta=ETA, wd=WD, seed=SEED)
    sh = S.ShardedStep(SHAPES, world, rank, make, update=S.grasp_update(ETA, WD), peer=peer)
    Ws = [WL.random_matrix((c, m, n), 80 + i, std=0.02).to(DEV) for i, (m, n, c) in enumerate(SHAPES)]
    for t in range(steps):
        Gs = [_grad(c, m, n, 90 + 10 * t + i).to(DEV) for i, (m, n, c) in enumerate(SHAPES)]
        sh(Ws, Gs)
    torch.cuda.synchronize()
    out = [w.cpu() for w in Ws]
    sh.close()
    return out


def test_sharded_peer_exchange_one_rank_equals_update_exchange(cuda_lib):
    a = _run_sharded(1, 0, True)
    b = _run_sharded(1, 0, False)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=120))
    try:
        Ws = _run_sharded(world, rank, True)
        dist.barrier()   # nobody frees a receive buffer another rank still maps
        q.put((rank, [w.numpy() for w in Ws]))
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_processes_share_one_gpu_through_ipc(cuda_lib):
    ref = _run_sharded(1, 0, True)
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=600) for _ in procs]
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    for _, Ws in out:
        for a, b in zip(Ws, ref):
            assert torch.equal(torch.from_numpy(a), b)
