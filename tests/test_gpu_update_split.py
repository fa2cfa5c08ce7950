"""Worked step 6 split at O: gm_grasp_orth writes O = NS(M_t), gm_weight_update
applies W <- W - eta (O + wd W).

* gm_weight_update against the update written out in fp64 on the same W and O:
  within two fp32 roundings of the result (the kernel may fuse the multiply-adds);
  skip flags (one per batch, one per matrix) leave the flagged weights untouched.
* state update + orth (O in fp32) + weight update against the fused step: the
  same state bit for bit, W within fp32 rounding; with O in bf16, within eta
  times bf16's half-ulp of O. O itself against the fp64 oracle's NS of the
  same M_t within the NS bar (relative Frobenius 2e-2).
* a non-finite gradient: orth writes nothing and the update, skipped on the
  state's flag, leaves W alone.
"""

import pytest
import torch

import oracle as O
from bit_muon_optimizer_b200 import workloads as WL

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _outlier(B, m, n, seed, std=1e-3, dtype=torch.float32):
    X = WL.random_matrix((B, m, n), seed, std=std)
    g = torch.Generator().manual_seed(seed + 1)
    for b in range(B):
        X[b, torch.randperm(m, generator=g)[:2], :] *= 10
        X[b, :, torch.randperm(n, generator=g)[:2]] *= 10
    return X.to(dtype)


@pytest.mark.parametrize("odt", [torch.float32, torch.bfloat16, torch.float16])
@pytest.mark.parametrize("B,m,n", [(3, 144, 272), (1, 16, 48), (2, 512, 1024)])
def test_weight_update_against_fp64(cuda_lib, odt, B, m, n):
    gm = cuda_lib
    W = WL.random_matrix((B, m, n), 11, std=0.02)
    Ov = (WL.random_matrix((B, m, n), 12, std=1.0) / (m * n) ** 0.25).to(odt)
    eta, wd = float(torch.tensor(0.02)), float(torch.tensor(0.1))   # fp32 values, as the kernel sees them
    ref = W.double() - eta * (Ov.double() + wd * W.double())
    Wd = W.to(DEV)
    gm.weight_update(Wd, Ov.to(DEV), eta, wd)
    torch.cuda.synchronize()
    err = (Wd.cpu().double() - ref).abs()
    bound = 2 * 2.0 ** -23 * (W.double().abs() + eta * (Ov.double().abs() + wd * W.double().abs())) * 2
    assert bool((err <= bound + 1e-30).all())


def test_weight_update_skip_flags(cuda_lib):
    gm = cuda_lib
    B, m, n = 4, 64, 96
    W = WL.random_matrix((B, m, n), 13, std=0.02).to(DEV)
    Ov = WL.random_matrix((B, m, n), 14, std=0.1).to(torch.bfloat16).to(DEV)
    W0 = W.clone()
    flags = torch.tensor([0, 1, 0, 1], dtype=torch.int32, device=DEV)
    gm.weight_update(W, Ov, 0.5, 0.0, skip=flags)
    torch.cuda.synchronize()
    for b in range(B):
        assert torch.equal(W[b], W0[b]) == bool(flags[b].item())
    W1 = W.clone()
    gm.weight_update(W, Ov, 0.5, 0.0, skip=torch.ones(1, dtype=torch.int32, device=DEV))
    torch.cuda.synchronize()
    assert torch.equal(W, W1)


@pytest.mark.parametrize("ns", ["standard", "gram"])
@pytest.mark.parametrize("B,m,n", [(2, 256, 640), (3, 272, 144)])
def test_orth_and_update_equal_the_fused_step(cuda_lib, ns, B, m, n):
    gm = cuda_lib
    k, eta, wd = 16, 0.02, 0.1
    mode = gm.GM_NS_GRAM if ns == "gram" else gm.GM_NS_STANDARD
    W0 = WL.random_matrix((B, m, n), 21, std=0.02).to(DEV)
    grads = [_outlier(B, m, n, 22 + t, dtype=torch.bfloat16).to(DEV) for t in (1, 2)]
    fused = gm.GraspStep(B, m, n, k, eta=eta, wd=wd, ns=mode, seed=3, device=DEV)
    sf = gm.GraspState.zeros(B, m, n, k, DEV)
    Wf = W0.clone()
    runs = {}
    for odt in (torch.float32, torch.bfloat16):
        step = gm.GraspStep(B, m, n, k, eta=eta, wd=wd, ns=mode, seed=3, device=DEV)
        runs[odt] = (step, gm.GraspState.zeros(B, m, n, k, DEV), W0.clone())
    for G in grads:
        fused(sf, Wf, G)
        for odt, (step, st, W) in runs.items():
            Od = step.direction(st, G, dtype=odt)
            M = step.stage_M().double().cpu()
            gm.weight_update(W, Od, eta, wd, skip=st.dev_status)
            torch.cuda.synchronize()
            for a, b in zip(st.tensors(), sf.tensors()):
                assert torch.equal(a, b)
            if odt == torch.float32:
                for b in range(B):
                    ref = O.gram_ns(M[b], None, 5, (2,)) if ns == "gram" else O.ns_standard(M[b], None, 5)
                    e = float((Od[b].double().cpu() - ref).norm() / ref.norm())
                    assert e <= 2e-2, (b, e)
    for odt, (step, st, W) in runs.items():
        d = (W - Wf).abs().max().item()
        if odt == torch.float32:
            tol = 4 * 2.0 ** -23 * Wf.abs().max().item() + 2 * eta * 2.0 ** -22
        else:
            tol = 2 * eta * 2.0 ** -8 + 4 * 2.0 ** -23 * Wf.abs().max().item()
        assert d <= tol, (odt, d, tol)


def test_orth_writes_nothing_after_a_nonfinite_state_update(cuda_lib):
    gm = cuda_lib
    B, m, n, k = 2, 256, 256, 8
    step = gm.GraspStep(B, m, n, k, device=DEV)
    st = gm.GraspState.zeros(B, m, n, k, DEV)
    W = WL.random_matrix((B, m, n), 31, std=0.02).to(DEV)
    G = WL.random_matrix((B, m, n), 32, std=1e-3).to(DEV)
    G[1, 5, 7] = float("nan")
    Ov = torch.full((B, m, n), 3.0, dtype=torch.bfloat16, device=DEV)
    W1 = W.clone()
    step.direction(st, G, out=Ov)
    gm.weight_update(W, Ov, 0.02, 0.1, skip=st.dev_status)
    torch.cuda.synchronize()
    assert int(st.dev_status.item()) == gm.GM_E_NONFINITE
    assert bool((Ov == 3.0).all())
    assert torch.equal(W, W1)


def test_sharded_step_with_update_exchange_on_one_rank(cuda_lib):
    """sharding.ShardedStep with the library's steps and the bf16 update exchange,
    one rank (no collective): two shape groups, two steps; states bit for bit those
    of the fused step, weights within eta times bf16's rounding of O per step."""
    from bit_muon_optimizer_b200 import sharding as S
    gm = cuda_lib
    k, eta, wd = 8, 0.02, 0.1
    shapes = [(256, 384, 3), (384, 256, 2)]
    make = S.grasp_make_step(k, torch.device(DEV), eta=eta, wd=wd, seed=5)
    sh = S.ShardedStep(shapes, 1, 0, make, update=S.grasp_update(eta, wd))
    Ws = [WL.random_matrix((c, m, n), 40 + i, std=0.02).to(DEV) for i, (m, n, c) in enumerate(shapes)]
    ref = []
    for i, (m, n, c) in enumerate(shapes):
        base = sum(cc for _, _, cc in shapes[:i])
        ref.append((gm.GraspStep(c, m, n, k, eta=eta, wd=wd, seed=5, device=DEV,
                                 matrix_ids=range(base, base + c)),
                    gm.GraspState.zeros(c, m, n, k, DEV), Ws[i].clone()))
    for t in (1, 2):
        Gs = [_outlier(c, m, n, 50 + 10 * t + i, dtype=torch.bfloat16).to(DEV)
              for i, (m, n, c) in enumerate(shapes)]
        sh(Ws, Gs)
        for (step, st, W), G in zip(ref, Gs):
            step(st, W, G)
    torch.cuda.synchronize()
    for g, (step, st, W) in enumerate(ref):
        mine = sh.steps[g].state
        for a, b in zip(mine.tensors(), st.tensors()):
            assert torch.equal(a, b)
        assert (Ws[g] - W).abs().max().item() <= 2 * 2 * eta * 2.0 ** -9 + 1e-6


def test_sharded_owner_step_in_sub_batches_equals_one_call(cuda_lib):
    """grasp_make_step with a small sub-batch limit steps an owner batch as several
    library calls (here of 2, 2 and 1 matrices): the weights, the direction O with
    its flags, the peer stores and the state are bit for bit those of the one-call
    step, and the batch state carries the step count and a sub-batch's status."""
    from bit_muon_optimizer_b200 import sharding as S
    gm = cuda_lib
    k, B, m, n = 8, 5, 256, 384
    ids = [3, 4, 5, 6, 7]
    one = S.grasp_make_step(k, torch.device(DEV), eta=0.02, wd=0.1, seed=5)(m, n, ids)
    split = S.grasp_make_step(k, torch.device(DEV), sub_batch_elements=2 * m * n, eta=0.02, wd=0.1,
                              seed=5)(m, n, ids)
    W1 = WL.random_matrix((B, m, n), 31, std=0.02).to(DEV)
    W2 = W1.clone()
    for t in (1, 2):
        G = _outlier(B, m, n, 60 + t, dtype=torch.bfloat16).to(DEV)
        one(W1, G)
        split(W2, G)
    torch.cuda.synchronize()
    assert torch.equal(W1, W2)
    for a, b in zip(one.state.tensors(), split.state.tensors()):
        assert torch.equal(a, b)
    assert int(split.state.step.item()) == 2
    G = _outlier(B, m, n, 63, dtype=torch.bfloat16).to(DEV)
    O1, f1 = one.direction(G)
    O2, f2 = split.direction(G)
    torch.cuda.synchronize()
    assert torch.equal(O1, O2) and torch.equal(f1, f2) and not f2.any()
    dst = torch.tensor([9, 1, 6, 0, 4], dtype=torch.int64, device=DEV)
    bufs = [torch.zeros((10, m, n), dtype=torch.bfloat16, device=DEV) for _ in range(2)]
    flags = [torch.full((10,), -1, dtype=torch.int32, device=DEV) for _ in range(2)]
    G = _outlier(B, m, n, 64, dtype=torch.bfloat16).to(DEV)
    one.orth_peers(G, [bufs[0].data_ptr()], [flags[0].data_ptr()], dst)
    split.orth_peers(G, [bufs[1].data_ptr()], [flags[1].data_ptr()], dst)
    torch.cuda.synchronize()
    assert torch.equal(bufs[0], bufs[1]) and torch.equal(flags[0], flags[1])
    for a, b in zip(one.state.tensors(), split.state.tensors()):
        assert torch.equal(a, b)
    # a non-finite gradient in the second sub-batch: the batch status says so, and
    # the direction's flags mark that sub-batch's matrices
    G = _outlier(B, m, n, 65, dtype=torch.bfloat16).to(DEV)
    G[2, 5, 7] = float("nan")
    O2, f2 = split.direction(G)
    torch.cuda.synchronize()
    assert f2.tolist()[2:4] == [gm.GM_E_NONFINITE] * 2 and f2.tolist()[:2] == [0, 0] and f2.tolist()[4] == 0
    assert int(split.state.dev_status.item()) == gm.GM_E_NONFINITE
