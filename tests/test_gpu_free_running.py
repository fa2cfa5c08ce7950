"""Free-running drift: the CUDA step and the fp64 oracle each run from the same zero
state over a workload's steps, each on its own state, with the same gradients.
The drift of the accumulated update W_T - W_0 is reported (printed), not gated:
the pages fix no bound for it, and the codes may round differently wherever the
two sides' fp32 inputs differ. Only a blow-up (non-finite or a drift of the order
of the update itself) fails.
"""

import pytest
import torch

import oracle as O
from bit_muon_optimizer_b200 import workloads as WL

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.mark.parametrize("cid,gi,count,steps", [(1, 0, 1, 3), (2, 2, 1, 10)])
def test_free_running_drift(cuda_lib, cid, gi, count, steps):
    gm = cuda_lib
    w = WL.WORKLOADS[cid]
    g = w.groups[gi]
    m, n, k = g.m, g.n, w.k
    base = w.group_base(gi)
    step = gm.GraspStep(count, m, n, k, mu=w.mu, eta=w.eta, wd=w.wd, T=w.T, seed=w.seed, device=DEV)
    st = gm.GraspState.zeros(count, m, n, k, DEV)
    W0 = torch.stack([WL.initial_weight(w, base + b, m, n) for b in range(count)])
    W = W0.clone().to(DEV)
    ost = [O.zero_state(m, n, k) for _ in range(count)]
    Wo = [W0[b].double() for b in range(count)]
    for t in range(1, steps + 1):
        G = torch.stack([WL.gradient(w, base + b, t, m, n) for b in range(count)])
        step(st, W, G.to(DEV))
        for b in range(count):
            r = O.grasp_step(ost[b], Wo[b], G[b], mu=w.mu, eta=w.eta, wd=w.wd, seed=w.seed, b=b, T=w.T)
            ost[b], Wo[b] = r.state, r.W
    torch.cuda.synchronize()
    assert int(st.dev_status.item()) == 0
    for b in range(count):
        du_gpu = W[b].double().cpu() - W0[b].double()
        du_ref = Wo[b] - W0[b].double()
        drift = float((du_gpu - du_ref).norm() / du_ref.norm())
        print(f"\n[{w.name} {m}x{n} b={b}, {steps} steps] free-running drift of W_T - W_0: {drift:.3e}")
        assert drift == drift and drift < 0.5
