"""offload.HostStreamedStep against the resident step: a batch whose weights
and gradients live in pinned host memory, stepped in chunks on three streams,
ends with the weights and the quantized state of one gm_grasp_step call over
the whole batch on the device, bit for bit (every matrix's step is independent
of its batch), for both NS forms and a ragged shape."""

import pytest
import torch

from bit_muon_optimizer_b200 import workloads as WL

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.mark.parametrize("ns,gdtype", [("standard", torch.bfloat16), ("gram", torch.bfloat16),
                                       ("standard", torch.float32)])
@pytest.mark.parametrize("B,m,n,chunk", [(5, 256, 384, 2), (3, 272, 144, 1), (4, 128, 256, 4)])
def test_host_streamed_step_equals_the_resident_step(cuda_lib, ns, gdtype, B, m, n, chunk):
    from bit_muon_optimizer_b200.offload import HostStreamedStep
    gm = cuda_lib
    k = 8
    mode = gm.GM_NS_GRAM if ns == "gram" else gm.GM_NS_STANDARD
    ids = [100 + 3 * b for b in range(B)]
    W0 = WL.random_matrix((B, m, n), 61, std=0.02)
    grads = [WL.random_matrix((B, m, n), 62 + t, std=1e-3).to(gdtype) for t in (1, 2, 3)]
    hs = HostStreamedStep(B, m, n, k, gdtype=gdtype, chunk=chunk, device=DEV, matrix_ids=ids,
                          ns=mode, seed=9, wd=0.1)
    Wh = W0.clone().pin_memory()
    ref = gm.GraspStep(B, m, n, k, ns=mode, seed=9, wd=0.1, device=DEV, matrix_ids=ids)
    st = gm.GraspState.zeros(B, m, n, k, DEV)
    Wd = W0.to(DEV)
    for G in grads:
        hs(Wh, G.pin_memory())
        ref(st, Wd, G.to(DEV))
    torch.cuda.synchronize()
    assert hs.status() == 0 and int(st.dev_status.item()) == 0
    assert torch.equal(Wh, Wd.cpu())
    for a, b in zip(hs.state.tensors()[:7], st.tensors()[:7]):
        assert torch.equal(a, b)
    assert all(int(s.step.item()) == 3 for s in hs.chunk_states)


def test_host_streamed_step_rejects_device_or_unpinned_buffers(cuda_lib):
    from bit_muon_optimizer_b200.offload import HostStreamedStep
    hs = HostStreamedStep(2, 128, 128, 4, device=DEV)
    W = torch.zeros((2, 128, 128))
    G = torch.zeros((2, 128, 128), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="pinned"):
        hs(W, G.pin_memory())
    with pytest.raises(ValueError, match="pinned"):
        hs(W.pin_memory(), G.to(DEV))
