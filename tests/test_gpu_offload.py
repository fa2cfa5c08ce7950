"""offload.HostStreamedStep against the resident step: a batch whose gradients
(and weights, or weights kept on the device) live in pinned host memory,
stepped in chunks on three streams, ends with the weights and the quantized
state of one gm_grasp_step call over the whole batch on the device, bit for bit
(every matrix's step is independent of its batch), for both NS forms and a
ragged shape; two batches sharing their streams, the first call not waited for,
end the same way."""

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
    assert not hs.status_host.any()


@pytest.mark.parametrize("ns", ["standard", "gram"])
def test_host_gradients_with_weights_on_the_device(cuda_lib, ns):
    from bit_muon_optimizer_b200.offload import HostStreamedStep
    gm = cuda_lib
    k = 8
    mode = gm.GM_NS_GRAM if ns == "gram" else gm.GM_NS_STANDARD
    shapes = [(5, 256, 384, 2), (3, 272, 144, 1)]
    streams = tuple(torch.cuda.Stream() for _ in range(3))
    runs = []
    for j, (B, m, n, chunk) in enumerate(shapes):
        ids = [7 * j + b for b in range(B)]
        W0 = WL.random_matrix((B, m, n), 71 + j, std=0.02)
        grads = [WL.random_matrix((B, m, n), 80 + 10 * j + t, std=1e-3).to(torch.bfloat16).pin_memory()
                 for t in (1, 2, 3)]
        hs = HostStreamedStep(B, m, n, k, chunk=chunk, device=DEV, matrix_ids=ids, ns=mode, seed=4,
                              streams=streams)
        ref = gm.GraspStep(B, m, n, k, ns=mode, seed=4, device=DEV, matrix_ids=ids)
        runs.append(dict(hs=hs, W=W0.to(DEV), grads=grads, ref=ref, Wr=W0.to(DEV),
                         st=gm.GraspState.zeros(B, m, n, k, DEV)))
    assert runs[0]["hs"].h2d_bytes(True) == 5 * 256 * 384 * 2
    assert runs[0]["hs"].d2h_bytes(True) == 4 * 3
    for t in range(3):
        for j, r in enumerate(runs):
            r["hs"](r["W"], r["grads"][t], wait=j == len(runs) - 1)
    torch.cuda.synchronize()
    for r in runs:
        r["ref"](r["st"], r["Wr"], r["grads"][0].to(DEV))
        r["ref"](r["st"], r["Wr"], r["grads"][1].to(DEV))
        r["ref"](r["st"], r["Wr"], r["grads"][2].to(DEV))
    torch.cuda.synchronize()
    for r in runs:
        hs = r["hs"]
        assert hs.status() == 0 and not hs.status_host.any()
        assert torch.equal(r["W"], r["Wr"])
        for a, b in zip(hs.state.tensors()[:7], r["st"].tensors()[:7]):
            assert torch.equal(a, b)
        assert hs.Wbuf is None


def test_host_streamed_step_rejects_device_or_unpinned_buffers(cuda_lib):
    from bit_muon_optimizer_b200.offload import HostStreamedStep
    hs = HostStreamedStep(2, 128, 128, 4, device=DEV)
    W = torch.zeros((2, 128, 128))
    G = torch.zeros((2, 128, 128), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="pinned"):
        hs(W, G.pin_memory())
    with pytest.raises(ValueError, match="pinned"):
        hs(W.pin_memory(), G.to(DEV))
