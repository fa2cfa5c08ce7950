"""The failure path of the bounded device waits, without a GPU fault.

Every mbarrier wait of the NS product kernel gives up after a time limit,
records GM_E_TIMEOUT in the device's error word and lets every role of the
kernel leave its loop; the tensor memory is released on the way out. The test
hook gm_test_wait_timeout launches that kernel on one tile with its operand
copies withheld (a barrier that nothing completes) and a 20 ms limit. The host
must then read GM_E_TIMEOUT from gm_device_errors(), the word must be cleared
by that read, and the device must stay usable: a normal Newton-Schulz call
right after it matches the oracle.
"""

import time

import pytest
import torch

import oracle as O
from bit_muon_optimizer_b200 import workloads as WL

pytestmark = pytest.mark.gpu


def test_bounded_wait_runs_out_and_the_device_stays_usable(cuda_lib):
    gm = cuda_lib
    gm.device_errors()                      # start from a clear error word
    t0 = time.perf_counter()
    bufs = gm.wait_timeout_probe(20_000_000)
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    with pytest.raises(gm.GmuonError) as e:
        gm.device_errors()
    assert e.value.status == gm.GM_E_TIMEOUT
    assert elapsed < 5.0                    # the waits ended on their limit, not a hang
    gm.device_errors()                      # read once: cleared
    del bufs
    X = WL.random_matrix((2, 256, 512), 5, std=1e-2)
    Og = gm.newton_schulz(X.cuda())
    torch.cuda.synchronize()
    gm.device_errors()
    for b in range(2):
        ref = O.ns_standard(X[b].double())
        assert float((Og[b].double().cpu() - ref).norm() / ref.norm()) <= 2e-2
