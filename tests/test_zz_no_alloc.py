"""gm_newton_schulz_noalloc against gm_newton_schulz.

The no-allocation entry point is for callers that must not allocate GPU memory
at the point where they orthogonalise: code inside a framework that owns every
device allocation through its own pool, plugins that may not call the device
allocator, or paths where an allocation would synchronise the device. It runs
the same Newton-Schulz chain as gm_newton_schulz, on a scratch array built into
the library, so its output must agree with the allocating entry point within
the NS tolerance the other tests use (2e-2 relative Frobenius). Two calls in a
row, with different shapes and dtypes, also exercise the reuse of the shared
scratch array.
"""

import ctypes

import pytest
import torch

from bit_muon_optimizer_b200 import workloads as WL

pytestmark = pytest.mark.gpu


def _rel(a, b):
    a, b = a.double().cpu(), b.double().cpu()
    return float((a - b).norm() / b.norm())


def test_noalloc_matches_allocating_entry_point_twice(cuda_lib):
    gm = cuda_lib
    calls = [(2, 256, 512, torch.float32), (3, 640, 384, torch.bfloat16)]
    for i, (B, m, n, dt) in enumerate(calls):
        X = WL.random_matrix((B, m, n), 900 + i, std=1e-2).to(dt).cuda()
        ref = gm.newton_schulz(X)
        got = gm.newton_schulz_noalloc(X)
        torch.cuda.synchronize()
        assert torch.isfinite(got).all()
        assert _rel(got, ref) <= 2e-2


def test_noalloc_call_allocates_no_device_memory(cuda_lib):
    """The property the entry point exists for. One warm-up call loads the
    library's kernels (and with them the built-in scratch array) on the device;
    after it, with the input and the output preallocated, a call on a new shape
    and new dtypes leaves the device's free memory exactly where it was. Both
    shapes are multiples of 64, so the two calls launch the same kernels."""
    gm = cuda_lib
    X0 = WL.random_matrix((2, 256, 512), 910, std=1e-2).cuda()
    gm.newton_schulz_noalloc(X0, out=torch.empty_like(X0))
    X1 = WL.random_matrix((3, 384, 640), 911, std=1e-2).to(torch.bfloat16).cuda()
    out = torch.empty((3, 384, 640), dtype=torch.float16, device="cuda")
    ref = gm.newton_schulz(X1)
    torch.cuda.synchronize()
    free_before, _ = torch.cuda.mem_get_info()
    gm.newton_schulz_noalloc(X1, out=out)
    torch.cuda.synchronize()
    free_after, _ = torch.cuda.mem_get_info()
    assert free_after == free_before
    assert _rel(out, ref) <= 2e-2


def test_noalloc_rejects_shapes_beyond_its_scratch(cuda_lib):
    gm = cuda_lib
    B, m, n = 64, 1024, 1024          # needs far more than the built-in 64 MiB
    assert gm.workspace_bytes(gm.GM_OP_NEWTON_SCHULZ, B, m, n) > gm.NOALLOC_SCRATCH_BYTES
    r = gm.lib.gm_newton_schulz_noalloc(B, m, n, ctypes.c_void_p(256), gm.GM_F32, None, 5,
                                        ctypes.c_float(1e-7), ctypes.c_void_p(256), gm.GM_F32, None)
    assert r == gm.GM_E_WORKSPACE
    assert b"built-in scratch" in gm.lib.gm_last_error()
