"""The C-ABI library loads, exports every symbol include/gmuon.h declares, and
its host-only logic works without a GPU (no compute call is made here)."""

import ctypes
import re

import pytest

from bit_muon_optimizer_b200 import flops as F
from bit_muon_optimizer_b200 import gmuon as gm


def _declared_functions():
    src = open(gm.HEADER_PATH).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(gm_[a-z0-9_]+)\s*\(", src)))


def test_every_declared_symbol_is_exported():
    names = _declared_functions()
    assert len(names) >= 14
    for name in names:
        assert hasattr(gm.lib, name), name


def test_version_and_status_strings():
    assert gm.lib.gm_version() == 1
    assert gm.lib.gm_status_string(gm.GM_E_NONFINITE) == b"GM_E_NONFINITE"
    assert gm.lib.gm_status_string(0) == b"GM_OK"


def test_workspace_sizes_are_host_only_and_consistent():
    b1 = gm.workspace_bytes(gm.GM_OP_GRASP_STEP, 1, 256, 512, 8, gm.GM_NS_STANDARD)
    b2 = gm.workspace_bytes(gm.GM_OP_GRASP_STEP, 2, 256, 512, 8, gm.GM_NS_STANDARD)
    bg = gm.workspace_bytes(gm.GM_OP_GRASP_STEP, 1, 256, 512, 8, gm.GM_NS_GRAM)
    assert 0 < b1 < b2 and bg > b1
    assert gm.workspace_bytes(gm.GM_OP_GRASP_STEP, 1, 250, 512, 8, 0) == 0    # m % 16 != 0
    assert gm.workspace_bytes(gm.GM_OP_GRASP_STEP, 1, 256, 512, 33, 0) == 0   # k > 32
    lay = gm.GraspWsLayout()
    assert gm.lib.gm_grasp_workspace_layout(1, 256, 512, 8, 0, ctypes.byref(lay)) == 0
    assert lay.total == b1
    offs = [lay.M, lay.Q, lay.P, lay.R, lay.X, lay.scale]
    assert all(o % 256 == 0 for o in offs) and len(set(offs)) == len(offs)
    assert lay.M + 256 * 512 * 4 <= lay.Q


@pytest.mark.parametrize("m,n", [(256, 512), (768, 2048), (2048, 768), (4096, 16384)])
def test_library_ns_schedule_matches_flop_counter(m, n):
    f, cnt = gm.ns_flops(gm.GM_NS_STANDARD, m, n, 5)
    assert f == F.ns_standard_flops(m, n, 5) and cnt == 15
    for restart in [(), (2,), (1, 3)]:
        f, cnt = gm.ns_flops(gm.GM_NS_GRAM, m, n, 5, restart)
        assert f == F.gram_ns_flops(m, n, 5, restart)
        assert cnt == F.gram_ns_gemm_count(5, restart)


def test_argument_errors_are_reported_before_any_launch():
    st = gm.GraspStateC()
    prm = gm.GraspParams(0.95, 0.02, 0.0, 8, 5, 0, None, None, 0, 1e-7, 0)
    # NULL state pointers
    r = gm.lib.gm_grasp_step(1, 256, 512, ctypes.byref(prm), ctypes.byref(st), None, None, 0,
                             None, 0, None)
    assert r == gm.GM_E_ARG
    assert b"NULL" in gm.lib.gm_last_error()
    # bad shape
    r = gm.lib.gm_grid_quant4(1, 250, 512, 128, 0, ctypes.c_void_p(256), None, None, ctypes.c_void_p(256),
                              ctypes.c_void_p(256), ctypes.c_void_p(256), None)
    assert r == gm.GM_E_ARG
    # k out of range
    r = gm.lib.gm_quant8(1, 100, 33, ctypes.c_void_p(256), ctypes.c_void_p(256),
                         ctypes.c_void_p(256), None)
    assert r == gm.GM_E_ARG
    # workspace too small
    prm2 = gm.GraspParams(0.95, 0.02, 0.0, 8, 5, 0, None, None, 0, 1e-7, 0)
    p = ctypes.c_void_p(256)
    st2 = gm.GraspStateC(256, 256, 256, 256, 256, 256, 256, 256, 256)
    r = gm.lib.gm_grasp_step(1, 256, 512, ctypes.byref(prm2), ctypes.byref(st2), p, p, 0, p, 16, None)
    assert r == gm.GM_E_WORKSPACE


def test_misaligned_arrays_are_rejected_before_any_launch():
    """Every device array must be 16-byte aligned (the kernels move 16-byte vectors)."""
    ok, bad = ctypes.c_void_p(4096), ctypes.c_void_p(4096 + 8)
    r = gm.lib.gm_grid_quant4(1, 256, 512, 128, 0, bad, None, None, ok, ok, ok, None)
    assert r == gm.GM_E_ARG and b"aligned" in gm.lib.gm_last_error()
    prm = gm.GraspParams(0.95, 0.02, 0.0, 8, 5, 0, None, None, 0, 1e-7, 0)
    st = gm.GraspStateC(4096, 4096, 4096, 4096, 4096, 4096, 4096 + 4, 4096, 4096)   # Rscale off by 4
    r = gm.lib.gm_grasp_step(1, 256, 512, ctypes.byref(prm), ctypes.byref(st), ok, ok, 1, ok, 1 << 30, None)
    assert r == gm.GM_E_ARG and b"aligned" in gm.lib.gm_last_error()
    r = gm.lib.gm_newton_schulz(1, 256, 512, bad, 1, None, 5, 1e-7, ok, 0, ok, 1 << 30, None)
    assert r == gm.GM_E_ARG
    r = gm.lib.gm_quant8(1, 777, 3, ok, bad, ok, None)
    assert r == gm.GM_E_ARG and b"aligned" in gm.lib.gm_last_error()


@pytest.mark.parametrize("B,m,n", [(0, 256, 512), (65536, 256, 512), (1, 0, 512), (1, 256, 0),
                                   (1, 8, 512), (1, 256, 65552), (1, 250, 512)])
def test_empty_and_out_of_range_shapes_are_argument_errors(B, m, n):
    """An empty batch or matrix is GM_E_ARG (not a silent no-op), as are sizes
    outside 16 <= m, n <= 65536 (multiples of 16) and 1 <= B <= 65535; all
    are caught on the host before any launch (this runs without a GPU)."""
    ok = ctypes.c_void_p(4096)
    prm = gm.GraspParams(0.95, 0.02, 0.0, 8, 5, 0, None, None, 0, 1e-7, 0)
    st = gm.GraspStateC(*([4096] * 9))
    calls = [
        lambda: gm.lib.gm_grasp_step(B, m, n, ctypes.byref(prm), ctypes.byref(st), ok, ok, 1, ok,
                                     1 << 40, None),
        lambda: gm.lib.gm_newton_schulz(B, m, n, ok, 1, None, 5, 1e-7, ok, 0, ok, 1 << 40, None),
        lambda: gm.lib.gm_grid_quant4(B, m, n, 128, 0, ok, None, None, ok, ok, ok, None),
        lambda: gm.lib.gm_dequant_rebuild(B, m, n, 0, ok, ok, ok, None, None, None, None, ok, None),
    ]
    for call in calls:
        assert call() == gm.GM_E_ARG
        assert b"shape" in gm.lib.gm_last_error()
    assert gm.workspace_bytes(gm.GM_OP_GRASP_STEP, B, m, n, 8) == 0


def test_quant8_row_range():
    ok = ctypes.c_void_p(4096)
    for B, rows in [(0, 16), (1, 0), (1, (1 << 20) + 1)]:
        assert gm.lib.gm_quant8(B, rows, 8, ok, ok, ok, None) == gm.GM_E_ARG


def test_group_codec_argument_errors():
    """The 4bit-Muon-base entry points reject bad shapes, NULL and misaligned
    arrays on the host, before any launch (this runs without a GPU)."""
    ok, bad = ctypes.c_void_p(4096), ctypes.c_void_p(4096 + 8)
    for B, m, n in [(0, 256, 512), (1, 250, 512), (1, 256, 8)]:
        assert gm.lib.gm_group_quant4(B, m, n, ok, ok, ok, None) == gm.GM_E_ARG
        assert gm.lib.gm_group_dequant4(B, m, n, ok, ok, ok, None) == gm.GM_E_ARG
    assert gm.lib.gm_group_quant4(1, 256, 512, None, ok, ok, None) == gm.GM_E_ARG
    assert gm.lib.gm_group_quant4(1, 256, 512, bad, ok, ok, None) == gm.GM_E_ARG
    assert b"aligned" in gm.lib.gm_last_error()
    assert gm.lib.gm_group_dequant4(1, 256, 512, ok, bad, ok, None) == gm.GM_E_ARG


def test_every_cuda_source_is_built():
    """The in-tree build compiles every .cu file of the package's csrc/ into
    libgmuon.so (a kernel file left out would only fail at link or call time)."""
    import os

    from bit_muon_optimizer_b200 import build as Bd
    on_disk = sorted(f for f in os.listdir(Bd.CSRC) if f.endswith(".cu"))
    assert sorted(Bd.SOURCES) == on_disk
    headers = sorted(f for f in os.listdir(Bd.CSRC) if f.endswith((".cuh", ".h")))
    assert sorted(Bd.HEADERS) == headers


def test_new_entry_points_argument_errors():
    """The step halves, the step's option fields, the mu-law codec, the Gram NS
    trace and the timeout hook reject bad arguments on the host, before any
    launch (this runs without a GPU)."""
    ok, bad = ctypes.c_void_p(4096), ctypes.c_void_p(4096 + 8)
    st = gm.GraspStateC(*([4096] * 9))

    def prm(**kw):
        p = gm.GraspParams(0.95, 0.02, 0.0, 8, 5, 0, None, None, 0, 1e-7, 0)
        for k, v in kw.items():
            setattr(p, k, v)
        return p

    big = 1 << 40
    for p in (prm(power_steps=4), prm(power_steps=-1), prm(residual_from_codes=2),
              prm(matrix_ids=4096 + 8)):
        assert gm.lib.gm_grasp_step(1, 256, 512, ctypes.byref(p), ctypes.byref(st), ok, ok, 1, ok,
                                    big, None) == gm.GM_E_ARG
        assert gm.lib.gm_grasp_state_update(1, 256, 512, ctypes.byref(p), ctypes.byref(st), ok, 1,
                                            ok, big, None) == gm.GM_E_ARG
    p = prm()
    assert gm.lib.gm_grasp_state_update(1, 256, 512, ctypes.byref(p), ctypes.byref(st), None, 1,
                                        ok, big, None) == gm.GM_E_ARG
    assert gm.lib.gm_grasp_apply(1, 256, 512, ctypes.byref(p), ctypes.byref(st), None, ok, big,
                                 None) == gm.GM_E_ARG
    assert gm.lib.gm_grasp_apply(1, 256, 512, ctypes.byref(p), ctypes.byref(st), ok, ok, 16,
                                 None) == gm.GM_E_WORKSPACE
    # mu-law codec: mu must be positive, shapes and alignment as the group codec
    assert gm.lib.gm_mulaw_quant4(1, 256, 512, 0.0, ok, ok, ok, None) == gm.GM_E_ARG
    assert gm.lib.gm_mulaw_quant4(1, 256, 512, -1.0, ok, ok, ok, None) == gm.GM_E_ARG
    assert gm.lib.gm_mulaw_quant4(1, 250, 512, 255.0, ok, ok, ok, None) == gm.GM_E_ARG
    assert gm.lib.gm_mulaw_dequant4(1, 256, 512, 255.0, ok, bad, ok, None) == gm.GM_E_ARG
    # Gram NS trace: both trace buffers required
    assert gm.lib.gm_gram_ns_trace(1, 256, 512, ok, 1, None, 5, None, 0, 1e-7, ok, 0, None, ok,
                                   ok, big, None) == gm.GM_E_ARG
    # timeout hook: the limit stays within [1 ms, 1 s]
    assert gm.lib.gm_test_wait_timeout(ok, ok, 10, None) == gm.GM_E_ARG
    assert gm.lib.gm_test_wait_timeout(ok, ok, 5_000_000_000, None) == gm.GM_E_ARG
    assert gm.lib.gm_test_wait_timeout(None, ok, 20_000_000, None) == gm.GM_E_ARG


def test_grid_block_other_than_128_is_an_argument_error():
    """The grid block side is an argument of gm_grid_quant4 and a field of the step's
    parameters; 128 (or 0 in the parameters, the default) is the only size built."""
    ok = ctypes.c_void_p(4096)
    for block in (64, 256, 0):
        r = gm.lib.gm_grid_quant4(1, 256, 512, block, 0, ok, None, None, ok, ok, ok, None)
        assert r == gm.GM_E_ARG and b"block" in gm.lib.gm_last_error()
    st = gm.GraspStateC(*([4096] * 9))
    prm = gm.GraspParams(0.95, 0.02, 0.0, 8, 5, 0, None, None, 0, 1e-7, 0)
    prm.block = 64
    r = gm.lib.gm_grasp_step(1, 256, 512, ctypes.byref(prm), ctypes.byref(st), ok, ok, 1, ok, 1 << 40, None)
    assert r == gm.GM_E_ARG and b"block" in gm.lib.gm_last_error()


def test_orth_and_weight_update_argument_errors():
    """gm_grasp_orth and gm_weight_update reject bad arguments on the host."""
    ok, bad = ctypes.c_void_p(4096), ctypes.c_void_p(4096 + 8)
    st = gm.GraspStateC(*([4096] * 9))
    prm = gm.GraspParams(0.95, 0.02, 0.0, 8, 5, 0, None, None, 0, 1e-7, 0)
    orth = lambda O, odt, ws_bytes=1 << 40: gm.lib.gm_grasp_orth(  # noqa: E731
        2, 256, 512, ctypes.byref(prm), ctypes.byref(st), O, odt, ok, ws_bytes, None)
    assert orth(None, gm.GM_BF16) == gm.GM_E_ARG
    assert orth(ok, 7) == gm.GM_E_ARG and b"odt" in gm.lib.gm_last_error()
    assert orth(bad, gm.GM_BF16) == gm.GM_E_ARG and b"aligned" in gm.lib.gm_last_error()
    assert orth(ok, gm.GM_BF16, 16) == gm.GM_E_WORKSPACE
    upd = gm.lib.gm_weight_update
    assert upd(2, 250, 512, 0.02, 0.0, ok, gm.GM_BF16, ok, None, 0, None) == gm.GM_E_ARG
    assert upd(2, 256, 512, 0.02, 0.0, None, gm.GM_BF16, ok, None, 0, None) == gm.GM_E_ARG
    assert upd(2, 256, 512, 0.02, 0.0, ok, 9, ok, None, 0, None) == gm.GM_E_ARG
    assert upd(2, 256, 512, 0.02, 0.0, ok, gm.GM_BF16, bad, None, 0, None) == gm.GM_E_ARG
    assert upd(2, 256, 512, 0.02, 0.0, ok, gm.GM_BF16, ok, ok, 2, None) == gm.GM_E_ARG
    assert upd(2, 256, 512, float("nan"), 0.0, ok, gm.GM_BF16, ok, None, 0, None) == gm.GM_E_ARG


def test_orth_peers_and_ipc_argument_errors():
    """gm_grasp_orth_peers and the IPC helpers reject bad arguments on the host."""
    ok = ctypes.c_void_p(4096)
    st = gm.GraspStateC(*([4096] * 9))
    prm = gm.GraspParams(0.95, 0.02, 0.0, 8, 5, 0, None, None, 0, 1e-7, 0)
    arr = lambda *v: (ctypes.c_void_p * len(v))(*[ctypes.c_void_p(x) for x in v])  # noqa: E731
    call = lambda po, pf, npeers, odt=gm.GM_BF16, dst=ok: gm.lib.gm_grasp_orth_peers(  # noqa: E731
        2, 256, 512, ctypes.byref(prm), ctypes.byref(st), po, pf, npeers, dst, odt, ok, 1 << 40, None)
    assert call(arr(4096), arr(4096), 0) == gm.GM_E_ARG                         # no destination
    assert call(arr(*[4096] * 9), arr(*[4096] * 9), 9) == gm.GM_E_ARG           # more than 8
    assert call(arr(4096, 0), arr(4096, 4096), 2) == gm.GM_E_ARG                # a NULL buffer
    assert call(arr(4096 + 8), arr(4096), 1) == gm.GM_E_ARG                     # misaligned
    assert call(arr(4096), arr(4096), 1, odt=5) == gm.GM_E_ARG
    assert call(arr(4096), arr(4096), 1, dst=ctypes.c_void_p(4096 + 4)) == gm.GM_E_ARG
    h = gm.IpcHandle()
    off = ctypes.c_size_t()
    assert gm.lib.gm_ipc_export(None, ctypes.byref(h), ctypes.byref(off)) == gm.GM_E_ARG
    assert gm.lib.gm_ipc_open(None, None) == gm.GM_E_ARG
    assert gm.lib.gm_ipc_close(None) == gm.GM_E_ARG
