"""The product's boundary rules, checked on the host.

* The Python binding is argument marshalling over libgmuon: importing it
  without the built library fails loudly (no silent fallback of any kind).
* The oracle is test infrastructure: nothing in the package imports it, and
  bench.py imports it only inside the two functions that time it (the GPU
  arm's CPU baseline and the reference arm).
* The oracle is independent of the CUDA path: it imports nothing from the
  package or the bench, and no CUDA or C source includes anything of it.
"""

import ast
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "bit_muon_optimizer_b200")
ORACLE = os.path.join(ROOT, "oracle")


def _py_files(top):
    for dirpath, _, files in os.walk(top):
        for f in files:
            if f.endswith(".py"):
                yield os.path.join(dirpath, f)


def _top_imports(node):
    """Top-level package names imported anywhere under an AST node."""
    names = set()
    for n in ast.walk(node):
        if isinstance(n, ast.Import):
            names |= {a.name.split(".")[0] for a in n.names}
        elif isinstance(n, ast.ImportFrom) and n.level == 0 and n.module:
            names.add(n.module.split(".")[0])
    return names


def _parse(path):
    with open(path) as f:
        return ast.parse(f.read(), path)


def test_binding_import_fails_loudly_without_the_library():
    code = ("import os\n"
            "real = os.path.exists\n"
            "os.path.exists = lambda p: False if str(p).endswith('libgmuon.so') else real(p)\n"
            "import bit_muon_optimizer_b200.gmuon\n")
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode != 0
    assert "ImportError" in r.stderr and "libgmuon.so is missing" in r.stderr


def test_package_never_imports_the_oracle():
    for path in _py_files(PKG):
        assert "oracle" not in _top_imports(_parse(path)), path


def test_bench_imports_the_oracle_only_where_it_is_timed():
    tree = _parse(os.path.join(ROOT, "bench.py"))
    module_level = set()
    for n in tree.body:
        if isinstance(n, (ast.Import, ast.ImportFrom)):
            module_level |= _top_imports(n)
    assert "oracle" not in module_level
    users = {f.name for f in ast.walk(tree)
             if isinstance(f, ast.FunctionDef) and "oracle" in _top_imports(f)}
    assert users == {"oracle_sample_seconds", "run_reference"}


def test_oracle_is_independent_of_the_cuda_path():
    for path in _py_files(ORACLE):
        imps = _top_imports(_parse(path))
        assert not imps & {"bit_muon_optimizer_b200", "bench", "__graft_entry__", "ctypes"}, path
    for dirpath, _, files in os.walk(PKG):
        for f in files:
            if f.endswith((".cu", ".cuh", ".h", ".c", ".cpp")):
                with open(os.path.join(dirpath, f)) as fh:
                    for line in fh:
                        if line.lstrip().startswith("#include"):
                            assert "oracle" not in line, (f, line)


def test_step_binding_checks_tensors_before_passing_pointers():
    """GraspStep hands W, G and the state to the library as raw pointers, so
    the binding checks their shapes, dtypes, device and layout first; every
    call here is rejected in Python, before the library is reached."""
    import pytest
    import torch

    from bit_muon_optimizer_b200 import gmuon as gm
    B, m, n, k = 2, 64, 96, 8
    step = gm.GraspStep(B, m, n, k, ws=torch.empty(0, dtype=torch.uint8))
    st = gm.GraspState.zeros(B, m, n, k, device="cpu")
    W = torch.zeros(B, m, n)
    G = torch.zeros(B, m, n, dtype=torch.bfloat16)
    bad = [
        (st, torch.zeros(B, m, n + 16), G, "W: expected shape"),
        (st, W, torch.zeros(B, m, n, dtype=torch.float64), "G: dtype"),
        (st, W.double(), G, "W: dtype"),
        (gm.GraspState.zeros(B, m, n, k + 1, device="cpu"), W, G, "P8: expected shape"),
        (gm.GraspState.zeros(B + 1, m, n, k, device="cpu"), W, G, "codes4: expected shape"),
        (st, W, G, "expected a CUDA tensor"),               # right layout, host memory
    ]
    for state, w_, g_, msg in bad:
        with pytest.raises(ValueError, match=msg):
            step(state, w_, g_)
    # a batch of one also takes plain [m, n] matrices
    one = gm.GraspStep(1, m, n, k, ws=torch.empty(0, dtype=torch.uint8))
    with pytest.raises(ValueError, match="expected a CUDA tensor"):
        one(gm.GraspState.zeros(1, m, n, k, device="cpu"), torch.zeros(m, n), torch.zeros(m, n))


def test_entry_point_bindings_check_tensors_before_passing_pointers():
    import pytest
    import torch

    from bit_muon_optimizer_b200 import gmuon as gm
    B, m, n, k = 2, 64, 256, 8
    f = lambda *s: torch.zeros(*s)                                   # noqa: E731
    st = gm.GraspState.zeros(B, m, n, k, device="cpu")
    parts = [st.codes4, st.rscale, st.cscale, st.P8, st.Pscale, st.R8, st.Rscale]
    cases = [
        (lambda: gm.dequant_rebuild(st.codes4, f(B, m, 1), *parts[2:]), "rscale: expected shape"),
        (lambda: gm.dequant_rebuild(*parts[:5], st.R8[:, :-16], st.Rscale), "R8: expected shape"),
        (lambda: gm.dequant_rebuild(*parts, out=f(B, m, n - 16)), "out: expected shape"),
        (lambda: gm.momentum_powerit(f(B, m, n), k, M_prev=f(B, m, n + 16)), "M_prev: expected"),
        (lambda: gm.momentum_powerit(f(B, m, n), k, R_prev=f(B, n, k + 1)), "R_prev: expected"),
        (lambda: gm.momentum_powerit(f(B, m, n).double(), k), "G: dtype"),
        (lambda: gm.grid_quant4(f(B, m, n), f(B, m, k)), "both be given"),
        (lambda: gm.grid_quant4(f(B, m, n), f(B, m, k), f(B, n + 16, k)), "R: expected shape"),
        (lambda: gm.grid_quant4(f(B, m, n).half()), "X: dtype"),
        (lambda: gm.quant8(f(B, m, k).double()), "X: dtype"),
        (lambda: gm.newton_schulz(f(B, m, n), out=f(B, n, m)), "out: expected shape"),
        (lambda: gm.newton_schulz(f(B, m, n), ws=torch.empty(16, dtype=torch.uint8)), "ws: 16 bytes"),
        (lambda: gm.gram_ns(f(B, m, n).double()), "X: dtype"),
        (lambda: gm.newton_schulz_noalloc(f(B, m, n), out=f(B, m, n).double()), "out: dtype"),
        (lambda: gm.group_quant4(f(B, m, n).double()), "X: dtype"),
        (lambda: gm.group_dequant4(st.codes4, f(B, m * n // 64)), "gscale: expected shape"),
        (lambda: gm.group_dequant4(st.codes4, f(B, m * n // 128), out=f(B, m, n).half()),
         "out: dtype"),
        # right shapes and dtypes, host memory: stopped before the library call
        (lambda: gm.group_quant4(f(B, m, n)), "expected a CUDA tensor"),
        (lambda: gm.dequant_rebuild(*parts), "expected a CUDA tensor"),
        (lambda: gm.grid_quant4(f(B, m, n), f(B, m, k), f(B, n, k)), "expected a CUDA tensor"),
        (lambda: gm.quant8(f(B, m, k)), "expected a CUDA tensor"),
    ]
    for call, msg in cases:
        with pytest.raises(ValueError, match=msg):
            call()


def test_offload_chunk_bounds():
    """offload.chunk_bounds covers 0 .. B-1 in order with runs of at most `chunk`."""
    from bit_muon_optimizer_b200.offload import chunk_bounds
    assert chunk_bounds(5, 2) == [(0, 2), (2, 4), (4, 5)]
    assert chunk_bounds(4, 4) == [(0, 4)]
    assert chunk_bounds(1, 8) == [(0, 1)]
    for B in range(1, 20):
        for c in range(1, 7):
            bounds = chunk_bounds(B, c)
            assert bounds[0][0] == 0 and bounds[-1][1] == B
            assert all(b1 == a2 for (_, b1), (a2, _) in zip(bounds, bounds[1:]))
            assert all(0 < b - a <= c for a, b in bounds)
    with pytest.raises(ValueError):
        chunk_bounds(0, 2)
    from bit_muon_optimizer_b200.offload import default_chunk
    assert default_chunk(56, 18944, 3584) == 1 and default_chunk(56, 3584, 3584) == 3
    assert default_chunk(48, 768, 768) == 6 and default_chunk(1, 256, 512) == 1


def test_offload_sub_batch_size():
    """offload.sub_batch_size: the fewest calls of at most `limit` elements (one
    matrix per call at least), as equal as the count allows."""
    from bit_muon_optimizer_b200.offload import sub_batch_size
    assert sub_batch_size(56, 18944, 3584) == 14 and sub_batch_size(56, 3584, 3584) == 56
    assert sub_batch_size(5, 256, 384, limit=2 * 256 * 384) == 2
    assert sub_batch_size(3, 100, 100, limit=1) == 1
    for B in range(1, 40):
        for limit in (1, 3, 7, 10, 64):
            c = sub_batch_size(B, 1, 1, limit=limit)
            calls = -(-B // c)
            assert c <= max(1, limit) and calls == -(-B // limit) or (limit >= B and c == B)
    with pytest.raises(ValueError):
        sub_batch_size(0, 16, 16)
