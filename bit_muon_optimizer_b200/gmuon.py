"""Thin ctypes binding of libgmuon (include/gmuon.h).

Argument marshalling only: every step of the optimizer runs in the library's
CUDA kernels. Tensors are torch CUDA tensors, contiguous, batch-first
([B, rows, cols]); work is enqueued on torch's current CUDA stream. Importing
this module fails loudly when the library has not been built.
"""

from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libgmuon.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "gmuon.h")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python -m bit_muon_optimizer_b200.build`")
lib = ctypes.CDLL(LIB_PATH)

GM_OK, GM_E_ARG, GM_E_CUDA, GM_E_NONFINITE, GM_E_WORKSPACE, GM_E_UNSUPPORTED, GM_E_TIMEOUT = (
    0, -1, -2, -3, -4, -5, -6)
GM_F32, GM_BF16, GM_F16 = 0, 1, 2
GM_NS_STANDARD, GM_NS_GRAM = 0, 1
GM_OP_MOMENTUM_POWERIT, GM_OP_NEWTON_SCHULZ, GM_OP_GRAM_NS, GM_OP_GRASP_STEP = 1, 2, 3, 4
GRID_BLOCK = 128

_DT = {torch.float32: GM_F32, torch.bfloat16: GM_BF16, torch.float16: GM_F16}

c_int, c_float, c_size_t, c_uint64, vp = (ctypes.c_int, ctypes.c_float, ctypes.c_size_t,
                                          ctypes.c_uint64, ctypes.c_void_p)


class GraspParams(ctypes.Structure):
    _fields_ = [("mu", c_float), ("eta", c_float), ("wd", c_float), ("k", c_int), ("T", c_int),
                ("ns", c_int), ("abc", ctypes.POINTER(c_float)),
                ("restart_after", ctypes.POINTER(c_int)), ("n_restart", c_int),
                ("eps", c_float), ("seed", c_uint64), ("power_steps", c_int),
                ("residual_from_codes", c_int), ("matrix_ids", vp), ("block", c_int)]


class GraspStateC(ctypes.Structure):
    _fields_ = [("codes4", vp), ("rscale", vp), ("cscale", vp), ("P8", vp), ("Pscale", vp),
                ("R8", vp), ("Rscale", vp), ("step", vp), ("dev_status", vp)]


class GraspWsLayout(ctypes.Structure):
    _fields_ = [("M", c_size_t), ("Q", c_size_t), ("P", c_size_t), ("R", c_size_t),
                ("X", c_size_t), ("scale", c_size_t), ("total", c_size_t)]


def _sig(name, res, args):
    f = getattr(lib, name)
    f.restype = res
    f.argtypes = args
    return f


_sig("gm_status_string", ctypes.c_char_p, [c_int])
_sig("gm_last_error", ctypes.c_char_p, [])
_sig("gm_version", c_int, [])
_sig("gm_workspace_bytes", c_size_t, [c_int, c_int, c_int, c_int, c_int, c_int])
_sig("gm_dequant_rebuild", c_int, [c_int, c_int, c_int, c_int, vp, vp, vp, vp, vp, vp, vp, vp, vp])
_sig("gm_momentum_powerit", c_int, [c_int, c_int, c_int, c_int, c_float, vp, vp, c_int, vp,
                                    c_uint64, vp, vp, vp, vp, c_size_t, vp])
_sig("gm_grid_quant4", c_int, [c_int, c_int, c_int, c_int, c_int, vp, vp, vp, vp, vp, vp, vp])
_sig("gm_quant8", c_int, [c_int, c_int, c_int, vp, vp, vp, vp])
_sig("gm_group_quant4", c_int, [c_int, c_int, c_int, vp, vp, vp, vp])
_sig("gm_group_dequant4", c_int, [c_int, c_int, c_int, vp, vp, vp, vp])
_sig("gm_mulaw_quant4", c_int, [c_int, c_int, c_int, c_float, vp, vp, vp, vp])
_sig("gm_mulaw_dequant4", c_int, [c_int, c_int, c_int, c_float, vp, vp, vp, vp])
_sig("gm_newton_schulz", c_int, [c_int, c_int, c_int, vp, c_int, vp, c_int, c_float, vp, c_int,
                                 vp, c_size_t, vp])
_sig("gm_newton_schulz_noalloc", c_int, [c_int, c_int, c_int, vp, c_int, vp, c_int, c_float, vp,
                                         c_int, vp])
_sig("gm_gram_ns", c_int, [c_int, c_int, c_int, vp, c_int, vp, c_int, vp, c_int, c_float, vp,
                           c_int, vp, c_size_t, vp])
_sig("gm_grasp_step", c_int, [c_int, c_int, c_int, ctypes.POINTER(GraspParams),
                              ctypes.POINTER(GraspStateC), vp, vp, c_int, vp, c_size_t, vp])
_sig("gm_grasp_state_update", c_int, [c_int, c_int, c_int, ctypes.POINTER(GraspParams),
                                      ctypes.POINTER(GraspStateC), vp, c_int, vp, c_size_t, vp])
_sig("gm_grasp_apply", c_int, [c_int, c_int, c_int, ctypes.POINTER(GraspParams),
                               ctypes.POINTER(GraspStateC), vp, vp, c_size_t, vp])
_sig("gm_grasp_orth", c_int, [c_int, c_int, c_int, ctypes.POINTER(GraspParams),
                              ctypes.POINTER(GraspStateC), vp, c_int, vp, c_size_t, vp])
_sig("gm_weight_update", c_int, [c_int, c_int, c_int, c_float, c_float, vp, c_int, vp, vp, c_int, vp])
_sig("gm_grasp_orth_peers", c_int, [c_int, c_int, c_int, ctypes.POINTER(GraspParams),
                                    ctypes.POINTER(GraspStateC), ctypes.POINTER(vp),
                                    ctypes.POINTER(vp), c_int, vp, c_int, vp, c_size_t, vp])


class IpcHandle(ctypes.Structure):
    _fields_ = [("bytes", ctypes.c_ubyte * 64)]


_sig("gm_ipc_export", c_int, [vp, ctypes.POINTER(IpcHandle), ctypes.POINTER(c_size_t)])
_sig("gm_ipc_open", c_int, [ctypes.POINTER(IpcHandle), ctypes.POINTER(vp)])
_sig("gm_ipc_close", c_int, [vp])
_sig("gm_grasp_workspace_layout", c_int, [c_int, c_int, c_int, c_int, c_int,
                                          ctypes.POINTER(GraspWsLayout)])
_sig("gm_ns_flops", c_int, [c_int, c_int, c_int, c_int, vp, c_int,
                            ctypes.POINTER(ctypes.c_double), ctypes.POINTER(c_int)])
_sig("gm_device_errors", c_int, [vp])
_sig("gm_test_wait_timeout", c_int, [vp, vp, ctypes.c_int64, vp])


class GmuonError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = lib.gm_last_error().decode(errors="replace")
        super().__init__(f"{where}: {lib.gm_status_string(status).decode()} ({msg})")


def _check(status: int, where: str):
    if status != GM_OK:
        raise GmuonError(status, where)


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return ctypes.c_void_p(t.data_ptr())


def _expect(t, shape, dtypes, name):
    """Checks the shape (a [m, n] matrix also stands for a batch of one) and
    dtype of a tensor handed to the library as a raw pointer."""
    shape = tuple(shape)
    got = tuple(t.shape)
    if got != shape and not (len(shape) >= 2 and shape[0] == 1 and got == shape[1:]):
        raise ValueError(f"{name}: expected shape {shape}, got {got}")
    if t.dtype not in dtypes:
        raise ValueError(f"{name}: dtype {t.dtype} is not one of {tuple(dtypes)}")


def _ws_fits(ws, nbytes, name="ws"):
    """Checks that a caller-supplied workspace holds at least `nbytes`."""
    have = ws.numel() * ws.element_size()
    if have < nbytes:
        raise ValueError(f"{name}: {have} bytes, the call needs {nbytes}")


def _placed(tensors, names):
    """Checks that tensors are contiguous CUDA tensors."""
    for t, name in zip(tensors, names):
        if not t.is_cuda:
            raise ValueError(f"{name}: expected a CUDA tensor")
        if not t.is_contiguous():
            raise ValueError(f"{name}: expected a contiguous tensor")


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _bmn(X):
    if X.dim() == 2:
        return 1, X.shape[0], X.shape[1]
    if X.dim() != 3:
        raise ValueError("expected [B, m, n] or [m, n]")
    return X.shape[0], X.shape[1], X.shape[2]


def _floats(vals):
    if vals is None:
        return None
    arr = (c_float * len(vals))(*vals)
    return arr


def abc_table(abc, T):
    """Flatten a list of (a, b, c) triples (or None: constant quintic)."""
    if abc is None:
        return None
    flat = [float(v) for tri in abc for v in tri]
    if len(flat) != 3 * T:
        raise ValueError("abc must hold T triples")
    return _floats(flat)


_WS = {}


def workspace(nbytes: int, device=None, tag="default") -> torch.Tensor:
    """A cached 256-byte-aligned device scratch buffer of at least nbytes."""
    device = torch.device(device or torch.cuda.current_device())
    key = (tag, device)
    buf = _WS.get(key)
    if buf is None or buf.numel() < nbytes:
        buf = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)
        _WS[key] = buf
    return buf


def workspace_bytes(op, B, m, n, k=0, ns=GM_NS_STANDARD) -> int:
    return int(lib.gm_workspace_bytes(op, B, m, n, k, ns))


# ----------------------------------------------------------------- entry points

def dequant_rebuild(codes4, rscale, cscale, P8=None, Pscale=None, R8=None, Rscale=None, out=None):
    B, m, n2 = _bmn(codes4)
    n = 2 * n2
    k = 0 if P8 is None else P8.shape[-1]
    mb, nb = -(-m // GRID_BLOCK), -(-n // GRID_BLOCK)
    _expect(codes4, (B, m, n2), (torch.uint8,), "codes4")
    _expect(rscale, (B, m, nb), (torch.float32,), "rscale")
    _expect(cscale, (B, mb, n), (torch.float32,), "cscale")
    if k:
        _expect(P8, (B, m, k), (torch.int8,), "P8")
        _expect(Pscale, (B, k), (torch.float32,), "Pscale")
        _expect(R8, (B, n, k), (torch.int8,), "R8")
        _expect(Rscale, (B, k), (torch.float32,), "Rscale")
    if out is None:
        out = torch.empty((B, m, n), dtype=torch.float32, device=codes4.device)
    _expect(out, (B, m, n), (torch.float32,), "out")
    _check(lib.gm_dequant_rebuild(B, m, n, k, _ptr(codes4), _ptr(rscale), _ptr(cscale), _ptr(P8),
                                  _ptr(Pscale), _ptr(R8), _ptr(Rscale), _ptr(out), _stream()),
           "gm_dequant_rebuild")
    return out


def momentum_powerit(G, k, mu=0.95, M_prev=None, R_prev=None, seed=0):
    B, m, n = _bmn(G)
    _expect(G, (B, m, n), tuple(_DT), "G")
    if M_prev is not None:
        _expect(M_prev, (B, m, n), (torch.float32,), "M_prev")
    if R_prev is not None:
        _expect(R_prev, (B, n, k), (torch.float32,), "R_prev")
    dev = G.device
    M = torch.empty((B, m, n), dtype=torch.float32, device=dev)
    P = torch.empty((B, m, k), dtype=torch.float32, device=dev)
    R = torch.empty((B, n, k), dtype=torch.float32, device=dev)
    nb = workspace_bytes(GM_OP_MOMENTUM_POWERIT, B, m, n, k)
    ws = workspace(nb, dev)
    _check(lib.gm_momentum_powerit(B, m, n, k, mu, _ptr(M_prev), _ptr(G), _DT[G.dtype],
                                   _ptr(R_prev), seed, _ptr(M), _ptr(P), _ptr(R), _ptr(ws), nb,
                                   _stream()), "gm_momentum_powerit")
    return M, P, R


def grid_quant4(X, P=None, R=None, out=None):
    B, m, n = _bmn(X)
    dev = X.device
    k = 0 if P is None else P.shape[-1]
    _expect(X, (B, m, n), (torch.float32,), "X")
    if (P is None) != (R is None):
        raise ValueError("P and R must both be given or both be None")
    if k:
        _expect(P, (B, m, k), (torch.float32,), "P")
        _expect(R, (B, n, k), (torch.float32,), "R")
    if out is not None:
        codes, rs, cs = out
        _expect(codes, (B, m, n // 2), (torch.uint8,), "codes")
        _expect(rs, (B, m, -(-n // GRID_BLOCK)), (torch.float32,), "rscale")
        _expect(cs, (B, -(-m // GRID_BLOCK), n), (torch.float32,), "cscale")
    else:
        codes = torch.empty((B, m, n // 2), dtype=torch.uint8, device=dev)
        rs = torch.empty((B, m, -(-n // GRID_BLOCK)), dtype=torch.float32, device=dev)
        cs = torch.empty((B, -(-m // GRID_BLOCK), n), dtype=torch.float32, device=dev)
    _check(lib.gm_grid_quant4(B, m, n, GRID_BLOCK, k, _ptr(X), _ptr(P), _ptr(R), _ptr(codes), _ptr(rs),
                              _ptr(cs), _stream()), "gm_grid_quant4")
    return codes, rs, cs


def quant8(X):
    B, rows, k = _bmn(X)
    _expect(X, (B, rows, k), (torch.float32,), "X")
    codes = torch.empty((B, rows, k), dtype=torch.int8, device=X.device)
    scale = torch.empty((B, k), dtype=torch.float32, device=X.device)
    _check(lib.gm_quant8(B, rows, k, _ptr(X), _ptr(codes), _ptr(scale), _stream()), "gm_quant8")
    return codes, scale


GROUP = 128   # elements per scale of the 4bit-Muon-base codec


def group_quant4(X, out=None):
    """4bit-Muon-base codes of fp32 [B, m, n] (or [m, n]): (codes [B, m, n/2]
    uint8, scales [B, m n / 128] fp32)."""
    B, m, n = _bmn(X)
    _expect(X, (B, m, n), (torch.float32,), "X")
    if out is not None:
        codes, gs = out
    else:
        codes = torch.empty((B, m, n // 2), dtype=torch.uint8, device=X.device)
        gs = torch.empty((B, m * n // GROUP), dtype=torch.float32, device=X.device)
    _expect(codes, (B, m, n // 2), (torch.uint8,), "codes")
    _expect(gs, (B, m * n // GROUP), (torch.float32,), "gscale")
    _check(lib.gm_group_quant4(B, m, n, _ptr(X), _ptr(codes), _ptr(gs), _stream()),
           "gm_group_quant4")
    return codes, gs


def group_dequant4(codes, gscale, out=None):
    """fp32 [B, m, n] from 4bit-Muon-base codes and scales."""
    B, m, n2 = _bmn(codes)
    n = 2 * n2
    _expect(codes, (B, m, n2), (torch.uint8,), "codes")
    _expect(gscale, (B, m * n // GROUP), (torch.float32,), "gscale")
    if out is None:
        out = torch.empty((B, m, n), dtype=torch.float32, device=codes.device)
    _expect(out, (B, m, n), (torch.float32,), "out")
    _check(lib.gm_group_dequant4(B, m, n, _ptr(codes), _ptr(gscale), _ptr(out), _stream()),
           "gm_group_dequant4")
    return out


MULAW_MU = 255.0


def mulaw_quant4(X, mu=MULAW_MU, out=None):
    """MuonQ's mu-law 4-bit codes of fp32 [B, m, n] (or [m, n]), in the group
    layout of ``group_quant4``: (codes [B, m, n/2] uint8, scales [B, m n / 128])."""
    B, m, n = _bmn(X)
    _expect(X, (B, m, n), (torch.float32,), "X")
    if out is not None:
        codes, gs = out
    else:
        codes = torch.empty((B, m, n // 2), dtype=torch.uint8, device=X.device)
        gs = torch.empty((B, m * n // GROUP), dtype=torch.float32, device=X.device)
    _expect(codes, (B, m, n // 2), (torch.uint8,), "codes")
    _expect(gs, (B, m * n // GROUP), (torch.float32,), "gscale")
    _check(lib.gm_mulaw_quant4(B, m, n, float(mu), _ptr(X), _ptr(codes), _ptr(gs), _stream()),
           "gm_mulaw_quant4")
    return codes, gs


def mulaw_dequant4(codes, gscale, mu=MULAW_MU, out=None):
    """fp32 [B, m, n] from mu-law codes and group scales."""
    B, m, n2 = _bmn(codes)
    n = 2 * n2
    _expect(codes, (B, m, n2), (torch.uint8,), "codes")
    _expect(gscale, (B, m * n // GROUP), (torch.float32,), "gscale")
    if out is None:
        out = torch.empty((B, m, n), dtype=torch.float32, device=codes.device)
    _expect(out, (B, m, n), (torch.float32,), "out")
    _check(lib.gm_mulaw_dequant4(B, m, n, float(mu), _ptr(codes), _ptr(gscale), _ptr(out),
                                 _stream()), "gm_mulaw_dequant4")
    return out


def newton_schulz(X, abc=None, T=5, eps=1e-7, out_dtype=torch.float32, out=None, ws=None):
    B, m, n = _bmn(X)
    _expect(X, (B, m, n), tuple(_DT), "X")
    O = out if out is not None else torch.empty((B, m, n), dtype=out_dtype, device=X.device)
    _expect(O, (B, m, n), tuple(_DT), "out")
    out_dtype = O.dtype
    nb = workspace_bytes(GM_OP_NEWTON_SCHULZ, B, m, n)
    ws = ws if ws is not None else workspace(nb, X.device)
    _ws_fits(ws, nb)
    _check(lib.gm_newton_schulz(B, m, n, _ptr(X), _DT[X.dtype], abc_table(abc, T), T, eps,
                                _ptr(O), _DT[out_dtype], _ptr(ws), nb, _stream()),
           "gm_newton_schulz")
    return O


NOALLOC_SCRATCH_BYTES = 64 << 20


def newton_schulz_noalloc(X, abc=None, T=5, eps=1e-7, out_dtype=torch.float32, out=None):
    """gm_newton_schulz through the entry point that allocates no device memory
    (its scratch is a fixed 64 MiB array inside the library). ``out`` must be
    preallocated by callers that cannot allocate either."""
    B, m, n = _bmn(X)
    _expect(X, (B, m, n), tuple(_DT), "X")
    O = out if out is not None else torch.empty((B, m, n), dtype=out_dtype, device=X.device)
    _expect(O, (B, m, n), tuple(_DT), "out")
    _check(lib.gm_newton_schulz_noalloc(B, m, n, _ptr(X), _DT[X.dtype], abc_table(abc, T), T, eps,
                                        _ptr(O), _DT[O.dtype], _stream()),
           "gm_newton_schulz_noalloc")
    return O


def gram_ns(X, abc=None, T=5, restart_after=(2,), eps=1e-7, out_dtype=torch.float32, out=None,
            ws=None):
    B, m, n = _bmn(X)
    _expect(X, (B, m, n), tuple(_DT), "X")
    O = out if out is not None else torch.empty((B, m, n), dtype=out_dtype, device=X.device)
    _expect(O, (B, m, n), tuple(_DT), "out")
    out_dtype = O.dtype
    nb = workspace_bytes(GM_OP_GRAM_NS, B, m, n)
    ws = ws if ws is not None else workspace(nb, X.device)
    _ws_fits(ws, nb)
    rl = list(restart_after)
    rarr = (c_int * max(1, len(rl)))(*rl) if rl else None
    _check(lib.gm_gram_ns(B, m, n, _ptr(X), _DT[X.dtype], abc_table(abc, T), T, rarr, len(rl),
                          eps, _ptr(O), _DT[out_dtype], _ptr(ws), nb, _stream()), "gm_gram_ns")
    return O


_sig("gm_gram_ns_trace", c_int, [c_int, c_int, c_int, vp, c_int, vp, c_int, vp, c_int, c_float,
                                 vp, c_int, vp, vp, vp, c_size_t, vp])


def gram_ns_trace(X, abc=None, T=5, restart_after=(2,), eps=1e-7, out_dtype=torch.float32):
    """gm_gram_ns_trace: returns (O, R_trace, Q_trace), the traces fp16
    [T, B, N, N] (N = min(m, n)): Q_t after every step, R_t where the chain
    computes it (zeros at t = T; the restarted Gram after a restart step)."""
    B, m, n = _bmn(X)
    _expect(X, (B, m, n), tuple(_DT), "X")
    N = min(m, n)
    Np = -(-N // 64) * 64
    O = torch.empty((B, m, n), dtype=out_dtype, device=X.device)
    Rt = torch.zeros((T, B, Np, Np), dtype=torch.float16, device=X.device)
    Qt = torch.zeros_like(Rt)
    nb = workspace_bytes(GM_OP_GRAM_NS, B, m, n)
    ws = workspace(nb, X.device)
    rl = list(restart_after)
    rarr = (c_int * max(1, len(rl)))(*rl) if rl else None
    _check(lib.gm_gram_ns_trace(B, m, n, _ptr(X), _DT[X.dtype], abc_table(abc, T), T, rarr, len(rl),
                                eps, _ptr(O), _DT[out_dtype], _ptr(Rt), _ptr(Qt), _ptr(ws), nb,
                                _stream()), "gm_gram_ns_trace")
    return O, Rt[..., :N, :N], Qt[..., :N, :N]


def ns_flops(ns, m, n, T=5, restart_after=(2,)):
    rl = list(restart_after) if ns == GM_NS_GRAM else []
    rarr = (c_int * max(1, len(rl)))(*rl) if rl else None
    f = ctypes.c_double()
    cnt = c_int()
    _check(lib.gm_ns_flops(ns, m, n, T, rarr, len(rl), ctypes.byref(f), ctypes.byref(cnt)),
           "gm_ns_flops")
    return f.value, cnt.value


def device_errors():
    _check(lib.gm_device_errors(_stream()), "gm_device_errors")


def wait_timeout_probe(limit_ns=20_000_000):
    """gm_test_wait_timeout: one product launch whose bounded wait runs out
    after limit_ns (a test hook of the failure path)."""
    X = torch.zeros((256, 256), dtype=torch.bfloat16, device="cuda")
    D = torch.empty_like(X)
    _check(lib.gm_test_wait_timeout(_ptr(X), _ptr(D), int(limit_ns), _stream()),
           "gm_test_wait_timeout")
    return X, D


@dataclass
class GraspState:
    """Device tensors of the quantized momentum of B same-shape matrices."""
    codes4: torch.Tensor
    rscale: torch.Tensor
    cscale: torch.Tensor
    P8: torch.Tensor
    Pscale: torch.Tensor
    R8: torch.Tensor
    Rscale: torch.Tensor
    step: torch.Tensor
    dev_status: torch.Tensor

    @staticmethod
    def zeros(B, m, n, k, device=None):
        d = device or torch.device("cuda")
        mb, nb = -(-m // GRID_BLOCK), -(-n // GRID_BLOCK)
        z = lambda shape, dt: torch.zeros(shape, dtype=dt, device=d)   # noqa: E731
        return GraspState(z((B, m, n // 2), torch.uint8), z((B, m, nb), torch.float32),
                          z((B, mb, n), torch.float32), z((B, m, k), torch.int8),
                          z((B, k), torch.float32), z((B, n, k), torch.int8),
                          z((B, k), torch.float32), z((1,), torch.int64), z((1,), torch.int32))

    def tensors(self):
        return [self.codes4, self.rscale, self.cscale, self.P8, self.Pscale, self.R8,
                self.Rscale, self.step, self.dev_status]

    def check(self, B, m, n, k):
        """Raises ValueError unless every tensor has the layout gm_grasp_step
        reads and writes for B matrices of m x n at top rank k."""
        mb, nb = -(-m // GRID_BLOCK), -(-n // GRID_BLOCK)
        f32, i8 = (torch.float32,), (torch.int8,)
        _expect(self.codes4, (B, m, n // 2), (torch.uint8,), "codes4")
        _expect(self.rscale, (B, m, nb), f32, "rscale")
        _expect(self.cscale, (B, mb, n), f32, "cscale")
        _expect(self.P8, (B, m, k), i8, "P8")
        _expect(self.Pscale, (B, k), f32, "Pscale")
        _expect(self.R8, (B, n, k), i8, "R8")
        _expect(self.Rscale, (B, k), f32, "Rscale")
        _expect(self.step, (1,), (torch.int64,), "step")
        _expect(self.dev_status, (1,), (torch.int32,), "dev_status")
        _placed(self.tensors(), ["codes4", "rscale", "cscale", "P8", "Pscale", "R8", "Rscale",
                                 "step", "dev_status"])

    def c_struct(self):
        return GraspStateC(*[t.data_ptr() for t in self.tensors()])

    def clone(self):
        return GraspState(*[t.clone() for t in self.tensors()])


def ipc_export(t):
    """(handle bytes, byte offset) of the device allocation holding tensor t (gm_ipc_export)."""
    _placed((t,), ("t",))
    h = IpcHandle()
    off = c_size_t()
    _check(lib.gm_ipc_export(_ptr(t), ctypes.byref(h), ctypes.byref(off)), "gm_ipc_export")
    return bytes(h.bytes), off.value


def ipc_open(handle: bytes) -> int:
    """Device address of the start of another process's exported allocation (gm_ipc_open)."""
    h = IpcHandle()
    ctypes.memmove(h.bytes, handle, 64)
    base = vp()
    _check(lib.gm_ipc_open(ctypes.byref(h), ctypes.byref(base)), "gm_ipc_open")
    return base.value


def ipc_close(base: int) -> None:
    _check(lib.gm_ipc_close(vp(base)), "gm_ipc_close")


def weight_update(W, O, eta, wd=0.0, skip=None):
    """W <- W - eta (O + wd W) in place (gm_weight_update); O in float32, bfloat16 or
    float16 of W's shape. ``skip`` (optional device int32): one flag for the batch
    ([1]) or one per matrix ([B]); a flagged matrix keeps its weights."""
    B, m, n = _bmn(W)
    _expect(W, (B, m, n), (torch.float32,), "W")
    _expect(O, (B, m, n), (torch.float32, torch.bfloat16, torch.float16), "O")
    stride = 0
    if skip is not None:
        if skip.dtype != torch.int32 or not skip.is_contiguous() or skip.numel() not in (1, B):
            raise ValueError("skip: a contiguous int32 tensor of 1 or B flags expected")
        stride = 0 if skip.numel() == 1 else 1
        _placed((W, O, skip), ("W", "O", "skip"))
    else:
        _placed((W, O), ("W", "O"))
    _check(lib.gm_weight_update(B, m, n, float(eta), float(wd), _ptr(O), _DT[O.dtype], _ptr(W),
                                _ptr(skip), stride, _stream()), "gm_weight_update")
    return W


class GraspStep:
    """Marshals one gm_grasp_step call for a fixed shape batch.

    ``matrix_ids`` (optional): each matrix's index in the whole parameter set,
    used by the Rademacher start vectors (default 0 .. B-1); ``power_steps``
    (1..3) and ``residual_from_codes`` select the ablation variants."""

    def __init__(self, B, m, n, k, mu=0.95, eta=0.02, wd=0.0, T=5, ns=GM_NS_STANDARD, abc=None,
                 restart_after=(2,), eps=1e-7, seed=0, device=None, ws=None, power_steps=1,
                 residual_from_codes=False, matrix_ids=None):
        self.B, self.m, self.n, self.k = B, m, n, k
        self._abc = abc_table(abc, T)
        rl = list(restart_after) if ns == GM_NS_GRAM else []
        self._rarr = (c_int * max(1, len(rl)))(*rl)
        dev = device or torch.device("cuda")
        self.ids = None
        if matrix_ids is not None:
            ids = [int(i) for i in matrix_ids]
            if len(ids) != B or not all(0 <= i < 65536 for i in ids):
                raise ValueError("matrix_ids: B indices in [0, 65536) expected")
            self.ids = torch.tensor(ids, dtype=torch.int64, device=dev)
        self.params = GraspParams(mu, eta, wd, k, T, ns,
                                  ctypes.cast(self._abc, ctypes.POINTER(c_float)) if self._abc else None,
                                  ctypes.cast(self._rarr, ctypes.POINTER(c_int)) if rl else None,
                                  len(rl), eps, seed, int(power_steps), int(bool(residual_from_codes)),
                                  self.ids.data_ptr() if self.ids is not None else None)
        self.ws_bytes = workspace_bytes(GM_OP_GRASP_STEP, B, m, n, k, ns)
        if ws is None:
            ws = torch.empty(self.ws_bytes, dtype=torch.uint8, device=dev)
        self.ws = ws
        lay = GraspWsLayout()
        _check(lib.gm_grasp_workspace_layout(B, m, n, k, ns, ctypes.byref(lay)),
               "gm_grasp_workspace_layout")
        self.layout = lay
        self.ns = ns

    def __call__(self, state: GraspState, W, G):
        B, m, n = self.B, self.m, self.n
        _expect(W, (B, m, n), (torch.float32,), "W")
        _expect(G, (B, m, n), tuple(_DT), "G")
        state.check(B, m, n, self.k)
        _placed((W, G), ("W", "G"))
        _ws_fits(self.ws, self.ws_bytes)
        st = state.c_struct()
        _check(lib.gm_grasp_step(self.B, self.m, self.n, ctypes.byref(self.params), ctypes.byref(st),
                                 _ptr(W), _ptr(G), _DT[G.dtype], _ptr(self.ws), self.ws_bytes,
                                 _stream()), "gm_grasp_step")

    def state_update(self, state: GraspState, G):
        """Worked steps 1-5 alone (gm_grasp_state_update)."""
        B, m, n = self.B, self.m, self.n
        _expect(G, (B, m, n), tuple(_DT), "G")
        state.check(B, m, n, self.k)
        _placed((G,), ("G",))
        _ws_fits(self.ws, self.ws_bytes)
        st = state.c_struct()
        _check(lib.gm_grasp_state_update(B, m, n, ctypes.byref(self.params), ctypes.byref(st),
                                         _ptr(G), _DT[G.dtype], _ptr(self.ws), self.ws_bytes,
                                         _stream()), "gm_grasp_state_update")

    def apply(self, state: GraspState, W):
        """Worked step 6 alone (gm_grasp_apply) on the NS input the state update left."""
        B, m, n = self.B, self.m, self.n
        _expect(W, (B, m, n), (torch.float32,), "W")
        state.check(B, m, n, self.k)
        _placed((W,), ("W",))
        _ws_fits(self.ws, self.ws_bytes)
        st = state.c_struct()
        _check(lib.gm_grasp_apply(B, m, n, ctypes.byref(self.params), ctypes.byref(st), _ptr(W),
                                  _ptr(self.ws), self.ws_bytes, _stream()), "gm_grasp_apply")

    def orth(self, state: GraspState, out=None, dtype=torch.bfloat16):
        """Worked step 6 up to O = NS(M_t) (gm_grasp_orth) on the NS input the state
        update left; O [B, m, n] in ``dtype`` (float32, bfloat16 or float16), not
        written when the state update flagged a non-finite value."""
        B, m, n = self.B, self.m, self.n
        state.check(B, m, n, self.k)
        if out is None:
            out = torch.empty((B, m, n), dtype=dtype, device=self.ws.device)
        _expect(out, (B, m, n), (torch.float32, torch.bfloat16, torch.float16), "O")
        _placed((out,), ("O",))
        _ws_fits(self.ws, self.ws_bytes)
        st = state.c_struct()
        _check(lib.gm_grasp_orth(B, m, n, ctypes.byref(self.params), ctypes.byref(st), _ptr(out),
                                 _DT[out.dtype], _ptr(self.ws), self.ws_bytes, _stream()),
               "gm_grasp_orth")
        return out

    def orth_peers(self, state: GraspState, peer_O, peer_flags, dst_index, dtype=torch.bfloat16):
        """O = NS(M_t) on the NS input the state update left, stored into every receive
        buffer of ``peer_O`` (device addresses of [.][m][n] ``dtype`` buffers, this
        process's or mapped from others) at matrix dst_index[b], with the step's status
        in ``peer_flags`` (int32 buffers) at the same index (gm_grasp_orth_peers)."""
        B, m, n = self.B, self.m, self.n
        state.check(B, m, n, self.k)
        if not 1 <= len(peer_O) == len(peer_flags) <= 8:
            raise ValueError("1 to 8 receive buffers, one flag buffer each")
        if dst_index.dtype != torch.int64 or tuple(dst_index.shape) != (B,):
            raise ValueError("dst_index: int64 [B] expected")
        _placed((dst_index,), ("dst_index",))
        _ws_fits(self.ws, self.ws_bytes)
        po = (vp * len(peer_O))(*[vp(int(a)) for a in peer_O])
        pf = (vp * len(peer_flags))(*[vp(int(a)) for a in peer_flags])
        st = state.c_struct()
        _check(lib.gm_grasp_orth_peers(B, m, n, ctypes.byref(self.params), ctypes.byref(st), po, pf,
                                       len(peer_O), _ptr(dst_index), _DT[dtype], _ptr(self.ws),
                                       self.ws_bytes, _stream()), "gm_grasp_orth_peers")

    def direction(self, state: GraspState, G, out=None, dtype=torch.bfloat16):
        """Worked steps 1-5 and O = NS(M_t): the state update, then ``orth``."""
        self.state_update(state, G)
        return self.orth(state, out, dtype)

    # stage buffers inside the workspace (views; valid after the step ran)
    def _view(self, off, shape, dtype):
        nbytes = 1
        for s in shape:
            nbytes *= s
        nbytes *= torch.empty((), dtype=dtype).element_size()
        return self.ws[off:off + nbytes].view(dtype).view(shape)

    def stage_M(self):
        return self._view(self.layout.M, (self.B, self.m, self.n), torch.float32)

    def stage_Q(self):
        return self._view(self.layout.Q, (self.B, self.n, self.k), torch.float32)

    def stage_P(self):
        return self._view(self.layout.P, (self.B, self.m, self.k), torch.float32)

    def stage_R(self):
        return self._view(self.layout.R, (self.B, self.n, self.k), torch.float32)

    def stage_scale(self):
        return self._view(self.layout.scale, (self.B,), torch.float32)

    def stage_X(self):
        N, Mp = min(self.m, self.n), max(self.m, self.n)
        dt = torch.float16 if self.ns == GM_NS_GRAM else torch.bfloat16
        return self._view(self.layout.X, (self.B, N, Mp), dt)
