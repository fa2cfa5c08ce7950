"""fp64 oracle of the 4-bit-Muon-GRASP step (test infrastructure only).

Everything is written for one matrix at a time with plain torch CPU ops; a
matmul is the only library primitive used as a step. Quantization decisions
(an integer code from a float) are taken in fp32, the precision the CUDA
kernels decide them in: IEEE fp32 division, fp32 multiply by 7 or 127,
round-half-to-even, clamp. All other arithmetic is fp64.

Readings of points the pages leave open:

* NS coefficients: T=5 steps of the constant quintic (a,b,c) =
  (3.4445, -4.7750, 2.0315) [LiMuon, key design 3], for both the standard
  and the Gram form.
* Grid scales are absolute maxima inside each block x block tile (the page
  prints "max x"); codes are symmetric signed 4-bit, q in [-7, 7], stored as a
  two's-complement nibble, low nibble = even column.
* 8-bit factors use one absmax scale per column; q in [-127, 127].
* A zero scale gives code 0.
* Step 1 (no stored R) and any all-zero column of R use a Rademacher start
  column: +-1/sqrt(n), sign = top bit of splitmix64(seed ^ b<<48 ^ j<<16 ^ l).
* Thin QR with positive diagonal; a column whose residual after removing the
  earlier live columns has norm <= 1e-6 * (largest column norm) is dead: it is
  zero in P and therefore in R.
* The residual uses the unquantized new P and R.
* NS runs on the fp64 momentum of this step; tall matrices (rows > cols) are
  transposed first, square ones are not.
* The 4bit-Muon-base codec the note compares against quantizes the whole
  matrix in groups of 128 consecutive row-major elements, one absmax scale
  per group, codes in [-7, 7] like the grid codec.
* MuonQ's mu-law codec (only its abstract is on the pages): the same groups
  and absmax normalisation, mu = 255, codes rint(7 F(x / s)) in [-7, 7].
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

DT = torch.float64
F32 = torch.float32

#: Constant quintic coefficients [LiMuon, key design 3 (NS version)].
QUINTIC_ABC = (3.4445, -4.7750, 2.0315)
#: Frobenius pre-normalisation epsilon [GramNS, Algorithm 1, first line].
NS_EPS = 1e-7
#: Group / grid size [GRASP, training strategy: group and grid size 128].
GRID_BLOCK = 128
#: Dead-column threshold of the QR (reading of [GRASP, worked step, step 4]).
QR_DEAD_TOL = 1e-6

__all__ = [
    "QUINTIC_ABC", "NS_EPS", "GRID_BLOCK", "QR_DEAD_TOL",
    "splitmix64", "rademacher_sign", "rademacher_column", "warm_start",
    "orth_positive", "power_iteration",
    "quant8", "dequant8", "grid_quant4", "grid_scale_matrix", "grid_dequant4",
    "pack_nibbles", "unpack_nibbles", "group_quant4", "group_dequant4",
    "MULAW_MU", "mulaw_compress", "mulaw_expand", "mulaw_quant4", "mulaw_dequant4",
    "ns_standard", "gram_ns", "quintic_scalar", "POLAR_EXPRESS_ABC", "safety_scaled",
    "GraspState", "zero_state", "rebuild_momentum", "grasp_step",
]

# --------------------------------------------------------------------------
# Counter-based generator for the step-1 start vectors
# --------------------------------------------------------------------------

_MASK64 = (1 << 64) - 1


def splitmix64(x: int) -> int:
    """splitmix64 output for counter ``x``.

    Published definition (Steele, Lea and Flood, "Fast splittable
    pseudorandom number generators", 2014): add the golden-ratio increment
    0x9E3779B97F4A7C15, then two xor-shift-multiply rounds and a final
    xor-shift.
    """
    z = (x + 0x9E3779B97F4A7C15) & _MASK64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _MASK64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _MASK64
    return z ^ (z >> 31)


def rademacher_sign(seed: int, b: int, j: int, l: int) -> int:
    """+1 or -1 from the top bit of splitmix64(seed ^ b<<48 ^ j<<16 ^ l)."""
    ctr = (seed ^ (b << 48) ^ (j << 16) ^ l) & _MASK64
    return -1 if (splitmix64(ctr) >> 63) & 1 else 1


def rademacher_column(seed: int, b: int, n: int, l: int) -> torch.Tensor:
    """Column l of the step-1 start matrix: entries +-1/sqrt(n)."""
    col = torch.tensor([rademacher_sign(seed, b, j, l) for j in range(n)], dtype=DT)
    return col / math.sqrt(n)


def warm_start(R_hat: torch.Tensor, seed: int, b: int) -> torch.Tensor:
    """Q_t = column-normalised R_{t-1} [GRASP, key design 1 and worked step 2].

    A column with zero norm (step 1, or a dead column) takes the Rademacher
    start column instead.
    """
    n, k = R_hat.shape
    Q = torch.empty((n, k), dtype=DT)
    for l in range(k):
        col = R_hat[:, l].to(DT)
        nrm = math.sqrt(float((col * col).sum()))
        if nrm == 0.0:
            Q[:, l] = rademacher_column(seed, b, n, l)
        else:
            Q[:, l] = col / nrm
    return Q


# --------------------------------------------------------------------------
# One-step power iteration [GRASP, worked step 4: P <- M Q, QR, R <- M^T P]
# --------------------------------------------------------------------------

def orth_positive(Ptil: torch.Tensor, tol: float = QR_DEAD_TOL):
    """Orthonormal basis of span(Ptil), thin-QR convention diag(R_qr) > 0.

    Gram-Schmidt over the columns in order, each projection applied twice;
    column j keeps v / |v| where v is Ptil[:, j] minus its components along
    the earlier live columns. |v| <= tol * max_l |Ptil[:, l]| marks the column
    dead (zero). Returns (P, live) with ``live`` a list of bools.
    """
    m, k = Ptil.shape
    Ptil = Ptil.to(DT)
    colnorms = [math.sqrt(float((Ptil[:, l] * Ptil[:, l]).sum())) for l in range(k)]
    maxnorm = max(colnorms) if k else 0.0
    P = torch.zeros((m, k), dtype=DT)
    live = [False] * k
    for j in range(k):
        v = Ptil[:, j].clone()
        for _ in range(2):
            for l in range(j):
                if live[l]:
                    v = v - (P[:, l] @ v) * P[:, l]
        nv = math.sqrt(float((v * v).sum()))
        if nv <= tol * maxnorm or nv == 0.0:
            continue
        P[:, j] = v / nv
        live[j] = True
    return P, live


def power_iteration(M: torch.Tensor, Q: torch.Tensor, steps: int = 1, seed: int = 0, b: int = 0):
    """P, R = PowerIter(M, Q) [GRASP, worked step 4; ablation table, 1/2/3
    power-iteration steps].

    One step: P~ = M Q; P = orth(P~); R = M^T P. Each further step starts
    again from Q = column-normalised R of the step before, the same rule as
    the warm start (so a zero column of R, a dead one, restarts from its
    Rademacher column, drawn with ``seed`` and ``b``). Returns
    (P, R, P~, live) of the last step.
    """
    M = M.to(DT)
    Q = Q.to(DT)
    for s in range(steps):
        if s > 0:
            Q = warm_start(R, seed, b)
        Ptil = M @ Q
        P, live = orth_positive(Ptil)
        R = M.T @ P
    return P, R, Ptil, live


# --------------------------------------------------------------------------
# 8-bit factors [GRASP, worked step 5 and training strategy: INT8 P, R]
# --------------------------------------------------------------------------

def quant8(X: torch.Tensor):
    """Per-column absmax INT8 codes of an fp32 (rows, k) matrix.

    s_l = max_i |x_il|; q = clamp(rint(fp32(x / s_l) * 127), -127, 127);
    s_l = 0 gives q = 0. Returns (codes int8, scales fp32 (k,)).
    """
    X = X.to(F32)
    s = X.abs().amax(dim=0) if X.shape[0] else torch.zeros(X.shape[1], dtype=F32)
    safe = torch.where(s > 0, s, torch.ones_like(s))
    r = X / safe                       # IEEE fp32 division
    r = r * torch.tensor(127.0, dtype=F32)
    q = torch.clamp(torch.round(r), -127, 127)   # round half to even
    q = torch.where(s > 0, q, torch.zeros_like(q))
    return q.to(torch.int8), s


def dequant8(codes: torch.Tensor, scale: torch.Tensor) -> torch.Tensor:
    """x^ = (q / 127) * s_l in fp64."""
    return codes.to(DT) / 127.0 * scale.to(DT)


# --------------------------------------------------------------------------
# 4-bit grid quantization [GRASP, key design 2: scale^r, scale^c, N_grid]
# --------------------------------------------------------------------------

def grid_quant4(X: torch.Tensor, block: int = GRID_BLOCK):
    """Grid quantization of an fp32 (m, n) matrix.

    Inside each block x block tile: r_i = max_j |x_ij| (row scale), c_j =
    max_i |x_ij| (column scale); every element is normalised by
    s_ij = min(r_i, c_j) and coded as q = clamp(rint(fp32(x / s) * 7), -7, 7),
    with s = 0 giving 0. Ragged edge tiles are smaller.

    Returns (codes int8 (m, n), rscale fp32 (m, nb), cscale fp32 (mb, n)).
    """
    X = X.to(F32)
    m, n = X.shape
    mb, nb = -(-m // block), -(-n // block)
    A = X.abs()
    rscale = torch.zeros((m, nb), dtype=F32)
    cscale = torch.zeros((mb, n), dtype=F32)
    for bi in range(mb):
        r0, r1 = bi * block, min(m, (bi + 1) * block)
        for bj in range(nb):
            c0, c1 = bj * block, min(n, (bj + 1) * block)
            tile = A[r0:r1, c0:c1]
            rscale[r0:r1, bj] = tile.amax(dim=1)
            cscale[bi, c0:c1] = tile.amax(dim=0)
    s = grid_scale_matrix(rscale, cscale, m, n, block)
    safe = torch.where(s > 0, s, torch.ones_like(s))
    r = (X / safe) * torch.tensor(7.0, dtype=F32)
    q = torch.clamp(torch.round(r), -7, 7)
    q = torch.where(s > 0, q, torch.zeros_like(q))
    return q.to(torch.int8), rscale, cscale


def grid_scale_matrix(rscale, cscale, m, n, block=GRID_BLOCK):
    """Per-element s_ij = min(rscale[i, j // block], cscale[i // block, j])."""
    cols = torch.arange(n) // block
    rows = torch.arange(m) // block
    r_full = rscale[:, cols]            # (m, n)
    c_full = cscale[rows, :]            # (m, n)
    return torch.minimum(r_full, c_full)


def grid_dequant4(codes, rscale, cscale, block: int = GRID_BLOCK) -> torch.Tensor:
    """x^ = (q / 7) * s_ij in fp64."""
    m, n = codes.shape
    s = grid_scale_matrix(rscale, cscale, m, n, block).to(DT)
    return codes.to(DT) / 7.0 * s


def group_quant4(X: torch.Tensor, group: int = 128):
    """The 4bit-Muon-base codec the GRASP note compares against (its results
    tables' "4bit-Muon-base" rows; the motivation's direct quantization of
    Muon's momentum): blockwise 4-bit of the whole matrix with one absmax
    scale per group of `group` consecutive elements in row-major order (a
    shorter last group when the count is not a multiple of `group`);
    q = clamp(rint(fp32(x / s) * 7), -7, 7), s = 0 giving 0.

    Returns (codes int8 (m, n), scales fp32 (ceil(m n / group),))."""
    x = X.to(F32).reshape(-1)
    ng = -(-x.numel() // group)
    scales = torch.zeros(ng, dtype=F32)
    codes = torch.zeros(x.numel(), dtype=torch.int8)
    for gi in range(ng):
        seg = x[gi * group:(gi + 1) * group]
        s = seg.abs().max()
        scales[gi] = s
        if s > 0:
            r = (seg / s) * torch.tensor(7.0, dtype=F32)
            codes[gi * group:(gi + 1) * group] = torch.clamp(torch.round(r), -7, 7).to(torch.int8)
    return codes.view(X.shape), scales


def group_dequant4(codes: torch.Tensor, scales: torch.Tensor, group: int = 128) -> torch.Tensor:
    """x^ = (q / 7) * s of the element's group, in fp64."""
    q = codes.reshape(-1).to(DT)
    s = scales.to(DT).repeat_interleave(group)[: q.numel()]
    return (q / 7.0 * s).view(codes.shape)


#: mu of the mu-law companding codec (the G.711 value; MuonQ states none).
MULAW_MU = 255.0


def mulaw_compress(x: torch.Tensor, mu: float = MULAW_MU) -> torch.Tensor:
    """F(x) = sign(x) ln(1 + mu |x|) / ln(1 + mu) for |x| <= 1, in fp64."""
    x = x.to(DT)
    return torch.sign(x) * torch.log1p(mu * x.abs()) / math.log1p(mu)


def mulaw_expand(y: torch.Tensor, mu: float = MULAW_MU) -> torch.Tensor:
    """F^-1(y) = sign(y) ((1 + mu)^|y| - 1) / mu, in fp64."""
    y = y.to(DT)
    return torch.sign(y) * torch.expm1(y.abs() * math.log1p(mu)) / mu


def mulaw_quant4(X: torch.Tensor, group: int = 128, mu: float = MULAW_MU):
    """4-bit mu-law companding codes, the third part of MuonQ (its abstract:
    finer steps where momentum values are dense, coarser at the outliers).
    Each group of `group` consecutive row-major elements is normalised by its
    absmax s (the plainest reading of MuonQ's unstated pre-quantization
    normalisation) and q = clamp(rint(7 F(x / s)), -7, 7); s = 0 gives 0.
    Returns (codes int8 (m, n), scales fp32 (ceil(m n / group),))."""
    x = X.to(F32).reshape(-1)
    ng = -(-x.numel() // group)
    scales = torch.zeros(ng, dtype=F32)
    codes = torch.zeros(x.numel(), dtype=torch.int8)
    for gi in range(ng):
        seg = x[gi * group:(gi + 1) * group]
        s = seg.abs().max()
        scales[gi] = s
        if s > 0:
            y = mulaw_compress(seg.to(DT) / float(s), mu)
            codes[gi * group:(gi + 1) * group] = torch.clamp(torch.round(7.0 * y), -7, 7).to(torch.int8)
    return codes.view(X.shape), scales


def mulaw_dequant4(codes: torch.Tensor, scales: torch.Tensor, group: int = 128,
                   mu: float = MULAW_MU) -> torch.Tensor:
    """x^ = s F^-1(q / 7), in fp64."""
    q = codes.reshape(-1).to(DT)
    s = scales.to(DT).repeat_interleave(group)[: q.numel()]
    return (s * mulaw_expand(q / 7.0, mu)).view(codes.shape)


def pack_nibbles(codes: torch.Tensor) -> torch.Tensor:
    """(m, n) int8 codes in [-8, 7] -> (m, n/2) uint8, low nibble = even column."""
    c = codes.to(torch.int16) & 0xF
    return (c[:, 0::2] | (c[:, 1::2] << 4)).to(torch.uint8)


def unpack_nibbles(packed: torch.Tensor) -> torch.Tensor:
    """Inverse of pack_nibbles: sign-extend each two's-complement nibble."""
    p = packed.to(torch.int16)
    lo, hi = p & 0xF, (p >> 4) & 0xF
    lo = torch.where(lo >= 8, lo - 16, lo)
    hi = torch.where(hi >= 8, hi - 16, hi)
    out = torch.empty((p.shape[0], 2 * p.shape[1]), dtype=torch.int8)
    out[:, 0::2] = lo.to(torch.int8)
    out[:, 1::2] = hi.to(torch.int8)
    return out


# --------------------------------------------------------------------------
# Newton-Schulz [GramNS §1.2 standard NS; Algorithm 1 / 2 Gram NS]
# --------------------------------------------------------------------------

def _wide(X: torch.Tensor):
    """Transpose rule: run NS on the orientation with rows <= cols
    [GramNS, Algorithm 1 input X in R^{n x m}, n <= m]."""
    tall = X.shape[0] > X.shape[1]
    return (X.T if tall else X), tall


def ns_standard(X: torch.Tensor, abc=None, T: int = 5, eps: float = NS_EPS) -> torch.Tensor:
    """Standard quintic Newton-Schulz [GramNS §1.2, eq. (2)].

    X <- X / (|X|_F + eps); then for each step A = X X^T,
    B = b A + c A^2, X <- a X + B X. ``abc`` is a list of T (a, b, c)
    triples (default: the constant quintic, T times).
    """
    if abc is None:
        abc = [QUINTIC_ABC] * T
    Y, tall = _wide(X.to(DT))
    Y = Y / (torch.linalg.matrix_norm(Y) + eps)
    for a, b, c in abc:
        A = Y @ Y.T
        B = b * A + c * (A @ A)
        Y = a * Y + B @ Y
    return Y.T if tall else Y


def gram_ns(X: torch.Tensor, abc=None, T: int = 5, restart_after=(2,),
            eps: float = NS_EPS, trace: list | None = None) -> torch.Tensor:
    """Gram Newton-Schulz [GramNS, Algorithm 2; Algorithm 1 when no restart].

    X <- X / (|X|_F + eps); R = X X^T; Q = I; for each step
    Z = b R + c R^2, Q <- Q Z + a Q, RZ = R Z + a R, R <- Z RZ + a RZ.
    After each step listed in ``restart_after`` (1-based, before the last
    step): X <- Q X, R <- X X^T, Q <- I. Returns Q X.

    With a list as ``trace``, every step t appends (t, smallest eigenvalue of
    R_t, condition number of Q_t), taken after the step's update and before
    any restart: the two quantities [GramNS §3.2] bounds for its restart
    choice.
    """
    if abc is None:
        abc = [QUINTIC_ABC] * T
    T = len(abc)
    Y, tall = _wide(X.to(DT))
    Y = Y / (torch.linalg.matrix_norm(Y) + eps)
    n = Y.shape[0]
    I = torch.eye(n, dtype=DT)
    R = Y @ Y.T
    Q = I.clone()
    for t, (a, b, c) in enumerate(abc, start=1):
        Z = b * R + c * (R @ R)
        Q = Q @ Z + a * Q
        RZ = R @ Z + a * R
        R = Z @ RZ + a * RZ
        if trace is not None:
            sq = torch.linalg.svdvals(Q)
            trace.append((t, float(torch.linalg.eigvalsh(R)[0]), float(sq[0] / sq[-1])))
        if t in restart_after and t < T:
            Y = Q @ Y
            R = Y @ Y.T
            Q = I.clone()
    O = Q @ Y
    return O.T if tall else O


#: The Polar Express quintics as printed in [GramNS §3.2] (one per step).
POLAR_EXPRESS_ABC = ((8.123737, -22.232240, 16.373715), (4.026529, -2.776323, 0.514551),
                     (3.870284, -2.739120, 0.520999), (3.253351, -2.343223, 0.481420),
                     (2.300652, -1.668904, 0.418807))


def safety_scaled(abc, s: float = 1.05):
    """A coefficient table whose every step evaluates p_t(x / s): (a / s,
    b / s^3, c / s^5). Reading of the safety factor of [GramNS §3.3], whose
    formula (eq. (12)) is lost from the page: only its purpose, convergence
    for singular values up to 1.05, survives."""
    return [(a / s, b / s ** 3, c / s ** 5) for a, b, c in abc]


def quintic_scalar(x: float, abc=None, T: int = 5) -> float:
    """The scalar map p_T o ... o p_1 of Proposition 1 [GramNS §2.2]."""
    if abc is None:
        abc = [QUINTIC_ABC] * T
    for a, b, c in abc:
        x = a * x + b * x ** 3 + c * x ** 5
    return x


# --------------------------------------------------------------------------
# The full step [GRASP, overall framework and worked step 1-6]
# --------------------------------------------------------------------------

@dataclass
class GraspState:
    """Quantized momentum of one m x n matrix [GRASP, worked step, last para]."""
    codes4: torch.Tensor      # uint8 (m, n/2) packed 4-bit residual codes
    rscale: torch.Tensor      # fp32 (m, nb)
    cscale: torch.Tensor      # fp32 (mb, n)
    P8: torch.Tensor          # int8 (m, k)
    Pscale: torch.Tensor      # fp32 (k,)
    R8: torch.Tensor          # int8 (n, k)
    Rscale: torch.Tensor      # fp32 (k,)
    step: int = 0


def zero_state(m: int, n: int, k: int, block: int = GRID_BLOCK) -> GraspState:
    mb, nb = -(-m // block), -(-n // block)
    return GraspState(
        codes4=torch.zeros((m, n // 2), dtype=torch.uint8),
        rscale=torch.zeros((m, nb), dtype=F32), cscale=torch.zeros((mb, n), dtype=F32),
        P8=torch.zeros((m, k), dtype=torch.int8), Pscale=torch.zeros(k, dtype=F32),
        R8=torch.zeros((n, k), dtype=torch.int8), Rscale=torch.zeros(k, dtype=F32),
        step=0)


def rebuild_momentum(st: GraspState, block: int = GRID_BLOCK) -> torch.Tensor:
    """M_{t-1} = deq4(M^q_res) + deq8(P^q) deq8(R^q)^T [GRASP, worked step 1]."""
    res = grid_dequant4(unpack_nibbles(st.codes4), st.rscale, st.cscale, block)
    return res + dequant8(st.P8, st.Pscale) @ dequant8(st.R8, st.Rscale).T


@dataclass
class StepResult:
    state: GraspState
    W: torch.Tensor                     # fp64 updated weight
    M: torch.Tensor                     # fp64 momentum M_t
    Q: torch.Tensor                     # fp64 warm start
    Ptil: torch.Tensor
    P: torch.Tensor
    R: torch.Tensor
    residual: torch.Tensor              # fp64 M_t - P R^T
    O: torch.Tensor                     # fp64 orthogonalised update
    live: list = field(default_factory=list)


def grasp_step(st: GraspState, W: torch.Tensor, G: torch.Tensor, *, mu: float, eta: float,
               wd: float = 0.0, seed: int = 0, b: int = 0, ns: str = "standard",
               abc=None, T: int = 5, restart_after=(2,), block: int = GRID_BLOCK,
               power_steps: int = 1, residual: str = "exact") -> StepResult:
    """One GRASP step for one matrix, in the order of [GRASP, worked step]:

    1. rebuild M_{t-1} from the stored codes;
    2. warm start Q_t = column-normalised R_{t-1};
    3. M_t = mu M_{t-1} + G;
    4. P, R = PowerIter(M_t, Q_t) (``power_steps`` steps: the ablation table's
       1/2/3-step rows; the method uses one);
    5. M_res = M_t - P R^T -> 4-bit grid codes; P, R -> 8-bit codes.
       ``residual="codes"`` is the variant that subtracts the dequantized
       8-bit factors instead, M_t - P^ R^T (the worked step writes the
       unquantized P, R, the default);
    6. O = NS(M_t); W <- W - eta (O + wd W).

    ``b`` is the matrix's index in the Rademacher counter.
    """
    M_prev = rebuild_momentum(st, block)
    Q = warm_start(dequant8(st.R8, st.Rscale), seed, b)
    M = mu * M_prev + G.to(DT)
    P, R, Ptil, live = power_iteration(M, Q, power_steps, seed, b)
    P8, Ps = quant8(P.to(F32))
    R8, Rs = quant8(R.to(F32))
    if residual == "exact":
        residual = M - P @ R.T
    elif residual == "codes":
        residual = M - dequant8(P8, Ps) @ dequant8(R8, Rs).T
    else:
        raise ValueError(residual)
    q4, rs, cs = grid_quant4(residual.to(F32), block)
    if ns == "standard":
        O = ns_standard(M, abc, T)
    elif ns == "gram":
        O = gram_ns(M, abc, T, restart_after)
    else:
        raise ValueError(ns)
    W64 = W.to(DT)
    Wn = W64 - eta * (O + wd * W64)
    new = GraspState(codes4=pack_nibbles(q4), rscale=rs, cscale=cs, P8=P8, Pscale=Ps,
                     R8=R8, Rscale=Rs, step=st.step + 1)
    return StepResult(state=new, W=Wn, M=M, Q=Q, Ptil=Ptil, P=P, R=R, residual=residual,
                      O=O, live=live)
