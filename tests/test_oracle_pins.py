"""Pins of the fp64 oracle against what the pages and the mathematics fix.

None of these tests compares the oracle with itself: each checks it against a
closed form, a theorem of the pages, brute force, a library routine or a
printed value (fixtures under tests/golden, each with its citation).
"""

import math
import os

import pytest
import torch

import oracle as O
from bit_muon_optimizer_b200 import flops as F

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
DT = torch.float64


def _orthogonal(n, gen):
    q, r = torch.linalg.qr(torch.randn(n, n, generator=gen, dtype=DT))
    return q * torch.sign(torch.diagonal(r))


def _read_sections(path):
    sec, out = None, {}
    for line in open(path):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        if line.startswith("["):
            sec = line.strip("[]")
            out[sec] = []
            continue
        out[sec].append(line.split())
    return out


# ---------------------------------------------------------------- generator

def test_splitmix64_published_stream():
    vals = []
    for line in open(os.path.join(GOLDEN, "splitmix64_seed0.txt")):
        if line.startswith("#") or not line.strip():
            continue
        i, v = line.split()
        vals.append((int(i), int(v, 16)))
    golden = 0x9E3779B97F4A7C15
    for i, v in vals:
        # splitmix64(x) adds the increment itself: counter (i-1)*golden gives output i
        assert O.splitmix64(((i - 1) * golden) & ((1 << 64) - 1)) == v


def test_rademacher_column_is_pm_one_over_sqrt_n_and_balanced():
    col = O.rademacher_column(1234, 3, 4096, 5)
    assert torch.all(torch.isclose(col.abs(), torch.full_like(col, 1 / 64.0)))
    frac_pos = float((col > 0).double().mean())
    assert 0.45 < frac_pos < 0.55
    assert float(col @ col) == pytest.approx(1.0, abs=1e-12)
    other = O.rademacher_column(1234, 3, 4096, 6)
    assert abs(float(col @ other)) < 0.1       # different counters -> different signs


# ---------------------------------------------------------- NS coefficients

def test_quintic_coefficients_match_printed_values():
    d = {}
    for line in open(os.path.join(GOLDEN, "ns_coefficients.txt")):
        if line.startswith("#") or not line.strip():
            continue
        k, v = line.split()
        d[k] = float(v)
    assert O.QUINTIC_ABC == (d["a"], d["b"], d["c"])


# ------------------------------------------------------ Proposition 1 (NS)

@pytest.mark.parametrize("m,n", [(6, 10), (24, 40), (40, 24), (32, 32)])
def test_ns_standard_proposition1_singular_vectors_kept(m, n):
    """NS(U S V^T) = U f(S) V^T, f the scalar composition [GramNS Prop. 1]."""
    gen = torch.Generator().manual_seed(7 + m * n)
    r = min(m, n)
    U = _orthogonal(m, gen)[:, :r]
    V = _orthogonal(n, gen)[:, :r]
    # sigma in [2e-3, 1] with |X|_F = 1: the top value absorbs the remaining norm
    rest = torch.logspace(math.log10(2e-3), math.log10(0.15), r - 1, dtype=DT)
    s = torch.cat([torch.sqrt(1 - (rest * rest).sum()).reshape(1), rest.flip(0)])
    X = U @ torch.diag(s) @ V.T
    out = O.ns_standard(X)
    scale = 1.0 / (1.0 + O.NS_EPS)
    fs = torch.tensor([O.quintic_scalar(float(v) * scale) for v in s], dtype=DT)
    expect = U @ torch.diag(fs) @ V.T
    assert torch.allclose(out, expect, atol=1e-10, rtol=0)
    sv = torch.linalg.svdvals(out)
    assert float(sv.min()) >= 0.6818 - 1e-4
    assert float(sv.max()) <= 1.2024 + 1e-4


def test_quintic_band_closed_form():
    """Scalar composition over [2e-3, 1] stays inside [0.6818, 1.2024]; f(1) = 0.6964."""
    xs = torch.linspace(2e-3, 1.0, 200001, dtype=DT)
    y = xs.clone()
    for a, b, c in [O.QUINTIC_ABC] * 5:
        y = a * y + b * y ** 3 + c * y ** 5
    assert 0.6818 <= float(y.min()) < 0.6819
    assert 1.2023 < float(y.max()) <= 1.2024
    assert O.quintic_scalar(1.0) == pytest.approx(0.6964, abs=1e-4)


def test_ns_standard_transpose_rule():
    gen = torch.Generator().manual_seed(3)
    X = torch.randn(12, 30, generator=gen, dtype=DT)
    assert torch.allclose(O.ns_standard(X.T), O.ns_standard(X).T, atol=1e-13)


# -------------------------------------------------------- Theorem 1 (Gram NS)

@pytest.mark.parametrize("m,n", [(4, 9), (16, 40), (64, 256), (40, 16)])
@pytest.mark.parametrize("restart", [(), (2,), (1, 3), (1, 2, 3, 4)])
def test_gram_ns_equals_standard_ns_in_fp64(m, n, restart):
    """Gram NS equals standard NS in exact arithmetic [GramNS Theorem 1]; a
    restart only regroups the same products [GramNS §3.2]."""
    gen = torch.Generator().manual_seed(m * 1000 + n)
    X = torch.randn(m, n, generator=gen, dtype=DT)
    a = O.ns_standard(X)
    g = O.gram_ns(X, restart_after=restart)
    assert float(torch.linalg.matrix_norm(g - a) / torch.linalg.matrix_norm(a)) < 1e-10


def test_gram_ns_polar_express_table_equivalence():
    """Theorem 1 holds for any per-step coefficients, e.g. the Polar Express
    table printed in [GramNS §3.2]."""
    pe = [(8.123737, -22.232240, 16.373715), (4.026529, -2.776323, 0.514551),
          (3.870284, -2.739120, 0.520999), (3.253351, -2.343223, 0.481420),
          (2.300652, -1.668904, 0.418807)]
    gen = torch.Generator().manual_seed(11)
    X = torch.randn(8, 20, generator=gen, dtype=DT) * 1e-3
    a = O.ns_standard(X, abc=pe)
    for restart in [(), (2,)]:
        g = O.gram_ns(X, abc=pe, restart_after=restart)
        assert float(torch.linalg.matrix_norm(g - a) / torch.linalg.matrix_norm(a)) < 1e-9


def test_gram_ns_negative_eigenvalue_grows():
    """[GramNS Prop. 2]: a negative eigenvalue of R grows under r <- r h(r)^2
    with h(x) = 15/8 - 10/8 x + 3/8 x^2. Checked on the oracle's R update by
    running it on a diagonal R with one negative entry."""
    abc = [(15 / 8, -10 / 8, 3 / 8)] * 5
    R = torch.diag(torch.tensor([0.5, 0.1, -1e-5], dtype=DT))
    # run the oracle's R recursion: Z = bR + cR^2; RZ = RZ + aR; R = Z RZ + a RZ
    mags = []
    for a, b, c in abc:
        Z = b * R + c * (R @ R)
        RZ = R @ Z + a * R
        R = Z @ RZ + a * RZ
        mags.append(abs(float(R[2, 2])))
    assert all(mags[i + 1] > 3.0 * mags[i] for i in range(4))
    # and the positive eigenvalues converge towards 1 (r_t = x_t^2)
    assert abs(float(R[0, 0]) - 1.0) < 0.05


def _composed(x, abc):
    for a, b, c in abc:
        x = a * x + b * x ** 3 + c * x ** 5
    return x


@pytest.mark.parametrize("restart", [(), (2,), (1, 3)])
def test_gram_ns_trace_closed_form(restart):
    """In exact arithmetic every iterate keeps X_0's singular vectors [GramNS
    Prop. 1, Theorem 1], so for X = U S V^T with normalised values s_i: R_t
    has eigenvalues f_t(s_i)^2 (f_t the first t polynomials composed) and Q_t,
    which maps the iterate at the last restart r (r = 0 at the start) to
    X_t, is U diag(f_t(s_i) / f_r(s_i)) U^T. The trace's smallest eigenvalue
    of R_t and condition number of Q_t must follow."""
    gen = torch.Generator().manual_seed(40)
    m, n = 24, 40
    U = _orthogonal(m, gen)
    V = _orthogonal(n, gen)[:, :m]
    s = torch.logspace(0, -3, m, dtype=DT)
    X = U @ torch.diag(s) @ V.T
    abc = O.safety_scaled(O.POLAR_EXPRESS_ABC)
    tr = []
    O.gram_ns(X, abc=abc, restart_after=restart, trace=tr)
    sh = s / (torch.linalg.matrix_norm(X) + O.NS_EPS)
    r = 0
    for t, lam, cond in tr:
        ft = _composed(sh, abc[:t])
        fr = _composed(sh, abc[:r])
        ratio = ft / fr
        assert lam == pytest.approx(float((ft * ft).min()), rel=1e-6, abs=1e-12)
        assert cond == pytest.approx(float(ratio.max() / ratio.min()), rel=1e-6)
        if t in restart:
            r = t


def test_polar_express_table_and_safety_factor_reading():
    """The Polar Express quintics printed in [GramNS §3.2] diverge as printed
    for singular values near 1 (the first maps 1 to 2.27); with the lost
    safety factor read as evaluating every step at x / 1.05 [GramNS §3.3],
    every normalised singular value in [1e-3, 1] lands in [0.68, 1.13]."""
    pe = O.POLAR_EXPRESS_ABC
    assert _composed(1.0, pe) > 1e6
    scaled = O.safety_scaled(pe, 1.05)
    xs = torch.cat([torch.logspace(-3, 0, 4001, dtype=DT)])
    y = _composed(xs, scaled)
    assert 0.68 < float(y.min()) and float(y.max()) < 1.13
    # the scaled coefficients evaluate each printed polynomial at x / 1.05
    gen = torch.Generator().manual_seed(41)
    x = torch.rand(50, generator=gen, dtype=DT) * 1.2
    for (a, b, c), (a2, b2, c2) in zip(pe, scaled):
        z = x / 1.05
        assert torch.allclose(a2 * x + b2 * x ** 3 + c2 * x ** 5, a * z + b * z ** 3 + c * z ** 5,
                              rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("smallest", [1e-3, 1e-4])
def test_restart_after_step_two_bounds_cond_q(smallest):
    """[GramNS §3.2]: with the Polar Express quintics, restarting after the
    second step keeps the condition number of Q_t below about 100. In exact
    arithmetic (no rounding) this already separates the two schedules on an
    input whose singular values fall to `smallest`: with the restart every
    cond(Q_t) stays below 100, without it some cond(Q_t) exceeds 100."""
    gen = torch.Generator().manual_seed(42)
    m, n = 24, 40
    U = _orthogonal(m, gen)
    V = _orthogonal(n, gen)[:, :m]
    X = U @ torch.diag(torch.logspace(0, math.log10(smallest), m, dtype=DT)) @ V.T
    abc = O.safety_scaled(O.POLAR_EXPRESS_ABC)
    with_restart, without = [], []
    O.gram_ns(X, abc=abc, restart_after=(2,), trace=with_restart)
    O.gram_ns(X, abc=abc, restart_after=(), trace=without)
    print(f"\n[singular values down to {smallest:g}] max cond(Q_t): "
          f"{max(c for _, _, c in with_restart):.1f} with the restart after step 2, "
          f"{max(c for _, _, c in without):.1f} without")
    assert max(c for _, _, c in with_restart) < 100
    assert max(c for _, _, c in without) > 100
    # and R_t stays positive semidefinite in exact arithmetic (the negative
    # eigenvalues the page bounds by -0.4 come from rounding)
    assert min(lam for _, lam, _ in with_restart + without) > -1e-12


# ------------------------------------------------------------ FLOP counters

def test_flop_counters_match_printed_savings():
    rows = []
    for line in open(os.path.join(GOLDEN, "gram_ns_flop_savings.txt")):
        if line.startswith("#") or not line.strip():
            continue
        v, a, s1, s2 = line.split()
        rows.append((v, int(a), int(s1), int(s2)))
    N = 64
    for v, alpha, s_sym, s_typ in rows:
        restart = () if v == "naive" else (2,)
        g = F.gram_ns_flops(N, alpha * N, 5, restart)
        std_sym = F.ns_standard_flops(N, alpha * N, 5, symmetric=True)
        std_typ = F.ns_standard_flops(N, alpha * N, 5, symmetric=False)
        assert round(100 * (1 - g / std_sym)) == s_sym
        assert round(100 * (1 - g / std_typ)) == s_typ


def test_flop_counter_closed_forms_and_gemm_counts():
    N = 32
    for alpha in [1, 2, 4, 8]:
        assert F.gram_ns_flops(N, alpha * N, 5, ()) == (17 + 3 * alpha) * N ** 3
        assert F.gram_ns_flops(N, alpha * N, 5, (2,)) == (14 + 6 * alpha) * N ** 3
        assert F.ns_standard_flops(N, alpha * N) == 5 * (3 * alpha + 1) * N ** 3
        assert F.ns_standard_flops(N, alpha * N, symmetric=False) == (20 * alpha + 10) * N ** 3
    assert F.gram_ns_gemm_count(5, ()) == 19
    # alpha = 1: Gram NS gives no saving over symmetric standard NS [GramNS §5.2]
    assert F.gram_ns_flops(N, N, 5, (2,)) == F.ns_standard_flops(N, N)
    # T-1 restarts regroup Gram NS into standard NS, product count aside [GramNS §3.4]
    assert F.ns_standard_flops(N, 4 * N) <= F.gram_ns_flops(N, 4 * N, 5, (1, 2, 3, 4))


# ------------------------------------------------------- power iteration + QR

def test_orth_positive_matches_library_qr_full_rank():
    gen = torch.Generator().manual_seed(5)
    A = torch.randn(200, 12, generator=gen, dtype=DT) * torch.logspace(0, -3, 12, dtype=DT)
    P, live = O.orth_positive(A)
    q, r = torch.linalg.qr(A)
    q = q * torch.sign(torch.diagonal(r))
    assert all(live)
    assert torch.allclose(P, q, atol=1e-11)
    Rqr = P.T @ A
    assert torch.all(torch.diagonal(Rqr) > 0)
    assert torch.allclose(torch.triu(Rqr), Rqr, atol=1e-11)   # upper triangular


def test_orth_positive_dead_columns():
    gen = torch.Generator().manual_seed(6)
    A = torch.randn(50, 4, generator=gen, dtype=DT)
    A[:, 2] = 2.0 * A[:, 0] - A[:, 1]          # exactly dependent
    A = torch.cat([A, torch.zeros(50, 1, dtype=DT)], dim=1)
    P, live = O.orth_positive(A)
    assert live == [True, True, False, True, False]
    assert torch.all(P[:, 2] == 0) and torch.all(P[:, 4] == 0)
    Pl = P[:, [0, 1, 3]]
    assert torch.allclose(Pl.T @ Pl, torch.eye(3, dtype=DT), atol=1e-13)
    # the live columns still span the input
    assert torch.allclose(Pl @ (Pl.T @ A), A, atol=1e-12)
    P0, live0 = O.orth_positive(torch.zeros(10, 3, dtype=DT))
    assert live0 == [False] * 3 and torch.all(P0 == 0)


def test_power_iteration_invariants():
    gen = torch.Generator().manual_seed(8)
    M = torch.randn(120, 90, generator=gen, dtype=DT)
    Q = O.warm_start(torch.zeros(90, 6), 99, 0)
    P, R, Ptil, live = O.power_iteration(M, Q)
    assert torch.allclose(P.T @ P, torch.eye(6, dtype=DT), atol=1e-13)
    assert torch.allclose(P @ (P.T @ Ptil), Ptil, atol=1e-11)       # P R_qr = P~
    res = M - P @ R.T
    assert float(torch.linalg.matrix_norm(P.T @ res)) < 1e-11       # P^T M_res = 0


def test_power_iteration_exact_rank_k_is_lossless():
    gen = torch.Generator().manual_seed(9)
    k = 5
    U = _orthogonal(80, gen)[:, :k]
    V = _orthogonal(60, gen)[:, :k]
    M = U @ torch.diag(torch.tensor([5.0, 4, 3, 2, 1], dtype=DT)) @ V.T
    Qs = V + 0.3 * torch.randn(60, k, generator=gen, dtype=DT)      # spans V_k generically
    P, R, _, live = O.power_iteration(M, Qs)
    assert all(live)
    assert float(torch.linalg.matrix_norm(M - P @ R.T)) < 1e-12


def test_power_iteration_subspace_bound():
    """One step of subspace iteration: tan(theta_1) <= (s_{k+1}/s_k) tan(theta_0)
    (textbook bound), and with s_k/s_{k+1} >= 20 from a warm start the relative
    error of the rank-k part is <= 0.01 (the 1-step figure of [GRASP, ablation])."""
    gen = torch.Generator().manual_seed(10)
    m, n, k = 300, 200, 8
    U = _orthogonal(m, gen)
    V = _orthogonal(n, gen)
    s = torch.cat([torch.linspace(40, 20, k, dtype=DT), torch.linspace(1.0, 0.01, n - k, dtype=DT)])
    M = U[:, :n] @ torch.diag(s) @ V.T
    Vk = V[:, :k]
    Mk = U[:, :k] @ torch.diag(s[:k]) @ Vk.T

    def tan_theta(B, target):
        B, _ = torch.linalg.qr(B)
        c = torch.linalg.svdvals(target.T @ B).min()
        return math.sqrt(max(0.0, 1 - float(c) ** 2)) / float(c)

    for noise in [0.05, 0.01]:
        Q0 = Vk + noise * torch.randn(n, k, generator=gen, dtype=DT)   # warm start near V_k
        Q0 = Q0 / torch.linalg.vector_norm(Q0, dim=0)
        P, R, _, _ = O.power_iteration(M, Q0)
        t0 = tan_theta(Q0, Vk)
        t1 = tan_theta(P, U[:, :k])
        assert t1 <= float(s[k] / s[k - 1]) * t0 + 1e-12
        # P P^T M - M_k = -(I - PP^T) U_k S_k V_k^T + PP^T U_perp S_perp V_perp^T, so
        # |.|_F <= sin(theta_1) (|S_k|_F + sqrt(k) s_{k+1})
        rel = float(torch.linalg.matrix_norm(P @ R.T - Mk) / torch.linalg.matrix_norm(Mk))
        sin1 = t1 / math.sqrt(1 + t1 * t1)
        skf = float(torch.linalg.vector_norm(s[:k]))
        assert rel <= sin1 * (1 + math.sqrt(k) * float(s[k]) / skf) + 1e-12
        if t0 <= 0.19:       # then tan(theta_1) <= 0.0095 and the 1-step error is <= 0.01
            assert rel <= 0.01


def test_power_iteration_steps_contract_the_subspace_angle_geometrically():
    """s steps of subspace iteration from Q_0 (each step restarting from the
    column-normalised R of the one before, which spans the same space as
    M^T P): tan(theta_s) <= (s_{k+1}/s_k)^s tan(theta_0), the textbook bound
    ([GRASP] ablation table: 1, 2 and 3 power-iteration steps). Also: two
    steps equal one step started from the normalised R of one step."""
    gen = torch.Generator().manual_seed(12)
    m, n, k = 200, 150, 6
    U = _orthogonal(m, gen)
    V = _orthogonal(n, gen)
    s = torch.cat([torch.linspace(10, 6, k, dtype=DT), torch.linspace(3.0, 0.1, n - k, dtype=DT)])
    M = U[:, :n] @ torch.diag(s) @ V.T
    Uk, Vk = U[:, :k], V[:, :k]

    def tan_theta(B, target):
        B, _ = torch.linalg.qr(B)
        c = torch.linalg.svdvals(target.T @ B).min()
        return math.sqrt(max(0.0, 1 - float(c) ** 2)) / float(c)

    Q0 = Vk + 0.4 * torch.randn(n, k, generator=gen, dtype=DT)
    Q0 = Q0 / torch.linalg.vector_norm(Q0, dim=0)
    t0 = tan_theta(Q0, Vk)
    ratio = float(s[k] / s[k - 1])
    prev = None
    for steps in (1, 2, 3):
        P, R, _, live = O.power_iteration(M, Q0, steps, seed=3, b=1)
        assert all(live)
        t = tan_theta(P, Uk)
        assert t <= ratio ** steps * t0 * (1 + 1e-9)
        if prev is not None:
            assert t < prev                     # each step gains
        prev = t
    P1, R1, _, _ = O.power_iteration(M, Q0, 1)
    P2, R2, _, _ = O.power_iteration(M, Q0, 2)
    Pc, Rc, _, _ = O.power_iteration(M, R1 / torch.linalg.vector_norm(R1, dim=0), 1)
    assert torch.allclose(P2, Pc, atol=1e-12) and torch.allclose(R2, Rc, atol=1e-11)


def test_residual_from_codes_bounds_the_rebuild_by_the_grid_half_step():
    """The residual-from-codes variant stores M_t - P^ R^T, so the next rebuild
    deq4 + P^ R^T misses M_t only by the 4-bit grid error: every element within
    half a code step s_ij / 14 (plus fp32 rounding of the residual). The
    worked step's own residual M_t - P R^T leaves the 8-bit factor error
    (P R^T - P^ R^T) in the rebuild on top, which this outlier input makes
    larger than the half step somewhere."""
    gen = torch.Generator().manual_seed(13)
    m, n, k = 256, 384, 8
    U = _orthogonal(m, gen)[:, :k]
    V = _orthogonal(n, gen)[:, :k]
    M = U @ torch.diag(torch.logspace(0, -1, k, dtype=DT)) @ V.T
    M = M + 1e-3 * torch.randn(m, n, generator=gen, dtype=DT)
    M[:, 5] *= 30.0
    st = O.zero_state(m, n, k)
    worst = {}
    for mode in ("codes", "exact"):
        r = O.grasp_step(st, torch.zeros(m, n), M.float(), mu=0.0, eta=0.0, seed=1, b=0,
                         residual=mode)
        M_t = r.M
        rebuilt = O.rebuild_momentum(r.state)
        s_ij = O.grid_scale_matrix(r.state.rscale, r.state.cscale, m, n).to(DT)
        excess = (rebuilt - M_t).abs() - s_ij / 14.0
        worst[mode] = float((excess / M_t.abs().max()).max())
    assert worst["codes"] <= 1e-6
    assert worst["exact"] > 1e-4


def test_warm_start_normalises_columns_and_uses_rademacher_for_zero_columns():
    Rh = torch.zeros(40, 3, dtype=DT)
    Rh[:, 0] = torch.arange(40, dtype=DT) - 20.0
    Q = O.warm_start(Rh, 5, 2)
    assert float(torch.linalg.vector_norm(Q[:, 0])) == pytest.approx(1.0, abs=1e-14)
    assert torch.allclose(Q[:, 0] * torch.linalg.vector_norm(Rh[:, 0]), Rh[:, 0])
    assert torch.equal(Q[:, 1], O.rademacher_column(5, 2, 40, 1))
    assert torch.equal(Q[:, 2], O.rademacher_column(5, 2, 40, 2))


# ------------------------------------------------------------- 4-bit grid

def test_grid_quant4_handworked_example():
    g = _read_sections(os.path.join(GOLDEN, "grid_quant4_handworked.txt"))
    bits = torch.tensor([[int(v, 16) for v in row] for row in g["X_bits_hex"]], dtype=torch.int64)
    X = bits.to(torch.int32).view(torch.float32)
    codes, rs, cs = O.grid_quant4(X, block=2)
    assert codes.tolist() == [[int(v) for v in row] for row in g["codes"]]
    assert torch.equal(rs, torch.tensor([[float(v) for v in r] for r in g["rscale"]], dtype=torch.float32))
    assert torch.equal(cs, torch.tensor([[float(v) for v in r] for r in g["cscale"]], dtype=torch.float32))
    packed = O.pack_nibbles(codes)
    assert packed.tolist() == [[int(v, 16) for v in row] for row in g["packed_hex"]]
    assert torch.equal(O.unpack_nibbles(packed), codes)


def test_grid_quant4_brute_force_codes():
    """q is the code minimising |x - (q/7) s| over all 16 nibble values; ties
    (equal distance) go to the even code."""
    gen = torch.Generator().manual_seed(12)
    for (m, n, blk) in [(8, 8, 4), (13, 22, 8), (130, 260, 128)]:
        X = (torch.randn(m, n, generator=gen) * torch.rand(m, 1, generator=gen) * 3).to(torch.float32)
        X[0, :] *= 50.0
        codes, rs, cs = O.grid_quant4(X, block=blk)
        s = O.grid_scale_matrix(rs, cs, m, n, blk)
        r = (X / torch.where(s > 0, s, torch.ones_like(s))) * torch.tensor(7.0)   # fp32 ratio
        cand = torch.arange(-8, 8, dtype=torch.float32)
        dist = (r.unsqueeze(-1) - cand).abs()
        best = dist.min(dim=-1).values
        chosen = dist.gather(-1, (codes.to(torch.int64) + 8).unsqueeze(-1)).squeeze(-1)
        assert torch.all(chosen[s > 0] == best[s > 0])
        ties = (dist == best.unsqueeze(-1)).sum(-1) > 1
        assert torch.all(codes[ties & (s > 0)] % 2 == 0)
        # half-step error bound |x - x^| <= s/14 (plus fp32 rounding)
        xh = O.grid_dequant4(codes, rs, cs, blk)
        err = (X.double() - xh).abs()
        assert torch.all(err <= s.double() / 14 * (1 + 1e-6) + 1e-30)


@pytest.mark.parametrize("m,n,blk", [(13, 22, 8), (21, 10, 4), (9, 9, 16)])
def test_grid_scales_brute_force_ragged(m, n, blk):
    """Element by element with plain loops, on ragged edge blocks: s_ij is the
    smaller of |x| maxima over row i and over column j, each taken only inside
    the block that holds (i, j) ("Achieving low-bit Muon through subspace
    preservation and grid quantization", key design 2); the oracle's row and
    column scales and its per-element scale must match, and its dequantized
    value must lie within half a step s_ij / 14 of x."""
    gen = torch.Generator().manual_seed(20 + m * n)
    X = (torch.randn(m, n, generator=gen) * torch.rand(1, n, generator=gen)).to(torch.float32)
    X[m - 1, :] = 0.0
    codes, rs, cs = O.grid_quant4(X, block=blk)
    s_or = O.grid_scale_matrix(rs, cs, m, n, blk)
    xh = O.grid_dequant4(codes, rs, cs, blk)
    for i in range(m):
        bi0 = (i // blk) * blk
        for j in range(n):
            bj0 = (j // blk) * blk
            r = max(abs(float(X[i, c])) for c in range(bj0, min(n, bj0 + blk)))
            c = max(abs(float(X[a, j])) for a in range(bi0, min(m, bi0 + blk)))
            assert float(rs[i, j // blk]) == r
            assert float(cs[i // blk, j]) == c
            s = min(r, c)
            assert float(s_or[i, j]) == s
            assert abs(float(X[i, j]) - float(xh[i, j])) <= s / 14 * (1 + 1e-6)


def test_grid_quant4_invariants():
    gen = torch.Generator().manual_seed(13)
    m, n, blk = 256, 384, 128
    X = torch.randn(m, n, generator=gen).to(torch.float32)
    X[128:256, 0:128] = 0.0                         # one zero block
    codes, rs, cs = O.grid_quant4(X, block=blk)
    assert torch.all(codes[128:256, 0:128] == 0)
    assert codes.abs().max() <= 7
    for bi in range(2):
        for bj in range(3):
            blkc = codes[bi * blk:(bi + 1) * blk, bj * blk:(bj + 1) * blk]
            blkx = X[bi * blk:(bi + 1) * blk, bj * blk:(bj + 1) * blk]
            nz_rows = blkx.abs().amax(dim=1) > 0
            nz_cols = blkx.abs().amax(dim=0) > 0
            # each nonzero row and column of a block holds a +-7 code (its absmax)
            assert torch.all((blkc.abs() == 7).any(dim=1)[nz_rows])
            assert torch.all((blkc.abs() == 7).any(dim=0)[nz_cols])


@pytest.mark.parametrize("m,n,group", [(5, 50, 128), (4, 64, 128), (3, 7, 4)])
def test_group_quant4_by_explicit_loops(m, n, group):
    """4bit-Muon-base codec, element by element: the scale of an element is
    the largest |x| among the `group` consecutive row-major elements of its
    group (a shorter last group), and its code is the one of the 16 nibble
    values nearest x / s * 7 (ties to the even code, 0 for a zero group)."""
    gen = torch.Generator().manual_seed(30 + m * n)
    X = (torch.randn(m, n, generator=gen) * torch.rand(m, 1, generator=gen)).to(torch.float32)
    X.view(-1)[:group] = 0.0                         # one all-zero group
    codes, scales = O.group_quant4(X, group=group)
    xh = O.group_dequant4(codes, scales, group=group)
    flat = X.reshape(-1)
    total = flat.numel()
    assert scales.numel() == -(-total // group)
    for e in range(total):
        g0 = (e // group) * group
        s = max(abs(float(flat[i])) for i in range(g0, min(total, g0 + group)))
        assert float(scales[e // group]) == s
        q = int(codes.reshape(-1)[e])
        if s == 0.0:
            assert q == 0 and float(xh.reshape(-1)[e]) == 0.0
            continue
        r = float(torch.tensor(float(flat[e]), dtype=torch.float32) / torch.tensor(s, dtype=torch.float32)
                  * torch.tensor(7.0, dtype=torch.float32))
        d = [abs(r - c) for c in range(-8, 8)]
        best = min(d)
        assert d[q + 8] == best
        if d.count(best) > 1:
            assert q % 2 == 0
        assert abs(float(flat[e]) - float(xh.reshape(-1)[e])) <= s / 14 * (1 + 1e-6)


def test_mulaw_function_inverse_and_endpoints():
    """The textbook mu-law pair: F maps [-1, 1] onto itself, odd and
    increasing, F(0) = 0, F(+-1) = +-1, and F^-1 undoes it."""
    x = torch.linspace(-1, 1, 2001, dtype=DT)
    y = O.mulaw_compress(x)
    assert float(y[0]) == pytest.approx(-1.0, abs=1e-15) and float(y[-1]) == pytest.approx(1.0, abs=1e-15)
    assert float(O.mulaw_compress(torch.zeros(1, dtype=DT))) == 0.0
    assert torch.all(y[1:] > y[:-1])
    assert torch.allclose(y, -O.mulaw_compress(-x), atol=0, rtol=0)
    assert float((O.mulaw_expand(y) - x).abs().max()) < 1e-14
    # mu = 255 at x = 0.5: ln(128.5) / ln(256)
    assert float(O.mulaw_compress(torch.tensor([0.5]))) == pytest.approx(math.log(128.5) / math.log(256))


def test_mulaw_codes_by_brute_force_and_small_mu_limit():
    """Each code is the nibble nearest 7 F(x / s) (ties to even); as mu -> 0,
    F -> identity and the codec becomes the uniform group codec."""
    gen = torch.Generator().manual_seed(50)
    X = (torch.randn(16, 64, generator=gen) * torch.rand(16, 1, generator=gen)).to(torch.float32)
    codes, scales = O.mulaw_quant4(X)
    s = scales.to(DT).repeat_interleave(128).view(X.shape)
    target = 7.0 * O.mulaw_compress(X.to(DT) / s)
    cand = torch.arange(-8, 8, dtype=DT)
    dist = (target.unsqueeze(-1) - cand).abs()
    best = dist.min(dim=-1).values
    chosen = dist.gather(-1, (codes.to(torch.int64) + 8).unsqueeze(-1)).squeeze(-1)
    assert torch.all(chosen == best)
    cu, su = O.group_quant4(X)
    cm, sm = O.mulaw_quant4(X, mu=1e-9)
    assert torch.equal(su, sm)
    diff = (cu.int() - cm.int()).abs()
    assert int(diff.max()) <= 1 and float((diff > 0).double().mean()) <= 1e-3


@pytest.mark.parametrize("dist", ["gauss", "student3"])
def test_mulaw_finer_in_the_dense_region(dist):
    """MuonQ's abstract: mu-law companding gives more resolution where momentum
    values are dense. Below the median magnitude its mean error is lower than
    the uniform group codec's, on Gaussian and on heavy-tailed data."""
    gen = torch.Generator().manual_seed(51)
    if dist == "gauss":
        X = torch.randn(128, 256, generator=gen)
    else:                                   # Student-t, 3 degrees of freedom
        z = torch.randn(128, 256, generator=gen, dtype=DT)
        chi2 = (torch.randn(3, 128, 256, generator=gen, dtype=DT) ** 2).sum(0)
        X = (z / torch.sqrt(chi2 / 3)).float()
    dense = X.abs() <= X.abs().median()
    cu, su = O.group_quant4(X)
    cm, sm = O.mulaw_quant4(X)
    eu = (O.group_dequant4(cu, su) - X.double()).abs()
    em = (O.mulaw_dequant4(cm, sm) - X.double()).abs()
    xn = float(X.double().norm())
    sweep = []
    for mu in (15.0, 63.0):
        c, sc = O.mulaw_quant4(X, mu=mu)
        sweep.append(float((O.mulaw_dequant4(c, sc, mu=mu) - X.double()).norm()) / xn)
    print(f"\n[{dist}] mean |error| below the median: uniform {float(eu[dense].mean()):.3f}, "
          f"mu-law {float(em[dense].mean()):.3f}; relative error: uniform {float(eu.norm()) / xn:.3f}, "
          f"mu = 15 / 63 / 255: {sweep[0]:.3f} / {sweep[1]:.3f} / {float(em.norm()) / xn:.3f}")
    assert float(em[dense].mean()) < 0.8 * float(eu[dense].mean())


def _low_rank_plus_outliers(m, n, r, seed, noise=0.05, outlier=10.0):
    """Synthetic momentum: rank-r part with singular values from 1 down to
    10^-1.5, a Gaussian floor, and 1 % of rows and of columns scaled by 10."""
    g = torch.Generator().manual_seed(seed)
    U, _ = torch.linalg.qr(torch.randn(m, r, generator=g, dtype=DT))
    V, _ = torch.linalg.qr(torch.randn(n, r, generator=g, dtype=DT))
    s = torch.logspace(0, -1.5, r, dtype=DT)
    M = U @ torch.diag(s) @ V.T + noise * torch.randn(m, n, generator=g, dtype=DT) / math.sqrt(n)
    M[torch.randperm(m, generator=g)[: max(1, m // 100)], :] *= outlier
    M[:, torch.randperm(n, generator=g)[: max(1, n // 100)]] *= outlier
    return M


def test_error_amplification_findings_on_synthetic_momentum():
    """The diagnosis of "Achieving low-bit Muon through subspace preservation
    and grid quantization", checked on the oracle's codecs with a synthetic
    low-rank-plus-outlier momentum (the note's own numbers come from trained
    models and are not reproduced; relative Frobenius errors throughout):

    * NS amplifies the error of direct 4-bit quantization (motivation: 0.07
      before NS, 1.78 after);
    * error in the top singular subspace is amplified more than error in the
      residual (entry angle, second diagnosis: about 40x against 5x);
    * without the top subspace, grid quantization leaves at most half the
      error of group quantization (key design 2, ablation: "halves the loss");
    * the full GRASP codec (top subspace kept, grid 4-bit residual) leaves far
      less error after NS than direct quantization (key design 2, last
      paragraph: 0.14 against 1.78 at rank 1/16)."""
    m, n = 256, 512
    k = min(m, n) // 16
    M = _low_rank_plus_outliers(m, n, 64, 3)
    Mf = M.float()
    NSM = O.ns_standard(M)

    def rel(a, b):
        return float(torch.linalg.matrix_norm(a - b) / torch.linalg.matrix_norm(b))

    def base(X):
        c, s = O.group_quant4(X.float())
        return O.group_dequant4(c, s)

    Mb = base(M)
    before, after = rel(Mb, M), rel(O.ns_standard(Mb), NSM)
    assert after >= 2.0 * before

    U, S, Vh = torch.linalg.svd(M, full_matrices=False)
    Mtop = U[:, :k] @ torch.diag(S[:k]) @ Vh[:k]
    Mres = M - Mtop
    qt, qr = base(Mtop), base(Mres)
    amp_top = rel(O.ns_standard(qt + Mres), NSM) / rel(qt, Mtop)
    amp_res = rel(O.ns_standard(Mtop + qr), NSM) / rel(qr, Mres)
    assert amp_top > amp_res > 1.0

    q4, rs, cs = O.grid_quant4(Mf)
    grid = O.grid_dequant4(q4, rs, cs)
    Mf64 = Mf.double()
    assert rel(grid, Mf64) <= 0.5 * rel(base(Mf64), Mf64)

    r = O.grasp_step(O.zero_state(m, n, k), torch.zeros(m, n), Mf, mu=0.0, eta=0.0)
    Mh = O.rebuild_momentum(r.state)
    ne_grasp = rel(O.ns_standard(Mh), O.ns_standard(r.M))
    ne_base = rel(O.ns_standard(base(r.M)), O.ns_standard(r.M))
    print(f"\n[{m}x{n}, k={k}] direct 4-bit: {before:.3f} before NS, {after:.3f} after; "
          f"amplification top {amp_top:.2f}x, residual {amp_res:.2f}x; grid {rel(grid, Mf64):.3f} vs "
          f"group {rel(base(Mf64), Mf64):.3f} before NS; GRASP {rel(Mh, r.M):.3f} before, NE "
          f"{ne_grasp:.3f} after (direct {ne_base:.3f})")
    assert ne_grasp <= 0.5 * ne_base


# ------------------------------------------------------------ 8-bit factors

def test_quant8_brute_force_and_bounds():
    gen = torch.Generator().manual_seed(14)
    X = (torch.randn(333, 7, generator=gen) * torch.logspace(-4, 1, 7)).to(torch.float32)
    X[:, 3] = 0.0
    codes, s = O.quant8(X)
    assert s[3] == 0 and torch.all(codes[:, 3] == 0)
    for l in [0, 1, 2, 4, 5, 6]:
        i = int(X[:, l].abs().argmax())
        assert abs(int(codes[i, l])) == 127
    safe = torch.where(s > 0, s, torch.ones_like(s))
    r = (X / safe) * torch.tensor(127.0)
    cand = torch.arange(-128, 128, dtype=torch.float32)
    for l in [0, 5]:
        dist = (r[:, l].unsqueeze(-1) - cand).abs()
        best = dist.min(dim=-1).values
        chosen = dist.gather(-1, (codes[:, l].to(torch.int64) + 128).unsqueeze(-1)).squeeze(-1)
        assert torch.all(chosen == best)
    err = (X.double() - O.dequant8(codes, s)).abs()
    assert torch.all(err <= s.double() / 254 * (1 + 1e-6))


# ------------------------------------------------------------ the full step

def test_step_zero_gradient_zero_state_stays_zero():
    st = O.zero_state(64, 96, 4, block=32)
    W = torch.zeros(64, 96)
    r = O.grasp_step(st, W, torch.zeros(64, 96), mu=0.95, eta=0.02, block=32)
    assert torch.all(r.M == 0) and torch.all(r.P == 0) and torch.all(r.R == 0)
    assert torch.all(r.state.codes4 == 0) and torch.all(r.state.P8 == 0)
    assert torch.all(r.O == 0) and torch.all(r.W == 0)


def test_step_mu_zero_momentum_is_gradient_and_k_full_is_lossless():
    gen = torch.Generator().manual_seed(15)
    m, n = 48, 80
    G = torch.randn(m, n, generator=gen) * 1e-3
    st = O.zero_state(m, n, 4, block=16)
    st.codes4 = torch.randint(0, 255, (m, n // 2), generator=gen, dtype=torch.uint8)
    st.rscale = torch.rand(st.rscale.shape, generator=gen)
    st.cscale = torch.rand(st.cscale.shape, generator=gen)
    r = O.grasp_step(st, torch.zeros(m, n), G, mu=0.0, eta=0.0, block=16)
    assert torch.equal(r.M, G.double())
    st2 = O.zero_state(m, n, m, block=16)
    r2 = O.grasp_step(st2, torch.zeros(m, n), G, mu=0.9, eta=0.0, block=16)
    assert float(torch.linalg.matrix_norm(r2.residual)) < 1e-12 * float(torch.linalg.matrix_norm(r2.M))


def test_step_momentum_is_undamped_heavy_ball():
    """Muon's momentum M_t = mu M_{t-1} + G_t ("Achieving low-bit Muon through
    subspace preservation and grid quantization", worked step 3) carries no
    (1 - mu) damping on the gradient. From a fixed non-zero state, M is
    therefore affine in G with unit slope and, at G = 0, linear in mu: a
    damped EMA or swapped operands break one of the two."""
    gen = torch.Generator().manual_seed(18)
    m, n, k = 32, 64, 4
    st = O.zero_state(m, n, k, block=16)
    st.codes4 = torch.randint(0, 255, (m, n // 2), generator=gen, dtype=torch.uint8)
    st.rscale = torch.rand(st.rscale.shape, generator=gen)
    st.cscale = torch.rand(st.cscale.shape, generator=gen)
    st.P8 = torch.randint(-127, 128, (m, k), generator=gen, dtype=torch.int8)
    st.R8 = torch.randint(-127, 128, (n, k), generator=gen, dtype=torch.int8)
    st.Pscale, st.Rscale = torch.rand(k, generator=gen), torch.rand(k, generator=gen)
    G = torch.randn(m, n, generator=gen)
    Z = torch.zeros(m, n)

    def M(mu, g):
        return O.grasp_step(st, Z, g, mu=mu, eta=0.0, block=16).M

    M1 = M(1.0, Z)
    assert float(M1.abs().max()) > 0.1
    assert float((M(0.9, G) - M(0.9, Z) - G.double()).abs().max()) <= 1e-12
    assert float((M(0.9, Z) - 0.9 * M1).abs().max()) <= 1e-12
    assert float((M(0.0, G) - G.double()).abs().max()) == 0.0


def test_step_warm_start_takes_the_stored_right_factor():
    """The warm start of step t is built from the stored R_{t-1} (the right
    factor, n x k), not P_{t-1} ("Achieving low-bit Muon through subspace
    preservation and grid quantization", worked step 2). Step 1 stores the
    exact factors of a square rank-k momentum U S V^T. Step 2 adds the gradient
    X S' U^T, with U, V, X mutually orthogonal k-frames, so M_2 = U S V^T +
    X S' U^T. One power iteration from Q ~ V gives M_2 Q ~ U S: P spans U.
    From Q ~ U (the left factor) it would give M_2 Q ~ X S': P would span X."""
    gen = torch.Generator().manual_seed(19)
    n, k = 64, 4
    Qo = _orthogonal(n, gen)
    U, V, X = Qo[:, :k], Qo[:, k:2 * k], Qo[:, 2 * k:3 * k]
    S = torch.diag(torch.tensor([0.4, 0.3, 0.2, 0.1], dtype=DT))
    Z = torch.zeros(n, n)
    r1 = O.grasp_step(O.zero_state(n, n, k, block=16), Z, U @ S @ V.T, mu=0.95, eta=0.0,
                      block=16)
    assert float(torch.linalg.matrix_norm(r1.residual)) < 1e-12
    r2 = O.grasp_step(r1.state, Z, X @ (0.3 * S) @ U.T, mu=1.0, eta=0.0, block=16)
    off = float(torch.linalg.matrix_norm(r2.P - U @ (U.T @ r2.P)))
    assert off < 0.05, off
    assert float(torch.linalg.matrix_norm(U.T @ r2.P)) > 0.99 * math.sqrt(k)


@pytest.mark.parametrize("m,n", [(96, 48), (48, 96)])
@pytest.mark.parametrize("ns", ["standard", "gram"])
def test_step_weight_update_closed_form_on_rank_one_gradient(m, n, ns):
    """From a zero state, M_1 = G. For G = sigma u v^T (unit u, v) the
    Frobenius norm is sigma, so NS sees one singular value s = sigma /
    (sigma + eps) and, by Proposition 1 of the Gram Newton-Schulz page,
    returns f(s) u v^T with f the composed scalar quintic. The update
    W <- W - eta (O + wd W) of "Achieving low-bit Muon through subspace
    preservation and grid quantization" (worked step 6) then has the closed
    form (1 - eta wd) W - eta f(s) u v^T: a flipped sign, a missing eta on the
    decay term or a mis-oriented O for a tall matrix all break it."""
    gen = torch.Generator().manual_seed(17)
    u = torch.randn(m, generator=gen, dtype=DT)
    v = torch.randn(n, generator=gen, dtype=DT)
    u, v = u / u.norm(), v / v.norm()
    sigma, eta, wd = 0.37, 0.02, 0.1
    G = sigma * torch.outer(u, v)
    W = torch.randn(m, n, generator=gen, dtype=DT)
    r = O.grasp_step(O.zero_state(m, n, 4, block=16), W, G, mu=0.95, eta=eta, wd=wd,
                     ns=ns, block=16)
    f = O.quintic_scalar(sigma / (sigma + O.NS_EPS))
    assert 0.5 < f < 1.5
    want = (1 - eta * wd) * W - eta * f * torch.outer(u, v)
    assert float((r.W - want).abs().max()) <= 1e-12
    assert float((r.O - f * torch.outer(u, v)).abs().max()) <= 1e-10


def test_step_rebuild_roundtrip():
    """After a step, rebuilding from the new state reproduces M_t up to the
    codes' half-step bounds: |M - M^| <= s/14 + 8-bit factor error."""
    gen = torch.Generator().manual_seed(16)
    m, n, k = 64, 128, 4
    G = torch.randn(m, n, generator=gen) * 1e-3
    G[3, :] *= 10
    G[:, 7] *= 10
    st = O.zero_state(m, n, k, block=32)
    r = O.grasp_step(st, torch.zeros(m, n), G, mu=0.95, eta=0.02, block=32)
    Mh = O.rebuild_momentum(r.state, block=32)
    rel = float(torch.linalg.matrix_norm(Mh - r.M) / torch.linalg.matrix_norm(r.M))
    assert rel < 0.1
    top = O.dequant8(r.state.P8, r.state.Pscale) @ O.dequant8(r.state.R8, r.state.Rscale).T
    rel_top = float(torch.linalg.matrix_norm(top - r.P @ r.R.T) / torch.linalg.matrix_norm(r.P @ r.R.T))
    assert rel_top < 0.02
