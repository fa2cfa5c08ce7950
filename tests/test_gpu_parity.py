"""CUDA path vs the fp64 oracle, element by element, on seeded inputs.

Tolerances (from the acceptance bar of the method's fixed reading):
* codes: bit-exact when both sides see identical fp32 inputs; when the GPU
  forms the residual itself (fp32 FMA vs the oracle's fp64), codes may differ
  by one step in at most 1e-4 of the elements (rounding-boundary ties);
* dequantized M, P, R: relative Frobenius error <= 1e-5;
* NS output: relative Frobenius error <= 2e-2 vs fp64 NS (bf16 standard NS,
  fp16 Gram NS).
Sizes span several 128-tiles and a ragged tail (144 = 128 + 16, 272 = 2*128 + 16).
"""

import pytest
import torch

import oracle as O
from bit_muon_optimizer_b200 import workloads as WL

pytestmark = pytest.mark.gpu

DEV = "cuda"


def rel(a, b):
    a, b = a.double().cpu(), b.double().cpu()
    return float((a - b).norm() / b.norm())


def _outlier_matrix(B, m, n, seed, std=1e-3, dtype=torch.float32):
    X = WL.random_matrix((B, m, n), seed, std=std)
    g = torch.Generator().manual_seed(seed + 1)
    for b in range(B):
        rows = torch.randperm(m, generator=g)[:2]
        cols = torch.randperm(n, generator=g)[:2]
        X[b, rows, :] *= 10
        X[b, :, cols] *= 10
    return X.to(dtype)


# ------------------------------------------------------------------ codec

@pytest.mark.parametrize("B,m,n", [(1, 256, 512), (3, 144, 272), (2, 128, 128), (1, 16, 48)])
def test_grid_quant4_bit_exact(cuda_lib, B, m, n):
    gm = cuda_lib
    X = _outlier_matrix(B, m, n, 100 + m)
    if m >= 144:
        X[0, 128:, :128] = 0.0                          # an all-zero ragged block
    codes, rs, cs = gm.grid_quant4(X.to(DEV))
    torch.cuda.synchronize()
    for b in range(B):
        q, r, c = O.grid_quant4(X[b])
        assert torch.equal(codes[b].cpu(), O.pack_nibbles(q)), f"codes differ in matrix {b}"
        assert torch.equal(rs[b].cpu(), r)
        assert torch.equal(cs[b].cpu(), c)


def test_grid_quant4_handworked_layout(cuda_lib):
    """A 16 x 16 matrix quantized in one block: zero block scales -> zero codes,
    and the packed byte layout (low nibble = even column)."""
    gm = cuda_lib
    X = torch.zeros(1, 16, 16)
    X[0, 0, 0], X[0, 0, 1], X[0, 1, 0] = 1.0, -0.5, 0.25
    codes, rs, cs = gm.grid_quant4(X.to(DEV))
    q, r, c = O.grid_quant4(X[0])
    assert torch.equal(codes[0].cpu(), O.pack_nibbles(q))
    assert int(codes[0, 0, 0]) == (7 & 0xF) | ((-7 & 0xF) << 4)


@pytest.mark.parametrize("k", [8, 32])
def test_grid_quant4_fused_residual(cuda_lib, k):
    gm = cuda_lib
    B, m, n = 2, 272, 400
    X = _outlier_matrix(B, m, n, 7)
    P = WL.random_matrix((B, m, k), 8) * 0.05
    R = WL.random_matrix((B, n, k), 9) * 0.05
    codes, rs, cs = gm.grid_quant4(X.to(DEV), P.to(DEV), R.to(DEV))
    torch.cuda.synchronize()
    for b in range(B):
        res = (X[b].double() - P[b].double() @ R[b].double().T).float()
        q, r, c = O.grid_quant4(res)
        got = O.unpack_nibbles(codes[b].cpu())
        diff = (got.int() - q.int()).abs()
        assert int(diff.max()) <= 1
        assert float((diff > 0).double().mean()) <= 1e-4
        assert rel(rs[b], r) < 1e-6 and rel(cs[b], c) < 1e-6


@pytest.mark.parametrize("rows,k", [(256, 8), (2048, 16), (777, 3), (18944, 32)])
def test_quant8_bit_exact(cuda_lib, rows, k):
    gm = cuda_lib
    X = WL.random_matrix((2, rows, k), rows + k) * torch.logspace(-3, 0, k)
    X[1, :, 0] = 0.0
    codes, scale = gm.quant8(X.to(DEV))
    for b in range(2):
        q, s = O.quant8(X[b])
        assert torch.equal(codes[b].cpu(), q)
        assert torch.equal(scale[b].cpu(), s)


def _random_state(B, m, n, k, seed):
    g = torch.Generator().manual_seed(seed)
    mb, nb = -(-m // 128), -(-n // 128)
    return dict(
        codes4=torch.randint(0, 256, (B, m, n // 2), generator=g, dtype=torch.uint8),
        rscale=torch.rand((B, m, nb), generator=g) * 1e-2,
        cscale=torch.rand((B, mb, n), generator=g) * 1e-2,
        P8=torch.randint(-127, 128, (B, m, k), generator=g, dtype=torch.int8),
        Pscale=torch.rand((B, k), generator=g),
        R8=torch.randint(-127, 128, (B, n, k), generator=g, dtype=torch.int8),
        Rscale=torch.rand((B, k), generator=g) * 1e-2,
    )


@pytest.mark.parametrize("B,m,n,k", [(2, 256, 512, 8), (1, 144, 272, 32), (3, 128, 384, 16)])
def test_dequant_rebuild(cuda_lib, B, m, n, k):
    gm = cuda_lib
    s = _random_state(B, m, n, k, 11)
    d = {key: v.to(DEV) for key, v in s.items()}
    M = gm.dequant_rebuild(d["codes4"], d["rscale"], d["cscale"], d["P8"], d["Pscale"], d["R8"],
                           d["Rscale"])
    for b in range(B):
        st = O.GraspState(s["codes4"][b], s["rscale"][b], s["cscale"][b], s["P8"][b],
                          s["Pscale"][b], s["R8"][b], s["Rscale"][b])
        assert rel(M[b], O.rebuild_momentum(st)) <= 1e-6


# ------------------------------------------------------------ power iteration

@pytest.mark.parametrize("B,m,n,k,warm", [(2, 256, 512, 8, False), (2, 512, 256, 8, True),
                                          (1, 144, 272, 32, True), (1, 768, 2048, 16, True)])
def test_momentum_powerit(cuda_lib, B, m, n, k, warm):
    gm = cuda_lib
    G = _outlier_matrix(B, m, n, 21, dtype=torch.bfloat16)
    Mp = _outlier_matrix(B, m, n, 22)
    Rp = WL.random_matrix((B, n, k), 23) if warm else None
    M, P, R = gm.momentum_powerit(G.to(DEV), k, mu=0.95, M_prev=Mp.to(DEV),
                                  R_prev=Rp.to(DEV) if warm else None, seed=1234)
    torch.cuda.synchronize()
    for b in range(B):
        Mo = 0.95 * Mp[b].double() + G[b].double()
        Rh = Rp[b].double() if warm else torch.zeros(n, k, dtype=torch.float64)
        Q = O.warm_start(Rh, 1234, b)
        Po, Ro, _, live = O.power_iteration(Mo, Q)
        assert all(live)
        assert rel(M[b], Mo) <= 1e-6
        assert rel(P[b], Po) <= 1e-5
        assert rel(R[b], Ro) <= 1e-5


def test_powerit_dead_columns(cuda_lib):
    """Rank-deficient M Q: dead columns are zero in P and R on both sides."""
    gm = cuda_lib
    m, n, k = 256, 384, 8
    U = WL.random_matrix((m, 3), 31, dtype=torch.float64)
    V = WL.random_matrix((n, 3), 32, dtype=torch.float64)
    Mo = (U @ V.T) * 1e-3                                   # exact rank 3
    G = Mo.float().unsqueeze(0)
    M, P, R = gm.momentum_powerit(G.to(DEV), k, mu=0.0, seed=5)
    Q = O.warm_start(torch.zeros(n, k, dtype=torch.float64), 5, 0)
    Po, Ro, _, live = O.power_iteration(G[0].double(), Q)
    assert sum(live) == 3
    for l in range(k):
        if not live[l]:
            assert float(P[0, :, l].abs().max()) == 0.0
    assert rel(P[0], Po) <= 1e-5 and rel(R[0], Ro) <= 1e-5


# --------------------------------------------------------------- Newton-Schulz

# multiples of 256, ragged 256-row pair tiles (384, 320: a 128-row half entirely
# outside the matrix or a 64-row box at the edge), a single 64-row block, and
# shapes that the chains zero-pad to multiples of 64 (144 x 400)
NS_SHAPES = [(2, 256, 512), (2, 512, 256), (1, 384, 384), (1, 320, 640), (3, 64, 192),
             (2, 144, 400), (1, 768, 2048)]


@pytest.mark.parametrize("B,m,n", NS_SHAPES)
def test_newton_schulz_vs_oracle(cuda_lib, B, m, n):
    gm = cuda_lib
    X = _outlier_matrix(B, m, n, 41)
    Og = gm.newton_schulz(X.to(DEV))
    for b in range(B):
        assert rel(Og[b], O.ns_standard(X[b].double())) <= 2e-2


@pytest.mark.parametrize("abc", [[(1.0, 0.0, 0.0)], [(0.0, 1.0, 0.0)], [(0.0, 0.0, 1.0)],
                                 [(0.5, -0.25, 0.125)]])
@pytest.mark.parametrize("B,m,n", [(2, 256, 512), (1, 400, 144)])
def test_newton_schulz_single_terms(cuda_lib, abc, B, m, n):
    """One NS step with one term at a time isolates the three products:
    a X (epilogue), b X X^T X (X X^T and the MN-major left product), c (XX^T)^2 X."""
    gm = cuda_lib
    X = WL.random_matrix((B, m, n), 43)
    Og = gm.newton_schulz(X.to(DEV), abc=abc, T=1)
    for b in range(B):
        assert rel(Og[b], O.ns_standard(X[b].double(), abc=abc, T=1)) <= 1e-2


def _conditioned_matrix(B, m, n, seed, smin=0.1):
    """U diag(s) V^T with random orthogonal frames and s spread evenly over
    [smin, 1]: a matrix whose Gram has no near-zero eigenvalue."""
    g = torch.Generator().manual_seed(seed)
    N = min(m, n)
    out = torch.empty(B, m, n)
    for b in range(B):
        U, _ = torch.linalg.qr(torch.randn(m, N, generator=g, dtype=torch.float64))
        V, _ = torch.linalg.qr(torch.randn(n, N, generator=g, dtype=torch.float64))
        s = torch.linspace(1.0, smin, N, dtype=torch.float64)
        out[b] = (U @ torch.diag(s) @ V.T).float() * 1e-2
    return out


@pytest.mark.parametrize("restart", [(2,), (1, 3), (1, 2, 3, 4), ()])
@pytest.mark.parametrize("B,m,n", NS_SHAPES)
def test_gram_ns_vs_oracle(cuda_lib, B, m, n, restart):
    """Stabilized Gram NS (restarts) within 2e-2 of fp64 NS on every shape. The
    restart-free (naive) form on a square matrix gets a well-conditioned input
    (singular values spread over [0.1, 1]): in half precision naive Gram NS is
    unstable when R has near-zero eigenvalues (Gram NS page, §3.1, Proposition
    2), which a square random matrix (sigma_min / sigma_max ~ 1e-5) has."""
    gm = cuda_lib
    if restart == () and m == n:
        X = _conditioned_matrix(B, m, n, 52)
    else:
        X = _outlier_matrix(B, m, n, 51)
    Og = gm.gram_ns(X.to(DEV), restart_after=restart)
    for b in range(B):
        ref = O.ns_standard(X[b].double())          # Gram NS equals NS in exact arithmetic
        assert rel(Og[b], ref) <= 2e-2


# Batches with more output tiles per product than the 74 CTA pairs of the
# persistent GEMM, so every pair walks several (matrix, tile) pairs: the
# accumulator double buffer flips, the operand ring wraps across tiles and
# the batch index advances inside one launch. 48 x 768^2: 288 lower-triangle
# tiles per symmetric product, 432 per left product; 8 x 768 x 2048: 192 left
# tiles; 160 x 256 x 512: 160 tiles of one matrix each.
MULTI_TILE = [(48, 768, 768), (8, 768, 2048), (160, 256, 512), (6, 2048, 768)]


@pytest.mark.parametrize("B,m,n", MULTI_TILE)
@pytest.mark.parametrize("form", ["standard", "gram"])
def test_ns_many_tiles_per_cta_pair(cuda_lib, B, m, n, form):
    gm = cuda_lib
    X = _outlier_matrix(B, m, n, 53)
    f = gm.gram_ns if form == "gram" else gm.newton_schulz
    Og = f(X.to(DEV)).cpu()
    torch.cuda.synchronize()
    for b in range(B):
        ref = O.gram_ns(X[b].double()) if form == "gram" else O.ns_standard(X[b].double())
        assert rel(Og[b], ref) <= 2e-2, f"matrix {b}"


# ----------------------------------------------------------------- full step

def _to_oracle_state(st, b):
    return O.GraspState(st.codes4[b].cpu(), st.rscale[b].cpu(), st.cscale[b].cpu(),
                        st.P8[b].cpu(), st.Pscale[b].cpu(), st.R8[b].cpu(), st.Rscale[b].cpu(),
                        int(st.step.item()))


def _run_teacher_forced(gm, cid, group, B, steps, ns, gdtype=None):
    w = WL.WORKLOADS[cid]
    g = w.groups[group]
    m, n, k = g.m, g.n, w.k
    base = w.group_base(group)
    nsmode = gm.GM_NS_GRAM if ns == "gram" else gm.GM_NS_STANDARD
    step = gm.GraspStep(B, m, n, k, mu=w.mu, eta=w.eta, wd=w.wd, T=w.T, ns=nsmode,
                        seed=w.seed, device=DEV)
    st = gm.GraspState.zeros(B, m, n, k, DEV)
    W = torch.stack([WL.initial_weight(w, base + b, m, n) for b in range(B)]).to(DEV)
    for t in range(1, steps + 1):
        G = torch.stack([WL.gradient(w, base + b, t, m, n) for b in range(B)]).to(DEV)
        if gdtype is not None:
            G = G.to(gdtype)
        before = [_to_oracle_state(st, b) for b in range(B)]
        W0 = W.clone()
        step(st, W, G)
        torch.cuda.synchronize()
        assert int(st.dev_status.item()) == 0
        assert int(st.step.item()) == t
        for b in range(B):
            r = O.grasp_step(before[b], W0[b].cpu(), G[b].cpu(), mu=w.mu, eta=w.eta, wd=w.wd,
                             seed=w.seed, b=b, ns=ns, T=w.T)
            assert rel(step.stage_M()[b], r.M) <= 1e-5
            assert rel(step.stage_P()[b], r.P) <= 1e-5
            assert rel(step.stage_R()[b], r.R) <= 1e-5
            # 8-bit codes: bit-exact on the GPU's own fp32 P and R
            q, s = O.quant8(step.stage_P()[b].cpu())
            assert torch.equal(st.P8[b].cpu(), q) and torch.equal(st.Pscale[b].cpu(), s)
            q, s = O.quant8(step.stage_R()[b].cpu())
            assert torch.equal(st.R8[b].cpu(), q) and torch.equal(st.Rscale[b].cpu(), s)
            # 4-bit codes: the GPU forms the residual in fp32
            got = O.unpack_nibbles(st.codes4[b].cpu())
            want = O.unpack_nibbles(r.state.codes4)
            diff = (got.int() - want.int()).abs()
            assert int(diff.max()) <= 1
            assert float((diff > 0).double().mean()) <= 1e-4
            # update direction recovered from W (wd = 0)
            Og = (W0[b].double() - W[b].double()).cpu() / w.eta
            assert rel(Og, r.O) <= 2e-2


def test_grasp_step_single_fp32_matrix(cuda_lib):
    """256 x 512 fp32 gradients, k = 8, 3 steps from a zero state."""
    _run_teacher_forced(cuda_lib, 1, 0, 1, 3, "standard")


@pytest.mark.parametrize("ns", ["standard", "gram"])
def test_grasp_step_llama130m_shapes(cuda_lib, ns):
    """2048 x 768 (tall) and 768 x 2048 gradients in bf16, k = 16."""
    _run_teacher_forced(cuda_lib, 2, 1, 2, 2, ns)
    _run_teacher_forced(cuda_lib, 2, 2, 1, 2, ns)


def test_grasp_step_fp16_gradients(cuda_lib):
    """fp16 gradients (the third gradient dtype of the C ABI), 768 x 2048, 2 steps."""
    _run_teacher_forced(cuda_lib, 2, 2, 2, 2, "standard", gdtype=torch.float16)


def test_grasp_step_nonfinite_leaves_state_and_weights(cuda_lib):
    gm = cuda_lib
    B, m, n, k = 2, 256, 512, 8
    step = gm.GraspStep(B, m, n, k, device=DEV)
    st = gm.GraspState.zeros(B, m, n, k, DEV)
    W = WL.random_matrix((B, m, n), 3).to(DEV)
    G = WL.random_matrix((B, m, n), 4, std=1e-3).to(DEV)
    step(st, W, G)
    torch.cuda.synchronize()
    snap = st.clone()
    W1 = W.clone()
    G[1, 5, 7] = float("nan")
    step(st, W, G)
    torch.cuda.synchronize()
    assert int(st.dev_status.item()) == gm.GM_E_NONFINITE
    assert torch.equal(W, W1)
    for a, b in zip(st.tensors(), snap.tensors()):
        if a is not st.dev_status:
            assert torch.equal(a, b)
    # the next finite step proceeds
    G[1, 5, 7] = 0.0
    step(st, W, G)
    torch.cuda.synchronize()
    assert int(st.dev_status.item()) == 0 and int(st.step.item()) == 2


def test_grasp_step_checkpoint_and_batch_consistency(cuda_lib):
    """5 steps straight == 2 steps, save/load, 3 steps (bit-exact); a batch of 3
    matrices == each matrix alone (bit-exact)."""
    gm = cuda_lib
    w = WL.WORKLOADS[2]
    m, n, k, B = 768, 768, 16, 3
    grads = [torch.stack([WL.gradient(w, b, t, m, n) for b in range(B)]).to(DEV) for t in range(1, 6)]
    W0 = torch.stack([WL.initial_weight(w, b, m, n) for b in range(B)]).to(DEV)

    def run(Bs, idx, st, W, ts):
        step = gm.GraspStep(Bs, m, n, k, seed=w.seed, device=DEV)
        for t in ts:
            step(st, W, grads[t][idx].contiguous())
        torch.cuda.synchronize()

    stA = gm.GraspState.zeros(B, m, n, k, DEV)
    WA = W0.clone()
    run(B, slice(0, B), stA, WA, range(5))
    stB = gm.GraspState.zeros(B, m, n, k, DEV)
    WB = W0.clone()
    run(B, slice(0, B), stB, WB, range(2))
    saved = {f: t.cpu() for f, t in zip("abcdefghi", stB.tensors())}
    stC = gm.GraspState(*[saved[f].to(DEV) for f in "abcdefghi"])
    WC = WB.cpu().to(DEV)
    run(B, slice(0, B), stC, WC, range(2, 5))
    assert torch.equal(WA, WC)
    for a, c in zip(stA.tensors(), stC.tensors()):
        assert torch.equal(a, c)
    # one matrix alone (its seed-index b differs, so compare the W of matrix 0 only)
    st1 = gm.GraspState.zeros(1, m, n, k, DEV)
    W1 = W0[0:1].clone()
    run(1, slice(0, 1), st1, W1, range(5))
    assert torch.equal(W1[0], WA[0])
    assert torch.equal(st1.codes4[0], stA.codes4[0])


@pytest.mark.parametrize("m,n,ns,k", [(144, 272, "standard", 8), (272, 144, "gram", 8),
                                      (256, 384, "standard", 12), (208, 336, "gram", 5)])
def test_grasp_step_ragged_shape(cuda_lib, m, n, ns, k):
    """The whole step at sizes that are not multiples of the 128-row grid
    blocks, the 64-row codec tiles or the NS tiles (144 = 128 + 16,
    272 = 2*128 + 16, 208, 336), wide and tall, and at ranks k that are not
    the factor widths 8, 16, 32 the MMA fragments are padded to, teacher-forced
    for two steps."""
    gm = cuda_lib
    B, mu, eta, seed = 2, 0.95, 0.02, 77
    nsmode = gm.GM_NS_GRAM if ns == "gram" else gm.GM_NS_STANDARD
    step = gm.GraspStep(B, m, n, k, mu=mu, eta=eta, ns=nsmode, seed=seed, device=DEV)
    st = gm.GraspState.zeros(B, m, n, k, DEV)
    W = WL.random_matrix((B, m, n), 41, std=0.02).to(DEV)
    for t in (1, 2):
        G = _outlier_matrix(B, m, n, 50 + t, dtype=torch.bfloat16).to(DEV)
        before = [_to_oracle_state(st, b) for b in range(B)]
        W0 = W.clone()
        step(st, W, G)
        torch.cuda.synchronize()
        assert int(st.dev_status.item()) == 0
        for b in range(B):
            r = O.grasp_step(before[b], W0[b].cpu(), G[b].cpu(), mu=mu, eta=eta, seed=seed,
                             b=b, ns=ns)
            assert rel(step.stage_M()[b], r.M) <= 1e-5
            assert rel(step.stage_P()[b], r.P) <= 1e-5
            assert rel(step.stage_R()[b], r.R) <= 1e-5
            q, s = O.quant8(step.stage_P()[b].cpu())
            assert torch.equal(st.P8[b].cpu(), q) and torch.equal(st.Pscale[b].cpu(), s)
            q, s = O.quant8(step.stage_R()[b].cpu())
            assert torch.equal(st.R8[b].cpu(), q) and torch.equal(st.Rscale[b].cpu(), s)
            assert torch.equal(st.rscale[b].cpu() > 0, r.state.rscale > 0)
            diff = (O.unpack_nibbles(st.codes4[b].cpu()).int()
                    - O.unpack_nibbles(r.state.codes4).int()).abs()
            assert int(diff.max()) <= 1 and int((diff > 0).sum()) <= 4
            Og = (W0[b].double() - W[b].double()).cpu() / eta
            assert rel(Og, r.O) <= 2e-2


@pytest.mark.parametrize("m,n", [(256, 512), (512, 256)])
@pytest.mark.parametrize("ns", ["standard", "gram"])
def test_grasp_step_weight_decay(cuda_lib, m, n, ns):
    """W <- W - eta (O + wd W). One step from a zero state with wd = 0.1 and
    with wd = 0: O and the new state depend only on the state and G, so the
    states match bit for bit and the updated weights differ by -eta wd W_0
    up to fp32 rounding (relative size ~1e-4 here). Wide and tall, both NS
    forms: the decay term sits in the epilogue of the last NS product."""
    gm = cuda_lib
    B, k, eta, wd = 2, 8, 0.02, 0.1
    nsmode = gm.GM_NS_GRAM if ns == "gram" else gm.GM_NS_STANDARD
    W0 = WL.random_matrix((B, m, n), 43, std=0.02).to(DEV)
    G = _outlier_matrix(B, m, n, 44, dtype=torch.bfloat16).to(DEV)
    out = {}
    for lam in (0.0, wd):
        step = gm.GraspStep(B, m, n, k, eta=eta, wd=lam, ns=nsmode, seed=3, device=DEV)
        st = gm.GraspState.zeros(B, m, n, k, DEV)
        W = W0.clone()
        step(st, W, G)
        torch.cuda.synchronize()
        assert int(st.dev_status.item()) == 0
        out[lam] = (W, st)
    (W_a, st_a), (W_b, st_b) = out[0.0], out[wd]
    for a, b in zip(st_a.tensors(), st_b.tensors()):
        assert torch.equal(a, b)
    assert rel(W_b - W_a, -eta * wd * W0) <= 1e-3


@pytest.mark.parametrize("odt", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("B,m,n,form", [(2, 256, 512, "standard"), (1, 400, 144, "gram")])
def test_ns_half_precision_outputs(cuda_lib, odt, B, m, n, form):
    """The NS entry points' 16-bit output dtypes (wide and tall, both forms):
    the same 2e-2 bar against fp64 NS, and the 16-bit output equal to the fp32
    output of the same call rounded to that dtype, up to one ulp of the fp32
    result's own rounding order."""
    gm = cuda_lib
    X = _outlier_matrix(B, m, n, 61).to(DEV)
    f = gm.gram_ns if form == "gram" else gm.newton_schulz
    O32 = f(X)
    O16 = f(X, out_dtype=odt)
    torch.cuda.synchronize()
    assert O16.dtype == odt
    for b in range(B):
        assert rel(O16[b], O.ns_standard(X[b].cpu().double())) <= 2e-2
    assert rel(O16, O32.to(odt)) <= 1e-2


@pytest.mark.parametrize("B,m,n", [(2, 256, 512), (3, 144, 272), (1, 16, 48)])
def test_group_codec_bit_exact(cuda_lib, B, m, n):
    """The 4bit-Muon-base codec (128 consecutive elements per absmax scale)
    against the oracle: codes and scales bit-exact, including a zero group and
    a group of exact rounding ties (s = 7, x = k + 1/2), which take the
    division path; the dequantized values within fp32 rounding."""
    gm = cuda_lib
    X = _outlier_matrix(B, m, n, 71)
    flat = X[0].view(-1)
    flat[:128] = 0.0
    ties = torch.tensor([7.0] + [k + 0.5 for k in range(-7, 7)], dtype=torch.float32)
    flat[128:256] = ties.repeat(10)[:128]
    codes, gs = gm.group_quant4(X.to(DEV))
    Xh = gm.group_dequant4(codes, gs)
    torch.cuda.synchronize()
    for b in range(B):
        q, s = O.group_quant4(X[b])
        assert torch.equal(codes[b].cpu(), O.pack_nibbles(q))
        assert torch.equal(gs[b].cpu(), s)
        assert rel(Xh[b], O.group_dequant4(q, s)) <= 1e-6
    assert float(gs[0, 0]) == 0.0 and int(codes[0].view(-1)[:64].abs().max()) == 0


def test_dequant_rebuild_residual_only(cuda_lib):
    """k = 0: gm_dequant_rebuild rebuilds the 4-bit residual alone (no factor
    arrays passed), at a ragged size."""
    gm = cuda_lib
    B, m, n = 2, 144, 272
    s = _random_state(B, m, n, 8, 12)
    M = gm.dequant_rebuild(s["codes4"].to(DEV), s["rscale"].to(DEV), s["cscale"].to(DEV))
    torch.cuda.synchronize()
    for b in range(B):
        want = O.grid_dequant4(O.unpack_nibbles(s["codes4"][b]), s["rscale"][b], s["cscale"][b])
        assert rel(M[b], want) <= 1e-6


@pytest.mark.parametrize("ns", ["standard", "gram"])
def test_grasp_step_zero_gradient(cuda_lib, ns):
    """The degenerate step: a zero gradient on a zero state gives M = 0, every
    power-iteration column dead (P = R = 0), zero codes and scales, O = 0, so
    W is unchanged bit for bit; twice, so the second step's warm start falls
    back to the Rademacher columns of an all-zero R."""
    gm = cuda_lib
    B, m, n, k = 2, 256, 512, 8
    nsmode = gm.GM_NS_GRAM if ns == "gram" else gm.GM_NS_STANDARD
    step = gm.GraspStep(B, m, n, k, ns=nsmode, seed=9, device=DEV)
    st = gm.GraspState.zeros(B, m, n, k, DEV)
    W = WL.random_matrix((B, m, n), 81, std=0.02).to(DEV)
    W0 = W.clone()
    G = torch.zeros((B, m, n), dtype=torch.bfloat16, device=DEV)
    for t in (1, 2):
        step(st, W, G)
        torch.cuda.synchronize()
        assert int(st.dev_status.item()) == 0 and int(st.step.item()) == t
    assert torch.equal(W, W0)
    for x in (st.codes4, st.rscale, st.cscale, st.P8, st.Pscale, st.R8, st.Rscale):
        assert int(torch.count_nonzero(x)) == 0
    assert int(torch.count_nonzero(step.stage_P())) == 0


# ------------------------------------------------- step options and halves

@pytest.mark.parametrize("power_steps,residual,ns", [(2, "exact", "standard"), (3, "exact", "gram"),
                                                     (1, "codes", "standard"), (2, "codes", "gram")])
def test_grasp_step_power_steps_and_residual_variant(cuda_lib, power_steps, residual, ns):
    """The ablation variants of the step ([GRASP] ablation table: 1/2/3
    power-iteration steps; the residual from the dequantized 8-bit factors),
    teacher-forced for two steps at a ragged wide and a tall size, with the
    matrices' Rademacher counter indices given explicitly (ids 5 and 11)."""
    gm = cuda_lib
    nsmode = gm.GM_NS_GRAM if ns == "gram" else gm.GM_NS_STANDARD
    ids = [5, 11]
    for m, n, k in ((144, 400, 8), (400, 144, 16)):
        B, seed = 2, 321
        step = gm.GraspStep(B, m, n, k, ns=nsmode, seed=seed, device=DEV, power_steps=power_steps,
                            residual_from_codes=residual == "codes", matrix_ids=ids)
        st = gm.GraspState.zeros(B, m, n, k, DEV)
        W = WL.random_matrix((B, m, n), 91, std=0.02).to(DEV)
        for t in (1, 2):
            G = _outlier_matrix(B, m, n, 90 + t, dtype=torch.bfloat16).to(DEV)
            before = [_to_oracle_state(st, b) for b in range(B)]
            W0 = W.clone()
            step(st, W, G)
            torch.cuda.synchronize()
            assert int(st.dev_status.item()) == 0
            for b in range(B):
                r = O.grasp_step(before[b], W0[b].cpu(), G[b].cpu(), mu=0.95, eta=0.02, seed=seed,
                                 b=ids[b], ns=ns, power_steps=power_steps, residual=residual)
                assert rel(step.stage_M()[b], r.M) <= 1e-5
                assert rel(step.stage_P()[b], r.P) <= 1e-5
                assert rel(step.stage_R()[b], r.R) <= 1e-5
                q, s = O.quant8(step.stage_P()[b].cpu())
                assert torch.equal(st.P8[b].cpu(), q) and torch.equal(st.Pscale[b].cpu(), s)
                q, s = O.quant8(step.stage_R()[b].cpu())
                assert torch.equal(st.R8[b].cpu(), q) and torch.equal(st.Rscale[b].cpu(), s)
                diff = (O.unpack_nibbles(st.codes4[b].cpu()).int()
                        - O.unpack_nibbles(r.state.codes4).int()).abs()
                assert int(diff.max()) <= 1 and float((diff > 0).double().mean()) <= 1e-4
                assert rel((W0[b].double() - W[b].double()).cpu() / 0.02, r.O) <= 2e-2


def test_grasp_step_halves_equal_the_step(cuda_lib):
    """gm_grasp_state_update followed by gm_grasp_apply is gm_grasp_step, bit for
    bit (state, weights and the stage buffers), over two steps."""
    gm = cuda_lib
    B, m, n, k = 3, 256, 640, 16
    W0 = WL.random_matrix((B, m, n), 95, std=0.02).to(DEV)
    grads = [_outlier_matrix(B, m, n, 96 + t, dtype=torch.bfloat16).to(DEV) for t in (1, 2)]
    runs = []
    for split in (False, True):
        step = gm.GraspStep(B, m, n, k, seed=4, device=DEV)
        st = gm.GraspState.zeros(B, m, n, k, DEV)
        W = W0.clone()
        for G in grads:
            if split:
                step.state_update(st, G)
                step.apply(st, W)
            else:
                step(st, W, G)
        torch.cuda.synchronize()
        runs.append((st, W, step.stage_M().clone(), step.stage_P().clone()))
    (sa, Wa, Ma, Pa), (sb, Wb, Mb, Pb) = runs
    assert torch.equal(Wa, Wb) and torch.equal(Ma, Mb) and torch.equal(Pa, Pb)
    for a, b in zip(sa.tensors(), sb.tensors()):
        assert torch.equal(a, b)


def test_grasp_apply_skips_after_a_nonfinite_state_update(cuda_lib):
    """A NaN in G: the state update flags GM_E_NONFINITE and leaves the state
    alone; the apply half then leaves W alone too."""
    gm = cuda_lib
    B, m, n, k = 1, 256, 256, 8
    step = gm.GraspStep(B, m, n, k, device=DEV)
    st = gm.GraspState.zeros(B, m, n, k, DEV)
    W = WL.random_matrix((B, m, n), 97, std=0.02).to(DEV)
    G = WL.random_matrix((B, m, n), 98, std=1e-3).to(DEV)
    G[0, 3, 3] = float("inf")
    W1 = W.clone()
    step.state_update(st, G)
    step.apply(st, W)
    torch.cuda.synchronize()
    assert int(st.dev_status.item()) == gm.GM_E_NONFINITE
    assert torch.equal(W, W1) and int(st.step.item()) == 0


@pytest.mark.parametrize("mu", [255.0, 15.0])
@pytest.mark.parametrize("B,m,n,dist", [(2, 256, 512, "gauss"), (3, 144, 272, "student"),
                                        (1, 16, 48, "gauss")])
def test_mulaw_codec_bit_exact(cuda_lib, mu, B, m, n, dist):
    """MuonQ's mu-law companding codec against the oracle's fp64 definition
    (codes = rint(7 F(x / s)), F the mu-law curve): codes and group scales bit
    for bit, including a zero group; the decoded values within fp32 rounding of
    the oracle's s F^-1(q / 7)."""
    gm = cuda_lib
    if dist == "gauss":
        X = _outlier_matrix(B, m, n, 81)
    else:
        g = torch.Generator().manual_seed(82)
        X = (torch.randn(B, m, n, generator=g)
             / torch.sqrt((torch.randn(3, B, m, n, generator=g) ** 2).sum(0) / 3.0)) * 1e-3
    X[0].view(-1)[:128] = 0.0
    codes, gs = gm.mulaw_quant4(X.to(DEV), mu=mu)
    Xh = gm.mulaw_dequant4(codes, gs, mu=mu)
    torch.cuda.synchronize()
    for b in range(B):
        q, s = O.mulaw_quant4(X[b], mu=mu)
        assert torch.equal(gs[b].cpu(), s)
        assert torch.equal(codes[b].cpu(), O.pack_nibbles(q)), f"codes differ in matrix {b}"
        assert rel(Xh[b], O.mulaw_dequant4(q, s, mu=mu)) <= 1e-6
    assert float(gs[0, 0]) == 0.0 and int(codes[0].view(-1)[:64].abs().max()) == 0
