"""Algorithmic FLOP and byte counts used for roofline reporting.

FLOP conventions follow "优化器 (3)（Gram Newton-Schulz）", §1.2 and §2.4:
for X of shape N x M' (N <= M', alpha = M'/N), a dense product of an
a x b and a b x c matrix is 2abc FLOPs and a symmetric product (only one
triangle computed) counts half, so X X^T is M' N^2 and an N x N symmetric
product is N^3.
"""

from __future__ import annotations


def wide(m: int, n: int):
    """(N, M') = (min, max) of the matrix sides: NS runs on the wide form."""
    return (m, n) if m <= n else (n, m)


def ns_standard_flops(m: int, n: int, T: int = 5, symmetric: bool = True) -> int:
    """Standard quintic NS, T steps of X X^T, A^2, B X (§1.2 eq. (3)).

    symmetric: T (3 alpha + 1) N^3; dense: T (4 alpha + 2) N^3.
    """
    N, Mp = wide(m, n)
    if symmetric:
        per = Mp * N * N + N ** 3 + 2 * Mp * N * N
    else:
        per = 2 * Mp * N * N + 2 * N ** 3 + 2 * Mp * N * N
    return T * per


def gram_ns_schedule(T: int = 5, restart_after=(2,)):
    """Products issued by Gram NS with the savings the page lists.

    Returns a list of (name, kind) with kind in {"xxt", "sym", "qx"}.
    Per step: R^2 always; Q Z unless Q = I (first step of a block); R Z and
    Z (R Z) unless the step is the last of its block (R is not needed again).
    Each block ends with Q X; a restart recomputes X X^T.
    """
    restarts = sorted(t for t in restart_after if 1 <= t < T)
    ends = set(restarts) | {T}
    sched = [("R=XX^T", "xxt")]
    first = True
    for t in range(1, T + 1):
        sched.append((f"R^2[{t}]", "sym"))
        if not first:
            sched.append((f"QZ[{t}]", "sym"))
        if t not in ends:
            sched.append((f"RZ[{t}]", "sym"))
            sched.append((f"Z(RZ)[{t}]", "sym"))
        first = False
        if t in ends:
            sched.append((f"QX[{t}]", "qx"))
            if t != T:
                sched.append((f"R=XX^T[{t}]", "xxt"))
                first = True
    return sched


def gram_ns_flops(m: int, n: int, T: int = 5, restart_after=(2,)) -> int:
    N, Mp = wide(m, n)
    cost = {"xxt": Mp * N * N, "sym": N ** 3, "qx": 2 * Mp * N * N}
    return sum(cost[k] for _, k in gram_ns_schedule(T, restart_after))


def gram_ns_gemm_count(T: int = 5, restart_after=(2,)) -> int:
    return len(gram_ns_schedule(T, restart_after))


def step_bytes_per_element(gdtype_bytes: int = 2) -> float:
    """HBM bytes per weight element of one GRASP step that the method must move.

    G (gdtype_bytes) + old and new 4-bit codes (0.5 + 0.5) + old and new grid
    scales (2 fp32 scales per 128 elements each way: 0.0625 + 0.0625) + fp32 W
    read and written (8). The k (m + n) factor bytes are ignored.
    """
    return gdtype_bytes + 0.5 + 0.5 + 0.0625 + 0.0625 + 8.0
