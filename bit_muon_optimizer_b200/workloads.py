"""Seeded synthetic workloads: parameter-set shapes and gradient generators.

This module only draws random inputs; it holds none of the optimizer's
arithmetic, so both the CUDA path and the CPU oracle may use it.

The five workloads stand in for the gradients of the trainings the GRASP
paper note reports (LLaMA 130M / 1.1B pre-training, Qwen2.5-7B fine-tuning;
"Achieving low-bit Muon through subspace preservation and grid quantization",
main experiments) plus an aspect-ratio / batching stress case. No dataset or
checkpoint is used: gradients are Gaussian (or Student-t) with a few outlier
rows and columns, the two-dimensional outlier structure the note's grid
quantization targets (key design 2).

Seeding: workload id ``cid`` uses ``seed = 20260 + cid``; matrix ``b`` (its
index in the parameter set) at step ``t`` draws from a generator seeded with
``seed * 1000003 + b * 1009 + t``. Step ``t = 0`` is reserved for the
per-matrix fixed draws (outlier rows / columns, initial weight).
"""

from __future__ import annotations

from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class ShapeGroup:
    m: int        # rows of the weight (natural orientation)
    n: int        # cols
    count: int    # same-shape matrices, batched in one library call


@dataclass(frozen=True)
class Workload:
    cid: int
    name: str
    groups: tuple
    k: int
    steps: int
    gdtype: torch.dtype
    dist: str               # "gauss" or "student_t3"
    std: float              # Gaussian std, or Student-t scale
    outlier_frac: float     # fraction of rows / cols scaled (0: none)
    outlier_count: int      # fixed count instead of a fraction (0: use frac)
    outlier_factor: float
    ns_modes: tuple = ("standard",)
    mu: float = 0.95
    eta: float = 0.02
    wd: float = 0.0
    T: int = 5

    @property
    def seed(self) -> int:
        return 20260 + self.cid

    def matrices(self):
        """(b, m, n, group index) for every matrix of the parameter set."""
        b = 0
        for gi, g in enumerate(self.groups):
            for _ in range(g.count):
                yield b, g.m, g.n, gi
                b += 1

    def group_base(self, gi: int) -> int:
        return sum(g.count for g in self.groups[:gi])

    @property
    def elements(self) -> int:
        return sum(g.m * g.n * g.count for g in self.groups)


WORKLOADS = {
    1: Workload(1, "single-256x512-fp32", (ShapeGroup(256, 512, 1),), k=8, steps=3,
                gdtype=torch.float32, dist="gauss", std=1e-3, outlier_frac=0.0,
                outlier_count=2, outlier_factor=10.0),
    2: Workload(2, "llama130m-2d-params", (ShapeGroup(768, 768, 48), ShapeGroup(2048, 768, 24),
                                           ShapeGroup(768, 2048, 12)), k=16, steps=10,
                gdtype=torch.bfloat16, dist="gauss", std=1e-3, outlier_frac=0.01,
                outlier_count=0, outlier_factor=10.0, ns_modes=("standard", "gram")),
    3: Workload(3, "llama1.1b-2d-params", (ShapeGroup(2048, 2048, 44), ShapeGroup(256, 2048, 44),
                                           ShapeGroup(5632, 2048, 44), ShapeGroup(2048, 5632, 22)),
                k=32, steps=5, gdtype=torch.bfloat16, dist="gauss", std=1e-3,
                outlier_frac=0.01, outlier_count=0, outlier_factor=10.0),
    4: Workload(4, "qwen2.5-7b-2d-params", (ShapeGroup(3584, 3584, 56), ShapeGroup(512, 3584, 56),
                                            ShapeGroup(18944, 3584, 56), ShapeGroup(3584, 18944, 28)),
                k=32, steps=3, gdtype=torch.bfloat16, dist="gauss", std=5e-4,
                outlier_frac=0.005, outlier_count=0, outlier_factor=20.0),
    5: Workload(5, "moe-experts-plus-alpha4", (ShapeGroup(1408, 2048, 64), ShapeGroup(4096, 16384, 1)),
                k=32, steps=3, gdtype=torch.bfloat16, dist="student_t3", std=1e-3,
                outlier_frac=0.0, outlier_count=0, outlier_factor=1.0,
                ns_modes=("standard", "gram")),
}


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _step_seed(w: Workload, b: int, t: int) -> int:
    return w.seed * 1000003 + b * 1009 + t


def outliers(w: Workload, b: int, m: int, n: int):
    """Fixed outlier row and column indices of matrix b (drawn at t = 0)."""
    if w.outlier_count:
        nr = nc = w.outlier_count
    elif w.outlier_frac > 0:
        nr, nc = max(1, round(w.outlier_frac * m)), max(1, round(w.outlier_frac * n))
    else:
        return torch.empty(0, dtype=torch.long), torch.empty(0, dtype=torch.long)
    g = _gen(_step_seed(w, b, 0), "cpu")
    rows = torch.randperm(m, generator=g)[:nr]
    cols = torch.randperm(n, generator=g)[:nc]
    return rows, cols


def gradient(w: Workload, b: int, t: int, m: int, n: int, device="cpu",
             out: torch.Tensor | None = None) -> torch.Tensor:
    """Synthetic gradient of matrix b at step t (t >= 1), dtype ``w.gdtype``.

    Gaussian N(0, std^2) (``std`` is the standard deviation) or Student-t with
    3 degrees of freedom times ``std``; then the fixed outlier rows and
    columns are multiplied by ``outlier_factor`` (so their intersections get
    the factor squared).
    """
    g = _gen(_step_seed(w, b, t), device)
    x = torch.randn((m, n), generator=g, device=device, dtype=torch.float32)
    if w.dist == "student_t3":
        chi = torch.randn((3, m, n), generator=g, device=device, dtype=torch.float32)
        chi2 = (chi * chi).sum(dim=0)
        x = x / torch.sqrt(chi2 / 3.0)
    x = x * w.std
    rows, cols = outliers(w, b, m, n)
    if rows.numel():
        rows, cols = rows.to(device), cols.to(device)
        x[rows, :] *= w.outlier_factor
        x[:, cols] *= w.outlier_factor
    x = x.to(w.gdtype)
    if out is not None:
        out.copy_(x)
        return out
    return x


def initial_weight(w: Workload, b: int, m: int, n: int, device="cpu") -> torch.Tensor:
    """fp32 master weight of matrix b: N(0, 0.02^2), drawn at t = 0."""
    g = _gen(_step_seed(w, b, 0) ^ 0x5A5A, device)
    return torch.randn((m, n), generator=g, device=device, dtype=torch.float32) * 0.02


def random_matrix(shape, seed: int, std: float = 1.0, device="cpu", dtype=torch.float32):
    """Plain seeded Gaussian matrix for unit tests."""
    g = _gen(seed, device)
    return (torch.randn(shape, generator=g, device=device, dtype=torch.float32) * std).to(dtype)
