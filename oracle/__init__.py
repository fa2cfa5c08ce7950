"""Plain, slow fp64 CPU oracle of one 4-bit-Muon-GRASP optimizer step.

TEST INFRASTRUCTURE ONLY. Nothing in the product path imports this package:
only ``tests/``, ``__graft_entry__.smoke()`` and the two legs of ``bench.py``
that time the oracle (the CPU baseline and the reference arm) may use it. It
shares no code with the CUDA library; the only module both sides use is the
seeded input generator (``bit_muon_optimizer_b200.workloads``), which holds
none of the method's arithmetic.

Sources (cited in each function by page and section):

* [GRASP]  "Achieving low-bit Muon through subspace preservation and grid
  quantization" (ICLR 2026 paper note) -- the step itself, and the direct
  4-bit codec it is compared with.
* [LiMuon] "LiMuon: Light and Fast Muon Optimizer for Large Models" (paper
  note) -- the constant quintic Newton-Schulz coefficients.
* [GramNS] "优化器 (3)（Gram Newton-Schulz）" (blog post on Gram
  Newton-Schulz) -- standard NS, Algorithms 1 and 2, Proposition 1,
  Theorem 1, the Polar Express table and the restart bounds.
* [MuonQ]  "MuonQ: Enhancing Low-Bit Muon Quantization via Directional
  Fidelity Optimization" (abstract) -- the mu-law companding codec.

Every function here is pinned by a ``-m "not gpu"`` test against something
other than itself (closed forms, brute force, library routines, the pages'
printed numbers). The end-to-end training quality the pages report needs
datasets and is "parity unpinned"; so are MuonQ's own choices (its mu and
normalisation), which the pages do not state.
"""

from .grasp import *  # noqa: F401,F403
