"""GRASP steps over weights and gradients held in pinned host memory.

The quantized momentum state stays on the device: it is the optimizer's own
memory (4.5 bits per element plus the 8-bit factors, "Achieving low-bit Muon
through subspace preservation and grid quantization", worked step, last
paragraph). The fp32 weights and the gradients of a batch stream in and the
updated weights stream out, a chunk of matrices at a time, on three CUDA
streams: while chunk i steps on the compute stream, chunk i + 1's weights and
gradient are copied in and chunk i - 1's updated weights copied out. A step
over host-resident data then costs about the largest of the copy-in time, the
copy-out time and the step, instead of their sum.

Every matrix's step is independent of the others in its batch, so cutting a
batch into chunks changes no result: each chunk is one library call on a
contiguous slice of the device state, with the matrices' own indices as
``matrix_ids``.
"""

from __future__ import annotations

import torch

from . import gmuon as gm


def chunk_bounds(B: int, chunk: int) -> list[tuple[int, int]]:
    """[a, b) ranges of at most ``chunk`` matrices covering 0 .. B-1 in order."""
    if B < 1 or chunk < 1:
        raise ValueError("B and chunk must be >= 1")
    return [(a, min(B, a + chunk)) for a in range(0, B, chunk)]


def default_chunk(B: int, m: int, n: int) -> int:
    """Matrices per chunk: about 2^25 elements, between 1 and B / 8 rounded up."""
    return max(1, min(-(-B // 8), -(-(1 << 25) // (m * n))))


class HostStreamedStep:
    """``step(W_host, G_host)``: one GRASP step of B same-shape matrices whose fp32
    weights ``W_host`` [B, m, n] (updated in place) and gradients ``G_host``
    [B, m, n] (fp32, bf16 or fp16) are pinned host tensors; the state lives on
    ``device``. ``chunk`` matrices per library call (default: about 2^25 elements,
    at least one matrix and at most B / 8 rounded up: the copies of one chunk are
    the part that nothing overlaps at either end); ``nbuf`` device buffer slots
    (three let chunk i + 1 come in while chunk i steps and chunk i - 1 goes out).
    The call returns once the work is queued; the caller's current stream is made
    to wait for the last copy out. Further keyword arguments are GraspStep's (mu,
    eta, wd, T, ns, seed, ...)."""

    def __init__(self, B: int, m: int, n: int, k: int, gdtype=torch.bfloat16, chunk: int | None = None,
                 device=None, matrix_ids=None, nbuf: int = 3, **params):
        dev = torch.device(device or "cuda")
        if nbuf < 2:
            raise ValueError("nbuf must be >= 2")
        self.B, self.m, self.n, self.k, self.gdtype, self.nbuf = B, m, n, k, gdtype, nbuf
        self.bounds = chunk_bounds(B, chunk or default_chunk(B, m, n))
        ids = list(range(B)) if matrix_ids is None else [int(i) for i in matrix_ids]
        if len(ids) != B:
            raise ValueError("matrix_ids: B indices expected")
        self.ids = torch.tensor(ids, dtype=torch.int64, device=dev)
        sizes = sorted({b - a for a, b in self.bounds})
        ns = params.get("ns", gm.GM_NS_STANDARD)
        # one workspace for every chunk: the steps run one after another on one stream
        ws_bytes = max(gm.workspace_bytes(gm.GM_OP_GRASP_STEP, s, m, n, k, ns) for s in sizes)
        self.ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
        self.steps = {s: gm.GraspStep(s, m, n, k, device=dev, ws=self.ws, matrix_ids=ids[:s],
                                      **params) for s in sizes}
        self.state = gm.GraspState.zeros(B, m, n, k, dev)
        st = self.state
        # each chunk's state: views of the batch arrays, its own step count and status
        self.chunk_states = [
            gm.GraspState(st.codes4[a:b], st.rscale[a:b], st.cscale[a:b], st.P8[a:b],
                          st.Pscale[a:b], st.R8[a:b], st.Rscale[a:b],
                          torch.zeros(1, dtype=torch.int64, device=dev),
                          torch.zeros(1, dtype=torch.int32, device=dev))
            for a, b in self.bounds]
        c = max(sizes)
        self.Wbuf = [torch.empty((c, m, n), dtype=torch.float32, device=dev) for _ in range(nbuf)]
        self.Gbuf = [torch.empty((c, m, n), dtype=gdtype, device=dev) for _ in range(nbuf)]
        self.s_in, self.s_comp, self.s_out = (torch.cuda.Stream(device=dev) for _ in range(3))
        self.ev_in = [torch.cuda.Event() for _ in range(nbuf)]
        self.ev_comp = [torch.cuda.Event() for _ in range(nbuf)]
        self.ev_out = [torch.cuda.Event() for _ in range(nbuf)]
        self.device = dev

    def h2d_bytes(self) -> int:
        return self.B * self.m * self.n * (4 + torch.empty((), dtype=self.gdtype).element_size())

    def d2h_bytes(self) -> int:
        return self.B * self.m * self.n * 4

    def status(self) -> int:
        """The first non-zero device status of the chunks' last steps (0: all clean);
        synchronises."""
        for s in self.chunk_states:
            v = int(s.dev_status.item())
            if v:
                return v
        return 0

    def __call__(self, W_host: torch.Tensor, G_host: torch.Tensor) -> None:
        B, m, n = self.B, self.m, self.n
        gm._expect(W_host, (B, m, n), (torch.float32,), "W_host")
        gm._expect(G_host, (B, m, n), (self.gdtype,), "G_host")
        for t, name in ((W_host, "W_host"), (G_host, "G_host")):
            if t.is_cuda or not t.is_pinned() or not t.is_contiguous():
                raise ValueError(f"{name}: expected a contiguous pinned host tensor")
        cur = torch.cuda.current_stream(self.device)
        start = torch.cuda.Event()
        start.record(cur)
        for s in (self.s_in, self.s_comp, self.s_out):
            s.wait_event(start)
        for i, (a, b) in enumerate(self.bounds):
            slot, c = i % self.nbuf, b - a
            Wd, Gd = self.Wbuf[slot][:c], self.Gbuf[slot][:c]
            with torch.cuda.stream(self.s_in):
                if i >= self.nbuf:
                    self.s_in.wait_event(self.ev_out[slot])   # the slot's last weights are out
                Wd.copy_(W_host[a:b], non_blocking=True)
                Gd.copy_(G_host[a:b], non_blocking=True)
                self.ev_in[slot].record(self.s_in)
            with torch.cuda.stream(self.s_comp):
                self.s_comp.wait_event(self.ev_in[slot])
                step = self.steps[c]
                step.ids.copy_(self.ids[a:b], non_blocking=True)
                step(self.chunk_states[i], Wd, Gd)
                self.ev_comp[slot].record(self.s_comp)
            with torch.cuda.stream(self.s_out):
                self.s_out.wait_event(self.ev_comp[slot])
                W_host[a:b].copy_(Wd, non_blocking=True)
                self.ev_out[slot].record(self.s_out)
        done = torch.cuda.Event()
        done.record(self.s_out)
        cur.wait_event(done)
