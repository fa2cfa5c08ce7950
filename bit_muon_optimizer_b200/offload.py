"""GRASP steps over gradients (and, optionally, weights) held in pinned host memory.

The quantized momentum state stays on the device: it is the optimizer's own
memory (4.5 bits per element plus the 8-bit factors, "Achieving low-bit Muon
through subspace preservation and grid quantization", worked step, last
paragraph). The gradients of a batch stream in a chunk of matrices at a time,
on three CUDA streams: while chunk i steps on the compute stream, chunk i + 1's
gradient is copied in. The fp32 weights either stay on the device (updated in
place: only the gradients cross PCIe) or live in pinned host memory too, and
then stream in with the gradients and out once updated (chunk i - 1's weights
go out while chunk i steps). A step over host-resident data then costs about
the largest of the copy-in time, the copy-out time and the step, instead of
their sum. Instances can share their three streams, so that one batch's copies
run under another batch's steps.

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


# Above this many elements a batch is best stepped as several library calls on
# contiguous sub-batches (each matrix's step is independent of its batch, so the
# results are the same bit for bit). Measured on one B200 under its 1 kW cap: the
# 3.8e9-element 56 x 18944 x 3584 batch ran both halves of the step 4-6 % faster as
# 4 calls of 14 matrices than as one call of 56 (a higher SM clock for the same
# cycles, a quarter of the workspace); 0.72e9 elements (56 x 3584^2) gained 1-2 %
# from splitting and 0.5e9 (44 x 5632 x 2048) nothing.
SUB_BATCH_ELEMENTS = 1.0e9


def sub_batch_size(B: int, m: int, n: int, limit: float = SUB_BATCH_ELEMENTS) -> int:
    """Matrices per library call for a batch of B m x n matrices: the batch in the
    fewest calls of at most ``limit`` elements each (one matrix per call at least),
    the calls as equal as the count allows."""
    if B < 1 or m < 1 or n < 1 or limit < 1:
        raise ValueError("B, m, n and limit must be >= 1")
    calls = max(1, -(-B * m * n // int(limit)))
    return -(-B // calls)


def default_chunk(B: int, m: int, n: int) -> int:
    """Matrices per chunk: about 2^25 elements, between 1 and B / 8 rounded up."""
    return max(1, min(-(-B // 8), -(-(1 << 25) // (m * n))))


class HostStreamedStep:
    """``step(W, G_host)``: one GRASP step of B same-shape matrices whose gradients
    ``G_host`` [B, m, n] (fp32, bf16 or fp16) are a pinned host tensor. The fp32
    weights ``W`` [B, m, n] are updated in place and are either a pinned host tensor
    (copied in with the gradients and out again, chunk by chunk) or a tensor on
    ``device`` (no copies). The state lives on ``device``. ``chunk`` matrices per
    library call (default: about 2^25 elements, at least one matrix and at most B / 8
    rounded up: the copies of one chunk are the part that nothing overlaps at either
    end); ``nbuf`` device buffer slots (three let chunk i + 1 come in while chunk i
    steps and chunk i - 1 goes out); ``streams``: the three CUDA streams (copy in,
    compute, copy out), to share them with other instances. Each call ends by copying
    the chunks' device statuses into ``status_host`` (pinned, one int32 per chunk)
    and returns once the work is queued; with ``wait`` (the default) the caller's
    current stream is made to wait for that last copy. Further keyword arguments are
    GraspStep's (mu, eta, wd, T, ns, seed, ...)."""

    def __init__(self, B: int, m: int, n: int, k: int, gdtype=torch.bfloat16, chunk: int | None = None,
                 device=None, matrix_ids=None, nbuf: int = 3, streams=None, **params):
        dev = torch.device(device or "cuda")
        if dev.index is None:
            dev = torch.device("cuda", torch.cuda.current_device())
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
        nc = len(self.bounds)
        self.status_dev = torch.zeros(nc, dtype=torch.int32, device=dev)
        self.status_host = torch.zeros(nc, dtype=torch.int32).pin_memory()
        # each chunk's state: views of the batch arrays, its own step count and status
        self.chunk_states = [
            gm.GraspState(st.codes4[a:b], st.rscale[a:b], st.cscale[a:b], st.P8[a:b],
                          st.Pscale[a:b], st.R8[a:b], st.Rscale[a:b],
                          torch.zeros(1, dtype=torch.int64, device=dev), self.status_dev[i:i + 1])
            for i, (a, b) in enumerate(self.bounds)]
        self.cmax = max(sizes)
        self.Wbuf = None   # weight slots, made on the first call with host weights
        self.Gbuf = [torch.empty((self.cmax, m, n), dtype=gdtype, device=dev) for _ in range(nbuf)]
        if streams is None:
            streams = tuple(torch.cuda.Stream(device=dev) for _ in range(3))
        if len(streams) != 3:
            raise ValueError("streams: (copy in, compute, copy out) expected")
        self.s_in, self.s_comp, self.s_out = streams
        self.ev_in = [torch.cuda.Event() for _ in range(nbuf)]
        self.ev_comp = [torch.cuda.Event() for _ in range(nbuf)]
        self.ev_out = [torch.cuda.Event() for _ in range(nbuf)]
        self.used = [False] * nbuf   # a slot's ev_out marks the end of its last use
        self.ev_status = None        # the last call's status copy
        self.device = dev

    def h2d_bytes(self, weights_on_device: bool = False) -> int:
        g = self.B * self.m * self.n * torch.empty((), dtype=self.gdtype).element_size()
        return g if weights_on_device else g + self.B * self.m * self.n * 4

    def d2h_bytes(self, weights_on_device: bool = False) -> int:
        st = 4 * len(self.bounds)
        return st if weights_on_device else st + self.B * self.m * self.n * 4

    def status(self) -> int:
        """The first non-zero device status of the chunks' last steps (0: all clean);
        synchronises."""
        for v in self.status_dev.cpu().tolist():
            if v:
                return v
        return 0

    def __call__(self, W: torch.Tensor, G_host: torch.Tensor, wait: bool = True) -> None:
        B, m, n = self.B, self.m, self.n
        gm._expect(W, (B, m, n), (torch.float32,), "W")
        gm._expect(G_host, (B, m, n), (self.gdtype,), "G_host")
        if G_host.is_cuda or not G_host.is_pinned() or not G_host.is_contiguous():
            raise ValueError("G_host: expected a contiguous pinned host tensor")
        resident = W.is_cuda
        if resident:
            if W.device != self.device or not W.is_contiguous():
                raise ValueError(f"W: expected a contiguous tensor on {self.device} or pinned host memory")
        elif not W.is_pinned() or not W.is_contiguous():
            raise ValueError("W: expected a contiguous pinned host tensor or a tensor on the device")
        if not resident and self.Wbuf is None:
            self.Wbuf = [torch.empty((self.cmax, m, n), dtype=torch.float32, device=self.device)
                         for _ in range(self.nbuf)]
        cur = torch.cuda.current_stream(self.device)
        start = torch.cuda.Event()
        start.record(cur)
        for s in (self.s_in, self.s_comp, self.s_out):
            s.wait_event(start)
        if self.ev_status is not None:   # the statuses are reset only once the last ones are out
            self.s_comp.wait_event(self.ev_status)
        for i, (a, b) in enumerate(self.bounds):
            slot, c = i % self.nbuf, b - a
            Gd = self.Gbuf[slot][:c]
            Wd = W[a:b] if resident else self.Wbuf[slot][:c]
            with torch.cuda.stream(self.s_in):
                if self.used[slot]:
                    self.s_in.wait_event(self.ev_out[slot])   # the slot's last use is over
                if not resident:
                    Wd.copy_(W[a:b], non_blocking=True)
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
                if not resident:
                    W[a:b].copy_(Wd, non_blocking=True)
                self.ev_out[slot].record(self.s_out)
            self.used[slot] = True
        with torch.cuda.stream(self.s_out):
            self.status_host.copy_(self.status_dev, non_blocking=True)
            self.ev_status = torch.cuda.Event()
            self.ev_status.record(self.s_out)
        if wait:
            cur.wait_event(self.ev_status)
