"""Benchmark of one GRASP optimizer step over a parameter set, on B200s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config 4] [--ns standard|gram]
                    [--impl ours|reference]
    python bench.py --profile S [--config c] [--group g] [--batch B]   (launches for profilers)

A "step" is one full GRASP step (rebuild, momentum, power iteration, 4/8-bit
re-quantization, Newton-Schulz, weight update) over every matrix of the
parameter set, with that step's synthetic gradients already resident in HBM.
The default parameter set is the largest one that fits one GPU: the
Qwen2.5-7B-shaped set (6.5e9 weight elements), measured one shape group at a
time (each group batched in gm_grasp_step calls of at most about 1e9 elements,
replayed from CUDA graphs); the set's time is the sum over its groups. N > 1 (torchrun): the set
is split by ownership across the ranks (each matrix's step runs on one owner,
then one NCCL all-gather per shape group gives every rank the updated set:
strong scaling); the time is the max over ranks.

Printed (rank 0): one JSON line with value = ms per parameter set for the
whole job; the NS chain's tensor-core roofline and the codec half's HBM rate,
both timed with CUDA events around the step's own two halves
(gm_grasp_state_update, gm_grasp_apply); an end-to-end number through pinned
host buffers; and the fp64 CPU oracle timed on a bounded sample.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402
import torch.distributed as dist  # noqa: E402

from bit_muon_optimizer_b200 import flops as FL  # noqa: E402
from bit_muon_optimizer_b200 import workloads as WL  # noqa: E402

METRIC = "GRASP-Muon step ms per param set; NS TFLOP/s; (de)quant HBM GB/s vs peak"
UNIT = "ms/param_set"


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d["hbm_gbs"], d["bf16_tflops"], d.get("bf16_tflops_sustained"), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during a region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.file = None

    def __enter__(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=self.file, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        if self.file is None:
            return None
        try:
            with open(self.file.name) as f:
                rows = [r.split(",") for r in f.read().strip().splitlines() if r.strip()]
            os.unlink(self.file.name)
        except Exception:
            return None
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            r = [x.strip() for x in r]
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                mx = float(r[2])
            except ValueError:
                continue
            for nm, v in zip(names, r[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def init_dist(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    if world != n_gpus and rank == 0:
        print(f"warning: --gpus {n_gpus} but WORLD_SIZE {world}", file=sys.stderr)
    return world, rank, local


def barrier(world):
    if world > 1:
        dist.barrier()


def max_over_ranks(v: float, world: int) -> float:
    if world == 1:
        return v
    t = torch.tensor([v], dtype=torch.float64, device="cuda" if torch.cuda.is_available() else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------ CPU oracle

def oracle_sample_seconds(w: WL.Workload, ns: str):
    """Time the fp64 oracle: one step (from a zero state) of one matrix of every
    shape group; returns (ms per parameter set = sum over groups of the group's
    count x its sample's time, sample text, cores)."""
    import oracle as O
    per_shape = []
    for gi, g in enumerate(w.groups):
        b = w.group_base(gi)
        W = WL.initial_weight(w, b, g.m, g.n)
        G = WL.gradient(w, b, 1, g.m, g.n)
        t0 = time.perf_counter()
        O.grasp_step(O.zero_state(g.m, g.n, w.k), W, G, mu=w.mu, eta=w.eta, wd=w.wd, seed=w.seed,
                     b=b, ns=ns_name(ns, g.m, g.n), T=w.T)
        per_shape.append((g, time.perf_counter() - t0))
    ms = 1e3 * sum(g.count * s for g, s in per_shape)
    sample = ("fp64 oracle, one step of one matrix per shape group ("
              + ", ".join(f"{g.m}x{g.n}: {s:.2f} s" for g, s in per_shape)
              + "), extrapolated by the group counts")
    return ms, sample, torch.get_num_threads()


def run_reference(args, world, rank):
    """The reference arm: the fp64 CPU oracle as it stands, on this host's cores.

    Every shape group has one sample matrix whose state and weight carry over
    from one of its steps to the next. Each reference step (warm-up or timed)
    runs one oracle step of one sample, the groups taken in turn, so a step
    costs one matrix step however large the set; it reports the parameter
    set's time as the sum over groups of (matrices in the group) x (the latest
    step time of the group's sample). Samples not yet timed after the warm-up
    steps get one untimed step first. Only rank 0 works; the other ranks
    return at once."""
    if rank != 0:
        return
    import oracle as O
    w = WL.WORKLOADS[args.config]
    samples = []
    for gi, g in enumerate(w.groups):
        b = w.group_base(gi)
        samples.append({"g": g, "b": b, "st": O.zero_state(g.m, g.n, w.k),
                        "W": WL.initial_weight(w, b, g.m, g.n), "t": 0, "s": None})

    def one(smp):
        g, b = smp["g"], smp["b"]
        smp["t"] += 1
        G = WL.gradient(w, b, smp["t"], g.m, g.n)
        t0 = time.perf_counter()
        r = O.grasp_step(smp["st"], smp["W"], G, mu=w.mu, eta=w.eta, wd=w.wd, seed=w.seed, b=b,
                         ns=ns_name(args.ns, g.m, g.n), T=w.T)
        smp["s"] = time.perf_counter() - t0
        smp["st"], smp["W"] = r.state, r.W.float()

    ng = len(samples)
    for i in range(args.warmup):
        one(samples[i % ng])
    for smp in samples:
        if smp["s"] is None:
            one(smp)
    vals = []
    for i in range(args.steps):
        one(samples[(args.warmup + i) % ng])
        vals.append(1e3 * sum(smp["g"].count * smp["s"] for smp in samples))
    v = statistics.median(vals)
    cores = torch.get_num_threads()
    sample = ("fp64 oracle, one sample matrix per shape group ("
              + ", ".join(f"{s['g'].m}x{s['g'].n}" for s in samples)
              + ") with its state carried across its steps; each reference step runs one "
              "sample's step, groups in turn; per-set time = sum over groups of the count x "
              "the sample's latest step time; median over the timed steps")
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": v, "higher_is_better": False,
        "scaling": "strong", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "ns": args.ns, "k": w.k, "matrices": sum(g.count for g in w.groups)},
        "cpu_baseline": {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ GPU arm

GRAD_POOL = 6   # distinct gradient buffers per group, used cyclically step after step

# DRAM bytes per k_gemm launch, averaged over one step's NS products of the named
# workload, from an ncu capture of dram__bytes_read.sum + dram__bytes_write.sum (the
# k_gemm summaries under profiles/); reported only while gm_gemm.cu is the source
# that capture measured.
GEMM_TRAFFIC = [
    {"config": 4, "ns": "standard", "bytes_per_launch": 4257.0e6,
     "source_sha256": "d8cac0d9bacf42c2a06c6af7b09cd89c2a32c210593a66093925bae5ae9b91a4"},
]


# Thread instructions per element of the codec half (the nine kernels of
# gm_grasp_state_update, k = 32), from the committed ncu summary of the codec
# passes (`smsp__inst_executed.sum` x 32 / elements on the 18944 x 3584 shape);
# valid only for the gm_codec.cu source it was captured on.
CODEC_INSTR = [
    {"configs": [4], "thread_instr_per_element": 112.69,
     "source_sha256": "214c383857469e9b96f3dcc4823d1632f9ee13bd46ff8f58043e62e9737de36d"},
]


def codec_instr(config: int):
    import hashlib
    path = os.path.join(ROOT, "bit_muon_optimizer_b200", "csrc", "gm_codec.cu")
    try:
        with open(path, "rb") as f:
            sha = hashlib.sha256(f.read()).hexdigest()
    except OSError:
        return None
    for t in CODEC_INSTR:
        if sha == t["source_sha256"] and config in t["configs"]:
            return t["thread_instr_per_element"]
    return None


def gemm_traffic(config: int, ns: str):
    import hashlib
    path = os.path.join(ROOT, "bit_muon_optimizer_b200", "csrc", "gm_gemm.cu")
    try:
        with open(path, "rb") as f:
            sha = hashlib.sha256(f.read()).hexdigest()
    except OSError:
        return None
    for t in GEMM_TRAFFIC:
        if sha == t["source_sha256"] and config == t["config"] and ns == t["ns"]:
            return t["bytes_per_launch"]
    return None


def est_bytes(w: WL.Workload, pool: int) -> int:
    """Device bytes of the benchmark per parameter-set element: fp32 W, the
    gradient pool, the step workspace (fp32 M, the 16-bit iterate, NS buffers)
    and the comparator's copies."""
    elems = sum(g.count * g.m * g.n for g in w.groups)
    return elems * (22 + 2 * pool)


def ns_name(ns: str, m: int, n: int) -> str:
    """The NS form ("standard" or "gram") that --ns gives an m x n matrix."""
    if ns == "auto":
        return "gram" if m != n else "standard"
    return ns


def ns_chooser(gm, ns: str):
    """The NS form of each shape: "standard" or "gram" everywhere, or "auto": the Gram
    form for non-square matrices, the standard form for square ones (the Gram NS
    page's FLOP comparison: (17 + 3 alpha) n^3 against 5 (3 alpha + 1) n^3 at T = 5,
    fewer exactly when the aspect ratio alpha > 1)."""
    std, gram = gm.GM_NS_STANDARD, gm.GM_NS_GRAM
    if ns == "gram":
        return lambda m, n: gram
    if ns == "auto":
        return lambda m, n: gram if m != n else std
    return lambda m, n: std


def sub_batches(B: int, m: int, n: int) -> int:
    """Matrices per library call for a group of B m x n matrices (offload.sub_batch_size:
    calls of at most about 1e9 elements)."""
    from bit_muon_optimizer_b200.offload import sub_batch_size
    return sub_batch_size(B, m, n)


def build_group(gm, w: WL.Workload, gi: int, nsf, pool: int, dev):
    from bit_muon_optimizer_b200.offload import chunk_bounds
    g = w.groups[gi]
    B, m, n = g.count, g.m, g.n
    base = w.group_base(gi)
    ids = list(range(base, base + B))
    ns = nsf(m, n)
    bounds = chunk_bounds(B, sub_batches(B, m, n))
    sizes = sorted({b - a for a, b in bounds})
    ws = torch.empty(max(gm.workspace_bytes(gm.GM_OP_GRASP_STEP, c, m, n, w.k, ns) for c in sizes),
                     dtype=torch.uint8, device=dev)
    steps = {c: gm.GraspStep(c, m, n, w.k, mu=w.mu, eta=w.eta, wd=w.wd, T=w.T, ns=ns, seed=w.seed,
                             device=dev, ws=ws, matrix_ids=ids[:c]) for c in sizes}
    st = gm.GraspState.zeros(B, m, n, w.k, dev)
    status = torch.zeros(len(bounds), dtype=torch.int32, device=dev)
    subs = []
    for i, (a, b) in enumerate(bounds):
        sub_st = gm.GraspState(st.codes4[a:b], st.rscale[a:b], st.cscale[a:b], st.P8[a:b],
                               st.Pscale[a:b], st.R8[a:b], st.Rscale[a:b],
                               torch.zeros(1, dtype=torch.int64, device=dev), status[i:i + 1])
        subs.append((a, b, steps[b - a], sub_st, torch.tensor(ids[a:b], dtype=torch.int64, device=dev)))
    W = torch.empty((B, m, n), dtype=torch.float32, device=dev)
    for b in range(B):
        W[b] = WL.initial_weight(w, base + b, m, n, device=dev)
    grads = []
    for t in range(1, pool + 1):
        G = torch.empty((B, m, n), dtype=w.gdtype, device=dev)
        for b in range(B):
            WL.gradient(w, base + b, t, m, n, device=dev, out=G[b])
        grads.append(G)
    return dict(subs=subs, ws=ws, st=st, status=status, W=W, grads=grads, B=B, m=m, n=n, ids=ids,
                ns=ns)


def group_step(g, G) -> None:
    """One GRASP step of the group (its sub-batches in order) on the current stream."""
    for a, b, step, st, ids in g["subs"]:
        step.ids.copy_(ids, non_blocking=True)
        step(st, g["W"][a:b], G[a:b])


def group_halves(g, G, events) -> None:
    """The same step as its two halves per sub-batch, CUDA events (before the codec
    half, between the halves, after the NS half) appended to `events`."""
    for a, b, step, st, ids in g["subs"]:
        step.ids.copy_(ids, non_blocking=True)
        e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        e[0].record()
        step.state_update(st, G[a:b])
        e[1].record()
        step.apply(st, g["W"][a:b])
        e[2].record()
        events.append(e)


def our_launches(gm, w: WL.Workload, nsf, groups=None) -> int:
    """Our kernels per step: per group 9 codec kernels (column norms, warm start
    with the factor fragments, rebuild + projection, three orthonormalisation
    kernels, back projection, its finalisation, the 4-bit quantisation with the
    8-bit one folded in), the NS products, and the zero-padding copy when a
    dimension is not a multiple of 64."""
    launches = 0
    for (B, m, n) in (groups if groups is not None else [(g.count, g.m, g.n) for g in w.groups]):
        pad = int(min(m, n) % 64 != 0 or max(m, n) % 64 != 0)
        calls = -(-B // sub_batches(B, m, n))
        launches += calls * (9 + gm.ns_flops(nsf(m, n), m, n, w.T)[1] + pad)
    return launches


def time_steps(groups, args, world, local):
    """args.steps graph-replayed GRASP steps over `groups` (each group on its own
    stream, one graph per gradient slot) after args.warmup untimed ones; returns
    (ms per step, max over ranks; clocks sampled during the timed region; the
    fork helper and streams for further work on the same groups)."""
    dev = groups[0]["W"].device
    streams = [torch.cuda.Stream(device=dev) for _ in groups]
    main = torch.cuda.Stream(device=dev)        # graphs are captured on a side stream

    def fork(enqueue):
        ev = torch.cuda.Event()
        ev.record(main)
        done = []
        for g, s in zip(groups, streams):
            s.wait_event(ev)
            with torch.cuda.stream(s):
                enqueue(g)
            e = torch.cuda.Event()
            e.record(s)
            done.append(e)
        for e in done:
            main.wait_event(e)

    # eager warm-up (also sets kernel attributes), then one graph per gradient slot
    main.wait_stream(torch.cuda.current_stream(dev))
    npool = len(groups[0]["grads"])
    fork(lambda g: group_step(g, g["grads"][0]))
    torch.cuda.synchronize()
    graphs = []
    for t in range(npool):
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, stream=main):
            fork(lambda g, t=t: group_step(g, g["grads"][t]))
        graphs.append(gr)
    torch.cuda.synchronize()
    with torch.cuda.stream(main):
        for t in range(1, args.warmup):
            graphs[t % npool].replay()
    torch.cuda.synchronize()
    barrier(world)

    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        time.sleep(0.3)
        torch.cuda.synchronize()
        barrier(world)
        with torch.cuda.stream(main):
            start.record(main)
            for t in range(args.warmup, args.warmup + args.steps):
                graphs[t % npool].replay()
            end.record(main)
        torch.cuda.synchronize()
        barrier(world)
    ms_step = max_over_ranks(start.elapsed_time(end) / args.steps, world)
    status = [int(g["status"].abs().max()) for g in groups]
    if any(status):
        raise RuntimeError(f"device status {status}")
    del graphs
    return ms_step, clk.summary(), fork, main


def measure(gm, w, groups, nsf, args, world, local, do_e2e):
    """Times args.steps graph-replayed GRASP steps over `groups` (time_steps);
    then the step's two halves with CUDA events around each (codec half:
    gm_grasp_state_update; NS half: gm_grasp_apply); the cuBLAS comparator; and
    (if asked) steps end to end through pinned host buffers."""
    dev = groups[0]["W"].device
    ms_step, clocks, fork, main = time_steps(groups, args, world, local)
    npool = len(groups[0]["grads"])

    # ---- the step's two halves, each bracketed by CUDA events on the stream
    # that launches it; groups one after another (no overlap between groups)
    nb = max(2, min(args.steps, 5))
    evs = []
    with torch.cuda.stream(main):
        for i in range(nb):
            for g in groups:
                group_halves(g, g["grads"][(args.warmup + args.steps + i) % npool], evs)
    torch.cuda.synchronize()
    cod_ms = sum(e0.elapsed_time(e1) for e0, e1, _ in evs) / nb
    ns_ms = sum(e1.elapsed_time(e2) for _, e1, e2 in evs) / nb
    ns_flops = sum(gm.ns_flops(nsf(g["m"], g["n"]), g["m"], g["n"], w.T)[0] * g["B"] for g in groups)
    ns_launches = sum(gm.ns_flops(nsf(g["m"], g["n"]), g["m"], g["n"], w.T)[1] * len(g["subs"])
                      for g in groups)

    # ---- the standalone 4-bit codecs of the same entry points a user calls
    # (4bit-Muon-base group codec, MuonQ's mu-law codec), on the first group's
    # fp32 M_t: HBM GB/s of their algorithmic bytes (4 + 0.5 + 4/128 B per element)
    codecs = None
    if args.codecs:
        g = groups[0]
        M = g["subs"][-1][2].stage_M()      # the group's last sub-batch
        codes = torch.empty((g["B"], g["m"], g["n"] // 2), dtype=torch.uint8, device=dev)
        gsc = torch.empty((g["B"], g["m"] * g["n"] // 128), dtype=torch.float32, device=dev)
        Xo = torch.empty_like(M)
        calls = {"group_quant4": lambda: gm.group_quant4(M, out=(codes, gsc)),
                 "group_dequant4": lambda: gm.group_dequant4(codes, gsc, out=Xo),
                 "mulaw_quant4": lambda: gm.mulaw_quant4(M, out=(codes, gsc)),
                 "mulaw_dequant4": lambda: gm.mulaw_dequant4(codes, gsc, out=Xo)}
        nbytes = M.numel() * (4 + 0.5 + 4 / 128)
        codecs = {"elements": M.numel(), "bytes_per_call": nbytes}
        with torch.cuda.stream(main):
            for name, call in calls.items():
                call()
                c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                c0.record(main)
                for _ in range(5):
                    call()
                c1.record(main)
                torch.cuda.synchronize()
                ms = c0.elapsed_time(c1) / 5
                codecs[name] = {"ms": ms, "gbs": nbytes / (ms * 1e-3) / 1e9}
        del codes, gsc, Xo

    # ---- comparator: the same standard NS chain written with torch.matmul
    # (cuBLAS, bf16, no symmetry) on the same normalised inputs, graph-replayed
    abc = [(3.4445, -4.7750, 2.0315)] * w.T
    for g in groups:                        # one more codec half per sub-batch, untimed
        g["Xc"] = torch.empty((g["B"], min(g["m"], g["n"]), max(g["m"], g["n"])), dtype=torch.bfloat16,
                              device=dev)
        G = g["grads"][0]
        for a, b, step, st, ids in g["subs"]:
            step.ids.copy_(ids)
            step.state_update(st, G[a:b])
            g["Xc"][a:b].copy_(step.stage_X())
        g["Xw"] = torch.empty_like(g["Xc"])

    def cublas_enqueue(g):
        X = g["Xc"]
        for a, b_, c in abc:
            A = torch.matmul(X, X.mT)
            B = torch.baddbmm(A, A, A, beta=b_, alpha=c)
            X = torch.baddbmm(X, B, X, beta=a, alpha=1.0)
        g["Xw"].copy_(X)

    reps = 20 if sum(g["B"] * g["m"] * g["n"] for g in groups) < 5e8 else 3
    fork(cublas_enqueue)
    torch.cuda.synchronize()
    gr = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gr, stream=main):
        fork(cublas_enqueue)
    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(main):
        gr.replay()
        torch.cuda.synchronize()
        s0.record(main)
        for _ in range(reps):
            gr.replay()
        s1.record(main)
    torch.cuda.synchronize()
    cub_ms = s0.elapsed_time(s1) / reps
    del gr
    cub_flops_dense = sum(w.T * g["B"] * (2.0 * min(g["m"], g["n"]) ** 2 * max(g["m"], g["n"]) * 2
                                          + 2.0 * min(g["m"], g["n"]) ** 3) for g in groups)
    for g in groups:
        del g["Xc"], g["Xw"]

    # ---- end to end through host buffers: every step copies W and G in from
    # pinned host memory and the updated W back out, through the library's
    # host-streamed step (offload.HostStreamedStep: chunks of the batch, copies
    # in and out overlapping the steps of neighbouring chunks)
    e2e = None
    if do_e2e:
        from bit_muon_optimizer_b200.offload import HostStreamedStep
        runs = []
        for g in groups:
            hs = HostStreamedStep(g["B"], g["m"], g["n"], w.k, gdtype=w.gdtype, device=dev,
                                  matrix_ids=g["ids"], mu=w.mu, eta=w.eta, wd=w.wd, T=w.T,
                                  ns=g["ns"], seed=w.seed)
            runs.append((hs, g["W"].cpu().pin_memory(), g["grads"][-1].cpu().pin_memory()))
        h2d = sum(hs.h2d_bytes() for hs, _, _ in runs)
        d2h = sum(hs.d2h_bytes() for hs, _, _ in runs)
        e_steps = 3 if h2d < 4e9 else 2
        for hs, Wh, Gh in runs:            # one untimed step (first use of the streams)
            hs(Wh, Gh)
        torch.cuda.synchronize()
        barrier(world)
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record()
        for _ in range(e_steps):
            for hs, Wh, Gh in runs:
                hs(Wh, Gh)
        s1.record()
        torch.cuda.synchronize()
        barrier(world)
        bad = [hs.status() for hs, _, _ in runs]
        if any(bad):
            raise RuntimeError(f"device status {bad}")
        e2e = (max_over_ranks(s0.elapsed_time(s1) / e_steps, world), h2d, d2h)
        del runs
    return dict(ms_step=ms_step, clocks=clocks, ns_ms=ns_ms, ns_flops=ns_flops,
                ns_launches=ns_launches, cod_ms=cod_ms, e2e=e2e, cub_ms=cub_ms,
                cub_flops_dense=cub_flops_dense, codecs=codecs)


def e2e_resident(gm, w: WL.Workload, nsf, args, world, local):
    """The set end to end with the weights and the state resident on the device and
    the gradients in pinned host memory: per step, every shape group's gradient is
    copied in (offload.HostStreamedStep with device weights, chunks of B / 8
    matrices rounded up) and the chunks' device statuses are read back. The groups
    share one copy-in, one compute and one copy-out stream, smallest group first,
    so each group's copies run under the previous group's steps. Returns (ms per
    step, max over ranks; H2D bytes; D2H bytes)."""
    from bit_muon_optimizer_b200.offload import HostStreamedStep
    dev = torch.device("cuda", local)
    streams = tuple(torch.cuda.Stream(device=dev) for _ in range(3))
    order = sorted(range(len(w.groups)), key=lambda gi: w.groups[gi].count * w.groups[gi].m * w.groups[gi].n)
    runs = []
    for gi in order:
        g = w.groups[gi]
        B, m, n = g.count, g.m, g.n
        base = w.group_base(gi)
        hs = HostStreamedStep(B, m, n, w.k, gdtype=w.gdtype, chunk=-(-B // 8), device=dev,
                              matrix_ids=range(base, base + B), mu=w.mu, eta=w.eta, wd=w.wd, T=w.T,
                              ns=nsf(m, n), seed=w.seed, streams=streams)
        W = torch.empty((B, m, n), dtype=torch.float32, device=dev)
        Gh = torch.empty((B, m, n), dtype=w.gdtype, pin_memory=True)
        for b in range(B):
            W[b] = WL.initial_weight(w, base + b, m, n, device=dev)
            Gh[b].copy_(WL.gradient(w, base + b, 1, m, n, device=dev))
        runs.append((hs, W, Gh))
    h2d = sum(hs.h2d_bytes(True) for hs, _, _ in runs)
    d2h = sum(hs.d2h_bytes(True) for hs, _, _ in runs)

    def one_step():
        for j, (hs, W, Gh) in enumerate(runs):
            hs(W, Gh, wait=j == len(runs) - 1)

    one_step()                         # untimed: first use of the streams and buffers
    torch.cuda.synchronize()
    e_steps = 3
    barrier(world)
    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s0.record()
    for _ in range(e_steps):
        one_step()
    s1.record()
    torch.cuda.synchronize()
    barrier(world)
    bad = [int(hs.status_host.abs().max()) for hs, _, _ in runs]
    if any(bad):
        raise RuntimeError(f"device status {bad}")
    ms = max_over_ranks(s0.elapsed_time(s1) / e_steps, world)
    del runs
    torch.cuda.empty_cache()
    return ms, h2d, d2h


def codec_bytes(w: WL.Workload, groups) -> float:
    """Algorithmic HBM bytes of the codec half (worked steps 1-5) per step: read
    G and the old 4-bit codes and grid scales, write the new ones and the
    16-bit NS input (the k (m + n) factor bytes are ignored)."""
    gb = 2 if w.gdtype != torch.float32 else 4
    return sum(g["B"] * g["m"] * g["n"] for g in groups) * (gb + 2 * (0.5 + 0.0625) + 2)


def run_single(gm, w, nsf, args, local):
    dev = torch.device("cuda", local)
    total_mem = torch.cuda.get_device_properties(dev).total_memory
    pool = min(GRAD_POOL, args.warmup + args.steps)
    if est_bytes(w, pool) > 0.7 * total_mem:
        pool = 2
    # a set too large to hold at once is measured one shape group at a time; the
    # groups are independent and each fills the GPU, so the set's time is the sum
    per_group = est_bytes(w, pool) > 0.7 * total_mem
    batches = [[gi] for gi in range(len(w.groups))] if per_group else [list(range(len(w.groups)))]
    res = []
    for i, gis in enumerate(batches):
        groups = [build_group(gm, w, gi, nsf, pool, dev) for gi in gis]
        args.codecs = i == 0
        r = measure(gm, w, groups, nsf, args, 1, local, not args.no_e2e)
        r["codec_bytes"] = codec_bytes(w, groups)
        res.append(r)
        del groups
        torch.cuda.empty_cache()
    out = {k: sum(r[k] for r in res) for k in ("ms_step", "ns_ms", "ns_flops", "ns_launches",
                                                 "cod_ms", "cub_ms", "cub_flops_dense",
                                                 "codec_bytes")}
    clk = [r["clocks"] for r in res if r["clocks"]]
    out["clocks"] = None
    if clk:
        out["clocks"] = {"sm_mhz": statistics.median([c["sm_mhz"] for c in clk]),
                         "sm_max_mhz": clk[0]["sm_max_mhz"],
                         "reasons": sorted(set(x for c in clk for x in c["reasons"])),
                         "samples": sum(c["samples"] for c in clk)}
    out["e2e"] = out["e2e_offload"] = None
    if not args.no_e2e:
        ms, h2d, d2h = e2e_resident(gm, w, nsf, args, 1, local)
        out["e2e"] = {"value": ms, "unit": UNIT, "h2d_bytes_per_step": int(h2d),
                      "d2h_bytes_per_step": int(d2h),
                      "api": "offload.HostStreamedStep per shape group with the weights and state "
                             "on the device: the pinned host gradients in, the chunks' device "
                             "statuses out, in chunks of B/8 matrices (rounded up) on three "
                             "streams shared by the groups (smallest first), 3 timed steps"}
    if all(r["e2e"] is not None for r in res):
        out["e2e_offload"] = {
            "value": sum(r["e2e"][0] for r in res), "unit": UNIT,
            "h2d_bytes_per_step": int(sum(r["e2e"][1] for r in res)),
            "d2h_bytes_per_step": int(sum(r["e2e"][2] for r in res)),
            "api": "offload.HostStreamedStep per shape group with the weights in pinned host memory "
                   "too: W and G in, the step, W out, in chunks of about 2^25 elements (at most "
                   "B/8 matrices) on three streams; groups one after another, set time = sum"}
    out["graph"] = ("one CUDA graph per gradient slot (each group's gm_grasp_step calls on "
                    "sub-batches of at most about 1e9 elements), one stream per shape group"
                    + ("; shape groups measured one at a time (device memory), set time = sum"
                       if per_group else ""))
    out["pool"] = pool
    out["codecs"] = res[0]["codecs"]
    out["launches"] = our_launches(gm, w, nsf) * args.steps
    # the same set with the Gram form on its non-square shapes (--ns auto), graph
    # replay only; batches whose forms do not change keep the time measured above
    out["ns_auto"] = None
    if args.ns == "standard" and not args.no_auto:
        auto = ns_chooser(gm, "auto")
        ms, clk_a = 0.0, []
        for gis, r in zip(batches, res):
            if all(auto(w.groups[gi].m, w.groups[gi].n) == nsf(w.groups[gi].m, w.groups[gi].n)
                   for gi in gis):
                ms += r["ms_step"]
                continue
            groups = [build_group(gm, w, gi, auto, pool, dev) for gi in gis]
            t, c, _, _ = time_steps(groups, args, 1, local)
            ms += t
            if c:
                clk_a.append(c["sm_mhz"])
            del groups
            torch.cuda.empty_cache()
        out["ns_auto"] = {
            "value": ms, "unit": UNIT,
            "ns_per_group": ["gram" if auto(g.m, g.n) == gm.GM_NS_GRAM else "standard"
                             for g in w.groups],
            "sm_mhz": statistics.median(clk_a) if clk_a else None,
            "what": "the same step and set with the Gram NS form (fp16) on non-square shapes "
                    "and the standard form on square ones (the Gram NS page's FLOP rule), "
                    "graph-replayed like the headline; not the headline"}
    return out


def run_sharded(gm, w, nsf, args, world, rank, local):
    """N > 1: the set split by ownership (sharding.ShardedStep: LPT owners, the
    owners' GRASP steps up to O, one NCCL all-gather of the bf16 O and skip
    flags per shape group, every rank's weight update; or, with --exchange
    weights, the owners' whole steps and an all-gather of the updated fp32
    weights), one shape group at a time; eager launches (the exchange is
    torch.distributed). Returns the max over ranks of the summed group times."""
    from bit_muon_optimizer_b200 import sharding as S
    dev = torch.device("cuda", local)
    update = S.grasp_update(w.eta, w.wd) if args.exchange in ("update", "peer") else None
    peer = args.exchange == "peer"
    ms_total, clocks, launches, owned = 0.0, [], 0, []
    for gi, g in enumerate(w.groups):
        base = w.group_base(gi)
        make = S.grasp_make_step(w.k, dev, mu=w.mu, eta=w.eta, wd=w.wd, T=w.T, ns=nsf(g.m, g.n),
                                 seed=w.seed)
        sh = S.ShardedStep([(g.m, g.n, g.count)], world, rank, make, first_index=base, update=update,
                           peer=peer)
        W = torch.empty((g.count, g.m, g.n), dtype=torch.float32, device=dev)
        grads = []
        for b in range(g.count):
            W[b] = WL.initial_weight(w, base + b, g.m, g.n, device=dev)
        for t in (1, 2):
            G = torch.empty((g.count, g.m, g.n), dtype=w.gdtype, device=dev)
            for b in range(g.count):
                WL.gradient(w, base + b, t, g.m, g.n, device=dev, out=G[b])
            grads.append(G)
        for t in range(args.warmup):
            sh([W], [grads[t % 2]])
        torch.cuda.synchronize()
        barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with ClockSampler(local) as clk:
            torch.cuda.synchronize()
            barrier(world)
            e0.record()
            for t in range(args.steps):
                sh([W], [grads[t % 2]])
            e1.record()
            torch.cuda.synchronize()
            barrier(world)
        ms_total += max_over_ranks(e0.elapsed_time(e1) / args.steps, world)
        if clk.summary():
            clocks.append(clk.summary())
        mine = len(sh.owned[0][rank])
        owned.append(mine)
        if mine:
            launches += our_launches(gm, w, nsf, [(mine, g.m, g.n)])   # the owner's sub-batch calls
        if update is not None:
            launches += 1                              # k_weight_update on every rank
        torch.cuda.synchronize()
        barrier(world)
        sh.close()           # unmap the other ranks' receive buffers before anyone frees them
        barrier(world)
        del sh, W, grads
        torch.cuda.empty_cache()
    clk = None
    if clocks:
        clk = {"sm_mhz": statistics.median([c["sm_mhz"] for c in clocks]),
               "sm_max_mhz": clocks[0]["sm_max_mhz"],
               "reasons": sorted(set(x for c in clocks for x in c["reasons"])),
               "samples": sum(c["samples"] for c in clocks)}
    return ms_total, clk, launches * args.steps, owned


def codec_issue(config: int, elements: int, ms: float, clocks):
    """The codec half against its instruction-issue bound: thread instructions per
    element (ncu) x elements / time, against 148 SMs x 4 schedulers x 32 lanes at
    the SM clock sampled during the timed region (the passes are issue-bound, not
    DRAM-bound). None without a matching capture or clock record."""
    ipe = codec_instr(config)
    if ipe is None or not clocks or not clocks.get("sm_mhz"):
        return None
    achieved = ipe * elements / (ms * 1e-3)
    peak = 148 * 4 * 32 * clocks["sm_mhz"] * 1e6
    return {"bound": "issue", "thread_instr_per_element": ipe, "achieved_tinstr_s": achieved,
            "peak_tinstr_s": peak, "frac": achieved / peak,
            "peak_kind": "148 SMs x 4 schedulers x 32 lanes x median SM clock of the timed region"}


def run_ours(args, world, rank, local):
    from bit_muon_optimizer_b200 import gmuon as gm
    w = WL.WORKLOADS[args.config]
    nsf = ns_chooser(gm, args.ns)
    hbm, bf16, bf16_sus, peak_kind = _peaks()
    elements = sum(g.count * g.m * g.n for g in w.groups)
    step_flops = sum(gm.ns_flops(nsf(g.m, g.n), g.m, g.n, w.T)[0] * g.count for g in w.groups)
    step_bytes = elements * FL.step_bytes_per_element(2 if w.gdtype != torch.float32 else 4)
    t_roof = max(step_flops / (bf16 * 1e12), step_bytes / (hbm * 1e9)) * 1e3
    config = {"workload": w.name, "ns": args.ns, "k": w.k,
              "shapes": [[g.m, g.n, g.count] for g in w.groups],
              "elements": elements, "grad_dtype": str(w.gdtype).replace("torch.", ""),
              "l2": "per-step working set (G, W, state, fp32 M) > L2; no flush"}
    modes = {nsf(g.m, g.n) for g in w.groups}
    dtype = "+".join(d for mode, d in ((gm.GM_NS_STANDARD, "bf16"), (gm.GM_NS_GRAM, "f16")) if mode in modes)
    if args.ns == "auto":
        config["ns_per_group"] = ["gram" if nsf(g.m, g.n) == gm.GM_NS_GRAM else "standard"
                                  for g in w.groups]
    if world > 1:
        ms_step, clocks, launches, owned = run_sharded(gm, w, nsf, args, world, rank, local)
        if rank == 0:
            what = {"update": "the owners' bf16 update directions O (2 B per element) and skip "
                              "flags, then every rank's weight update",
                    "peer": "none: the owners' last NS product stores O (bf16) and the skip flags "
                            "into every rank's receive buffers over NVLink (CUDA IPC), then every "
                            "rank's weight update",
                    "weights": "the owners' updated fp32 weights (4 B per element)"}[args.exchange]
            config.update(parallelism=f"ownership sharding x{world}: LPT owners per shape group, "
                                      f"exchange per group: {what}",
                          graph="eager launches, shape groups one at a time, set time = sum",
                          owned_per_group_rank0=owned)
            line = {"metric": METRIC, "value": ms_step, "unit": UNIT, "n_gpus": world,
                    "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
                    "higher_is_better": False, "scaling": "strong", "vs_baseline": None,
                    "dtype": dtype, "data": "synthetic", "config": config,
                    "step_roofline": {"ms": t_roof, "frac": t_roof / world / ms_step,
                                      "flops": step_flops, "bytes": step_bytes,
                                      "note": "single-GPU roofline / N"},
                    "gpu_launches": launches, "clocks": clocks, "e2e": None, "cpu_baseline": None}
            print(json.dumps(line), flush=True)
        return
    r = run_single(gm, w, nsf, args, local)
    ns_tflops = r["ns_flops"] / (r["ns_ms"] * 1e-3) / 1e12
    codec_gbs = r["codec_bytes"] / (r["cod_ms"] * 1e-3) / 1e9
    long_step = r["ms_step"] > 50.0
    peak = bf16_sus if long_step else bf16
    cpu = None
    if not args.no_cpu:
        ms_cpu, sample, cores = oracle_sample_seconds(w, args.ns)
        cpu = {"value": ms_cpu, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample}
    config.update(parallelism="single GPU", graph=r["graph"], grad_pool=r["pool"])
    line = {
        "metric": METRIC, "value": r["ms_step"], "unit": UNIT, "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": r["ms_step"],
        "higher_is_better": False, "scaling": "strong", "vs_baseline": None,
        "dtype": dtype, "data": "synthetic", "config": config,
        "roofline": {"bound": "tensor", "achieved": ns_tflops, "peak": peak, "unit": "TFLOP/s",
                     "frac": ns_tflops / peak, "traffic": gemm_traffic(args.config, args.ns),
                     "kernel": "k_gemm: the NS half of the step (gm_grasp_apply: "
                               f"{r['ns_launches']} tcgen05 products per step), CUDA events "
                               "around it on its launching stream",
                     "peak_kind": f"{peak_kind} bf16 dense "
                                  + ("sustained (kernel timed inside a step of "
                                     f"{r['ms_step']:.0f} ms)" if long_step else "burst")},
        "ns": {"tflops": ns_tflops, "ms": r["ns_ms"], "flops": r["ns_flops"],
               "frac_of_burst_peak": ns_tflops / bf16},
        "cublas_ns": {"ms": r["cub_ms"],
                      "tflops_algorithmic": r["ns_flops"] / (r["cub_ms"] * 1e-3) / 1e12
                      if args.ns == "standard" else None,
                      "tflops_dense": r["cub_flops_dense"] / (r["cub_ms"] * 1e-3) / 1e12,
                      "what": "standard NS, T steps of torch.matmul / baddbmm (cuBLAS bf16, "
                              "dense products), same inputs"},
        "codec": {"gbs": codec_gbs, "peak_gbs": hbm, "frac": codec_gbs / hbm, "ms": r["cod_ms"],
                  "bytes": r["codec_bytes"],
                  "kernels": "the codec half of the step (gm_grasp_state_update: 9 kernels per "
                             "call), CUDA events around each call; algorithmic bytes G + old and "
                             "new codes and scales + the 16-bit NS input",
                  "issue": codec_issue(args.config, elements, r["cod_ms"], r["clocks"])},
        "step_roofline": {"ms": t_roof, "frac": t_roof / r["ms_step"], "flops": step_flops,
                          "bytes": step_bytes},
        "standalone_codecs": dict(r["codecs"] or {}, peak_gbs=hbm,
                                  what="gm_group_quant4 / gm_group_dequant4 (4bit-Muon-base) and "
                                       "gm_mulaw_quant4 / gm_mulaw_dequant4 (MuonQ mu-law, mu = 255) "
                                       "on the first shape group's fp32 M_t; not part of the step"),
        "ns_auto": r["ns_auto"],
        "gpu_launches": r["launches"],
        "clocks": r["clocks"],
        "e2e": r["e2e"],
        "e2e_offload": r["e2e_offload"],
        "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)


def run_profile(args):
    """A fixed launch sequence for profilers: args.profile eager GRASP steps of
    each shape group (or of group args.group only), one group after the other,
    optionally with args.batch matrices instead of the group's count. No timing
    and no JSON line; the device status is checked after every group."""
    from bit_muon_optimizer_b200 import gmuon as gm
    w = WL.WORKLOADS[args.config]
    nsf = ns_chooser(gm, args.ns)
    dev = torch.device("cuda", 0)
    gis = range(len(w.groups)) if args.group < 0 else [args.group]
    for gi in gis:
        g = w.groups[gi]
        B = args.batch or g.count
        base = w.group_base(gi)
        # the bench's sub-batch calls, unless a batch size is given
        c = B if args.batch else sub_batches(B, g.m, g.n)
        step = gm.GraspStep(c, g.m, g.n, w.k, mu=w.mu, eta=w.eta, wd=w.wd, T=w.T, ns=nsf(g.m, g.n),
                            seed=w.seed, device=dev, matrix_ids=list(range(base, base + c)))
        st = gm.GraspState.zeros(B, g.m, g.n, w.k, dev)
        W = torch.empty((B, g.m, g.n), dtype=torch.float32, device=dev)
        G = torch.empty((B, g.m, g.n), dtype=w.gdtype, device=dev)
        for b in range(B):
            W[b] = WL.initial_weight(w, base + b, g.m, g.n, device=dev)
            WL.gradient(w, base + b, 1, g.m, g.n, device=dev, out=G[b])
        subs = [(a, min(B, a + c)) for a in range(0, B, c)]
        sts = [gm.GraspState(st.codes4[a:e], st.rscale[a:e], st.cscale[a:e], st.P8[a:e], st.Pscale[a:e],
                             st.R8[a:e], st.Rscale[a:e], torch.zeros(1, dtype=torch.int64, device=dev),
                             torch.zeros(1, dtype=torch.int32, device=dev)) for a, e in subs]
        if any(e - a != c for a, e in subs):
            raise ValueError("--profile: the sub-batches must be of equal size")
        ids = torch.arange(base, base + B, dtype=torch.int64, device=dev)
        for _ in range(args.profile):
            for (a, e), sst in zip(subs, sts):
                step.ids.copy_(ids[a:e])
                step(sst, W[a:e], G[a:e])
        torch.cuda.synchronize()
        bad = [int(s.dev_status.item()) for s in sts]
        if any(bad):
            raise RuntimeError(f"device status {bad}")
        print(f"profile: group {gi} ({g.m} x {g.n} x {B}, calls of {c}): {args.profile} steps", flush=True)
        del step, st, sts, W, G
        torch.cuda.empty_cache()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", type=int, default=4)
    ap.add_argument("--ns", choices=["standard", "gram", "auto"], default="standard",
                    help="NS form; auto: Gram NS for non-square shapes, standard for square ones")
    ap.add_argument("--exchange", choices=["update", "peer", "weights"], default="update",
                    help="N > 1: all-gather the bf16 update direction (default), store it into "
                         "every rank's buffers from the NS epilogue (peer), or all-gather the fp32 "
                         "weights")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-auto", action="store_true",
                    help="skip the extra timing of the set with Gram NS on non-square shapes")
    ap.add_argument("--profile", type=int, default=0,
                    help="run this many eager steps per shape group for a profiler, then exit")
    ap.add_argument("--group", type=int, default=-1, help="--profile: this shape group only")
    ap.add_argument("--batch", type=int, default=0, help="--profile: matrices per group")
    args = ap.parse_args()
    if args.profile:
        if torch.cuda.is_available():
            torch.cuda.set_device(0)
        run_profile(args)
        return
    if args.warmup < 3:
        args.warmup = 3
    world, rank, local = init_dist(args.gpus)
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            run_ours(args, world, rank, local)
    finally:
        if world > 1:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
