"""Benchmark of one GRASP optimizer step over a parameter set, on B200s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config 2] [--ns standard|gram]
                    [--impl ours|reference]

A "step" is one full GRASP step (rebuild, momentum, power iteration, 4/8-bit
re-quantization, Newton-Schulz, weight update) over every matrix of the
parameter set, with that step's synthetic gradients already resident in HBM.
Each shape group is one batched gm_grasp_step call; the three calls of a step
run on three streams and are replayed from a CUDA graph (one graph per step,
since each step has its own gradient buffer). N > 1 (torchrun): every rank
steps its own parameter set (weak scaling, no collective on the data path);
the time is the max over ranks.

Printed (rank 0): one JSON line with value = ms per parameter set for the
whole job, the NS chain's tensor-core roofline, the codec passes' HBM rate,
an end-to-end number through host buffers, and the fp64 CPU oracle timed on a
bounded sample as the CPU baseline.
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

def oracle_sample_seconds(w: WL.Workload, ns: str, budget_s: float):
    """Time the fp64 oracle on one matrix of every shape group, step 1 and 2,
    repeated until ~budget_s; returns (ms per parameter set, sample text, cores)."""
    import oracle as O
    per_shape = []
    t_all = time.perf_counter()
    for gi, g in enumerate(w.groups):
        m, n, k = g.m, g.n, w.k
        b = w.group_base(gi)
        st = O.zero_state(m, n, k)
        W = WL.initial_weight(w, b, m, n)
        times = []
        t = 1
        while True:
            G = WL.gradient(w, b, t, m, n)
            t0 = time.perf_counter()
            r = O.grasp_step(st, W, G, mu=w.mu, eta=w.eta, wd=w.wd, seed=w.seed, b=0, ns=ns, T=w.T)
            times.append(time.perf_counter() - t0)
            st, W = r.state, r.W.float()
            t += 1
            if t > 2 and (time.perf_counter() - t_all) > budget_s * (gi + 1) / len(w.groups):
                break
            if t > 6:
                break
        per_shape.append((g, statistics.median(times[1:] if len(times) > 1 else times)))
    ms = 1e3 * sum(g.count * s for g, s in per_shape)
    sample = ("fp64 oracle, one matrix per shape group ("
              + ", ".join(f"{g.m}x{g.n}" for g, _ in per_shape)
              + "), median of its steps 2+, extrapolated by the group counts")
    return ms, sample, torch.get_num_threads()


def run_reference(args, world, rank):
    """The reference arm: the fp64 CPU oracle as it stands, on this host's cores.

    Each step (warm-up or timed) is one oracle step of one sample matrix of
    every shape group, with each sample's state and weight carried from step
    to step, so the timed steps start from a warm quantized state like the
    GPU arm's; the step's time per parameter set is sum over groups of
    (matrices in the group) x (the sample's step time). The whole run costs
    (W + K) times one oracle step per group, about 0.4 s a step for LLaMA-130M.
    Only rank 0 works; the other ranks return at once."""
    if rank != 0:
        return
    import oracle as O
    w = WL.WORKLOADS[args.config]
    samples = []
    for gi, g in enumerate(w.groups):
        b = w.group_base(gi)
        samples.append([g, b, O.zero_state(g.m, g.n, w.k), WL.initial_weight(w, b, g.m, g.n)])
    vals = []
    for i in range(args.warmup + args.steps):
        t = i + 1
        ms = 0.0
        for smp in samples:
            g, b, st, W = smp
            G = WL.gradient(w, b, t, g.m, g.n)
            t0 = time.perf_counter()
            r = O.grasp_step(st, W, G, mu=w.mu, eta=w.eta, wd=w.wd, seed=w.seed, b=0, ns=args.ns,
                             T=w.T)
            ms += 1e3 * g.count * (time.perf_counter() - t0)
            smp[2], smp[3] = r.state, r.W.float()
        if i >= args.warmup:
            vals.append(ms)
    v = statistics.median(vals)
    cores = torch.get_num_threads()
    sample = ("fp64 oracle, one matrix per shape group ("
              + ", ".join(f"{g.m}x{g.n}" for g, _, _, _ in samples)
              + "), one step of each per reference step from a state carried across steps, "
              "extrapolated by the group counts; median over the timed steps")
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": v, "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "ns": args.ns, "k": w.k, "matrices": sum(g.count for g in w.groups)},
        "cpu_baseline": {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ GPU arm

GRAD_POOL = 6   # distinct gradient buffers per group, used cyclically step after step

# DRAM bytes per k_gemm launch (average over one step's 45 NS products of the
# LLaMA-130M set, standard NS), from an ncu capture of dram__bytes_read.sum +
# dram__bytes_write.sum (the k_gemm summary under profiles/); reported only while
# gm_gemm.cu is the source that capture measured.
GEMM_TRAFFIC = {"config": 2, "ns": "standard", "bytes_per_launch": 87.56e6,
                "source_sha256": "aa52586b7c8ef53cef64f66392279f880c35c449ce72813d6b82ec7d5a190d0a"}


def gemm_traffic(config: int, ns: str):
    import hashlib
    path = os.path.join(ROOT, "bit_muon_optimizer_b200", "csrc", "gm_gemm.cu")
    try:
        with open(path, "rb") as f:
            sha = hashlib.sha256(f.read()).hexdigest()
    except OSError:
        return None
    t = GEMM_TRAFFIC
    if sha != t["source_sha256"] or config != t["config"] or ns != t["ns"]:
        return None
    return t["bytes_per_launch"]


def est_bytes(w: WL.Workload, pool: int) -> int:
    """Device bytes of the benchmark per parameter-set element: fp32 W, the
    gradient pool, the step workspace (fp32 M, the 16-bit iterate, NS buffers),
    and the separately timed NS / codec passes (fp32 O, their workspace, codes)."""
    elems = sum(g.count * g.m * g.n for g in w.groups)
    return elems * (22 + 2 * pool)


def matrix_base(w: WL.Workload, gi: int, rank: int) -> int:
    """Index of the first matrix of shape group gi in rank's parameter set: rank r
    steps matrices r * count ... (r + 1) * count - 1 of the workload's sequence."""
    return rank * sum(x.count for x in w.groups) + w.group_base(gi)


def build_group(gm, w: WL.Workload, gi: int, ns_mode: int, rank: int, pool: int, dev):
    g = w.groups[gi]
    B, m, n = g.count, g.m, g.n
    base = matrix_base(w, gi, rank)
    step = gm.GraspStep(B, m, n, w.k, mu=w.mu, eta=w.eta, wd=w.wd, T=w.T, ns=ns_mode,
                        seed=w.seed + rank, device=dev)
    st = gm.GraspState.zeros(B, m, n, w.k, dev)
    W = torch.empty((B, m, n), dtype=torch.float32, device=dev)
    for b in range(B):
        W[b] = WL.initial_weight(w, base + b, m, n, device=dev)
    grads = []
    for t in range(1, pool + 1):
        G = torch.empty((B, m, n), dtype=w.gdtype, device=dev)
        for b in range(B):
            WL.gradient(w, base + b, t, m, n, device=dev, out=G[b])
        grads.append(G)
    return dict(step=step, st=st, W=W, grads=grads, B=B, m=m, n=n)


def measure(gm, w, groups, ns_mode, args, world, local, do_e2e):
    """Times args.steps graph-replayed GRASP steps over `groups` (each group on
    its own stream), then the NS chains and the codec passes alone, then (if
    asked) steps end to end through pinned host buffers."""
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
    fork(lambda g: g["step"](g["st"], g["W"], g["grads"][0]))
    torch.cuda.synchronize()
    graphs = []
    for t in range(npool):
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, stream=main):
            fork(lambda g, t=t: g["step"](g["st"], g["W"], g["grads"][t]))
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
    status = [int(g["st"].dev_status.item()) for g in groups]
    if any(status):
        raise RuntimeError(f"device status {status}")
    del graphs

    # ---- NS chain alone (tensor-core roofline) and codec passes alone (HBM), each
    # replayed from a graph with the groups on their own streams, as in the step
    def graph_ms(enqueue, reps):
        fork(enqueue)                            # eager once (attributes, workspaces)
        torch.cuda.synchronize()
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, stream=main):
            fork(enqueue)
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(main):       # replay on the stream the events are recorded on
            for _ in range(3):
                gr.replay()
            torch.cuda.synchronize()
            s0.record(main)
            for _ in range(reps):
                gr.replay()
            s1.record(main)
        torch.cuda.synchronize()
        del gr
        return s0.elapsed_time(s1) / reps

    for g in groups:
        g["Mx"] = g["step"].stage_M()            # the last step's fp32 M_t, read-only below
        g["O"] = torch.empty_like(g["Mx"])       # NS output, then the codec's rebuilt M
        g["ws_ns"] = torch.empty(gm.workspace_bytes(gm.GM_OP_GRAM_NS if ns_mode == gm.GM_NS_GRAM
                                                    else gm.GM_OP_NEWTON_SCHULZ, g["B"], g["m"], g["n"]),
                                 dtype=torch.uint8, device=dev)
        g["codes"] = (torch.empty_like(g["st"].codes4), torch.empty_like(g["st"].rscale),
                      torch.empty_like(g["st"].cscale))

    def ns_enqueue(g):
        if ns_mode == gm.GM_NS_GRAM:
            gm.gram_ns(g["Mx"], T=w.T, out=g["O"], ws=g["ws_ns"])
        else:
            gm.newton_schulz(g["Mx"], T=w.T, out=g["O"], ws=g["ws_ns"])

    def codec_enqueue(g):
        st = g["st"]
        gm.dequant_rebuild(st.codes4, st.rscale, st.cscale, st.P8, st.Pscale, st.R8, st.Rscale,
                           out=g["O"])
        gm.grid_quant4(g["Mx"], g["step"].stage_P(), g["step"].stage_R(), out=g["codes"])

    reps = 20 if sum(g["B"] * g["m"] * g["n"] for g in groups) < 5e8 else 5
    ns_ms = graph_ms(ns_enqueue, reps)
    ns_flops = sum(gm.ns_flops(ns_mode, g["m"], g["n"], w.T)[0] * g["B"] for g in groups)
    cod_ms = graph_ms(codec_enqueue, reps)

    # comparator: the same standard NS chain written with torch.matmul (cuBLAS,
    # bf16, no symmetry), on the same normalised wide-form inputs
    abc = [(3.4445, -4.7750, 2.0315)] * w.T
    for g in groups:
        g["Xc"] = g["step"].stage_X().to(torch.bfloat16).clone()
        g["Xw"] = torch.empty_like(g["Xc"])

    def cublas_enqueue(g):
        X = g["Xc"]
        for a, b_, c in abc:
            A = torch.matmul(X, X.mT)
            B = torch.baddbmm(A, A, A, beta=b_, alpha=c)
            X = torch.baddbmm(X, B, X, beta=a, alpha=1.0)
        g["Xw"].copy_(X)

    cub_ms = graph_ms(cublas_enqueue, reps)
    cub_flops_dense = sum(T_ * g["B"] * (2.0 * min(g["m"], g["n"]) ** 2 * max(g["m"], g["n"]) * 2
                                         + 2.0 * min(g["m"], g["n"]) ** 3)
                          for g in groups for T_ in [w.T])
    for g in groups:
        del g["Xc"], g["Xw"]
    # algorithmic bytes: rebuild reads codes + scales and writes fp32 M; quant reads fp32 M
    # and writes codes + scales (the k (m + n) factor bytes are ignored)
    cod_bytes = sum(2 * g["B"] * g["m"] * g["n"] * (4 + 0.5 + 0.0625) for g in groups)
    for g in groups:
        del g["Mx"], g["O"], g["ws_ns"], g["codes"]

    # ---- end to end through host buffers: H2D W and G, the step, D2H W
    e2e = None
    if do_e2e:
        host = []
        for g in groups:
            host.append(dict(W=g["W"].cpu().pin_memory(), G=g["grads"][-1].cpu().pin_memory()))
        h2d = sum(h["W"].numel() * 4 + h["G"].numel() * h["G"].element_size() for h in host)
        d2h = sum(h["W"].numel() * 4 for h in host)
        Wd = [torch.empty_like(g["W"]) for g in groups]
        Gd = [torch.empty_like(g["grads"][-1]) for g in groups]
        e_steps = max(2, min(args.steps, 5))
        torch.cuda.synchronize()
        barrier(world)
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record()
        for _ in range(e_steps):
            for g, h, wd_, gd_ in zip(groups, host, Wd, Gd):
                wd_.copy_(h["W"], non_blocking=True)
                gd_.copy_(h["G"], non_blocking=True)
                g["step"](g["st"], wd_, gd_)
                h["W"].copy_(wd_, non_blocking=True)
        s1.record()
        torch.cuda.synchronize()
        barrier(world)
        e2e = (max_over_ranks(s0.elapsed_time(s1) / e_steps, world), h2d, d2h)
    return dict(ms_step=ms_step, clocks=clk.summary(), ns_ms=ns_ms, ns_flops=ns_flops,
                cod_ms=cod_ms, cod_bytes=cod_bytes, e2e=e2e, cub_ms=cub_ms,
                cub_flops_dense=cub_flops_dense)


def run_ours(args, world, rank, local):
    from bit_muon_optimizer_b200 import gmuon as gm
    dev = torch.device("cuda", local)
    w = WL.WORKLOADS[args.config]
    ns_mode = gm.GM_NS_GRAM if args.ns == "gram" else gm.GM_NS_STANDARD
    hbm, bf16, bf16_sus, peak_kind = _peaks()
    total_mem = torch.cuda.get_device_properties(dev).total_memory
    pool = min(GRAD_POOL, args.warmup + args.steps)
    if est_bytes(w, pool) > 0.7 * total_mem:
        pool = 2
    # a set too large to hold at once is measured one shape group at a time; the
    # groups are independent and each fills the GPU, so the set's time is the sum
    per_group = est_bytes(w, pool) > 0.7 * total_mem
    batches = [[gi] for gi in range(len(w.groups))] if per_group else [list(range(len(w.groups)))]
    do_e2e = not args.no_e2e and not per_group
    res = []
    for gis in batches:
        groups = [build_group(gm, w, gi, ns_mode, rank, pool, dev) for gi in gis]
        res.append(measure(gm, w, groups, ns_mode, args, world, local, do_e2e))
        del groups
        torch.cuda.empty_cache()
    ms_step = sum(r["ms_step"] for r in res)
    ns_ms = sum(r["ns_ms"] for r in res)
    ns_flops = sum(r["ns_flops"] for r in res)
    cod_ms = sum(r["cod_ms"] for r in res)
    cod_bytes = sum(r["cod_bytes"] for r in res)
    cub_ms = sum(r["cub_ms"] for r in res)
    cub_dense = sum(r["cub_flops_dense"] for r in res)
    ns_tflops = ns_flops / (ns_ms * 1e-3) / 1e12
    codec_gbs = cod_bytes / (cod_ms * 1e-3) / 1e9
    clk = [r["clocks"] for r in res if r["clocks"]]
    clocks = None
    if clk:
        clocks = {"sm_mhz": statistics.median([c["sm_mhz"] for c in clk]),
                  "sm_max_mhz": clk[0]["sm_max_mhz"],
                  "reasons": sorted(set(x for c in clk for x in c["reasons"])),
                  "samples": sum(c["samples"] for c in clk)}
    e2e = None
    if res[0]["e2e"] is not None:
        e_ms, h2d, d2h = res[0]["e2e"]
        e2e = {"value": e_ms / world, "unit": UNIT, "h2d_bytes_per_step": int(h2d),
               "d2h_bytes_per_step": int(d2h)}

    # ---- our kernels launched per step: per group 9 codec kernels (column norms,
    # warm start with the factor fragments, rebuild + projection, three
    # orthonormalisation kernels, back projection, its finalisation, the 4-bit
    # quantisation with the 8-bit one folded in), the NS products, and the
    # zero-padding copy when a dimension is not a multiple of 64
    launches = 0
    for g in w.groups:
        pad = int(min(g.m, g.n) % 64 != 0 or max(g.m, g.n) % 64 != 0)
        launches += 9 + gm.ns_flops(ns_mode, g.m, g.n, w.T)[1] + pad
    launches *= args.steps

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        ms_cpu, sample, cores = oracle_sample_seconds(w, args.ns, 20.0)
        cpu = {"value": ms_cpu, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample}

    elements = sum(g.count * g.m * g.n for g in w.groups)
    step_flops = sum(gm.ns_flops(ns_mode, g.m, g.n, w.T)[0] * g.count for g in w.groups)
    step_bytes = elements * FL.step_bytes_per_element(2 if w.gdtype != torch.float32 else 4)
    t_roof = max(step_flops / (bf16 * 1e12), step_bytes / (hbm * 1e9)) * 1e3
    if rank == 0:
        line = {
            "metric": METRIC, "value": ms_step / world, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": False, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if ns_mode == gm.GM_NS_STANDARD else "f16",
            "data": "synthetic",
            "config": {"workload": w.name, "ns": args.ns, "k": w.k,
                       "shapes": [[g.m, g.n, g.count] for g in w.groups],
                       "elements": elements, "grad_dtype": str(w.gdtype).replace("torch.", ""),
                       "l2": "per-step working set (G, W, state, fp32 M) > L2; no flush",
                       "parallelism": f"weak x{world}, one parameter set per rank",
                       "graph": ("one CUDA graph per gradient slot, one stream per shape group"
                                 + ("; shape groups measured one at a time (device memory), "
                                    "set time = sum" if per_group else "")),
                       "grad_pool": pool},
            "roofline": {"bound": "tensor", "achieved": ns_tflops, "peak": bf16, "unit": "TFLOP/s",
                         "frac": ns_tflops / bf16, "traffic": gemm_traffic(args.config, args.ns),
                         "kernel": "k_gemm: the NS chains' tcgen05 products of all groups, graph-replayed alone",
                         "peak_kind": f"{peak_kind} bf16 dense burst"},
            "ns": {"tflops": ns_tflops, "ms": ns_ms, "flops": ns_flops},
            "cublas_ns": {"ms": cub_ms, "tflops_algorithmic": ns_flops / (cub_ms * 1e-3) / 1e12
                          if args.ns == "standard" else None,
                          "tflops_dense": cub_dense / (cub_ms * 1e-3) / 1e12,
                          "what": "standard NS, T steps of torch.matmul / baddbmm (cuBLAS bf16, "
                                  "dense products), same inputs and streams"},
            "codec": {"gbs": codec_gbs, "peak_gbs": hbm, "frac": codec_gbs / hbm,
                      "ms": cod_ms,
                      "kernels": "rebuild (k_dequant_rebuild) + residual grid quantisation "
                                 "(k_residual_quant4) through the standalone entry points, "
                                 "which stage the factor fragments in each CTA"},
            "step_minus_ns_ms": ms_step - ns_ms,
            "step_roofline": {"ms": t_roof, "frac": t_roof / ms_step, "flops": step_flops,
                              "bytes": step_bytes},
            "gpu_launches": launches,
            "clocks": clocks,
            "e2e": e2e,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", type=int, default=2)
    ap.add_argument("--ns", choices=["standard", "gram"], default="standard")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    args = ap.parse_args()
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
