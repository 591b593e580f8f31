#!/usr/bin/env python
"""Benchmark of the fused low-bit GEMM on B200.

Headline: ternary low-bit W.A GEMM at M=4608 tokens (1024x1024 image + 512
text tokens), K=3072, N=9216 (MLP-up of a hidden-3072 MMDiT block), in
FP16-equivalent TFLOP/s (2*M*N*K per launch) and as a fraction of the
tensor-core roofline.  A step is one call of bonsai_lowbit_gemm: TMA staging,
unpack + scale, tcgen05 MMA and the FP16 epilogue.  The weights are packed
once before timing (packing is an offline, once-per-weight step); the
small-M line reports the bandwidth-bound regime (M=16, ternary MLP-down
3072x9216) in GB/s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl bonsai|reference]

Under torchrun each rank runs an independent replica of the same per-GPU
workload (weak scaling, no collective on the data path); the timed region
is bracketed by barriers and the slowest rank's time is reported.
`--impl reference` times the CPU oracle on bounded samples of the same
workload on this host's cores (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

WORKLOAD = workloads.TERNARY_MLP_UP_4608
SMALL = [workloads.TERNARY_MLP_DOWN_16, workloads.TERNARY_QKV_16]
METRIC = "low-bit W.A GEMM TFLOP/s (M=4608,K=3072,N=9216 ternary)"
UNIT = "TFLOP/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["bonsai", "reference"], default="bonsai")
    ap.add_argument("--sets", type=int, default=4, help="rotating input sets (their sum exceeds L2)")
    ap.add_argument("--no-extras", action="store_true", help="skip small-M, e2e, CPU baseline, clocks")
    ap.add_argument("--small-only", action="store_true", help="time only the M=16 workload (for profiling)")
    ap.add_argument("--offline-only", action="store_true", help="time only pack and dequant (for profiling)")
    ap.add_argument("--layers-only", action="store_true", help="time only the single-stream layer shapes")
    ap.add_argument("--case", default=None,
                    help="run one configuration --launches times, untimed (the command the committed ncu summaries "
                         "profile): MODE:M:N:K for the GEMM (MODE binary, ternary, ternary_b3 or hqq4), "
                         "pack-MODE:N:K, dequant-MODE:N:K, or batch-MODE:M:N:K:L for L layers in one batch call")
    ap.add_argument("--launches", type=int, default=3)
    ap.add_argument("--m-sweep", action="store_true",
                    help="time the GEMM over M = 16..4608 on the stack's five layer shapes and print one JSON line")
    return ap.parse_args()


def flops(p) -> int:
    return 2 * p.M * p.N * p.K


def packed_weight_bytes(mode, N, K) -> int:
    """Packed weight bytes: K/8 (binary), K/4 (INT2) or 112 per 512 weights
    (base-3 blocks) per row."""
    if mode == "ternary_b3":
        return N * 112 * -(-(K // 128) // 4)
    return N * K // (8 if mode == "binary" else 4)


def algorithmic_bytes(p) -> int:
    """Packed weights + FP16 scales + FP16 activations in + FP16 output."""
    return packed_weight_bytes(p.mode, p.N, p.K) + 2 * p.N * (p.K // 128) + 2 * p.M * p.K + 2 * p.M * p.N


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "bit_weight_gemm_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel_key: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel sources; else None."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except (OSError, ValueError):
        return None
    e = d.get(kernel_key)
    if not e or e.get("source_hash") != kernel_source_hash():
        return None
    return e.get("dram_bytes_per_launch")


# ------------------------------------------------------------------ clocks
class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()
        time.sleep(0.3)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for name, flag in zip(names, parts[5:9]):
                if flag.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# --------------------------------------------------------------- helpers
def max_over_ranks(torch, seconds: float, dist=None, device="cuda") -> float:
    """The slowest rank's time: every rank contributes its own device time."""
    t = torch.tensor([seconds], dtype=torch.float64, device=device)
    if dist is not None:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(work_per_step: float, steps: int, world: int, seconds_max: float) -> float:
    """Aggregate throughput: every rank ran `steps` steps of the same work
    (weak scaling), in the slowest rank's time."""
    return work_per_step * steps * world / seconds_max


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def cpu_baseline(problem, budget_s: float = 15.0, rows: int = 512):
    """The oracle, as it stands, on a bounded sample of the workload: `rows`
    token rows against as many weight rows as fit the time budget."""
    import oracle

    d = workloads.make(problem)
    packed = oracle.pack(d["codes"], problem.mode)
    threads = oracle.default_threads()
    # calibrate on a small block, then size the sample to the budget
    n_cal = 256
    t0 = time.perf_counter()
    oracle.gemm(d["A"][:rows], packed[:n_cal], d["scales"][:n_cal], problem.K, problem.mode, threads=threads,
                want_acc=False)
    t_cal = time.perf_counter() - t0
    n = int(min(problem.N, max(n_cal, n_cal * budget_s / max(t_cal, 1e-3))))
    t0 = time.perf_counter()
    oracle.gemm(d["A"][:rows], packed[:n], d["scales"][:n], problem.K, problem.mode, threads=threads,
                want_acc=False)
    dt = time.perf_counter() - t0
    value = 2 * rows * n * problem.K / dt / 1e12
    return {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{rows} token rows x {n} weight rows x K={problem.K} of {problem.name} "
                      f"({dt:.1f} s, C oracle, double accumulation, {threads} threads)"}


# ------------------------------------------------------------- reference
def run_reference(args):
    world, rank, _ = dist_setup(args)
    if rank != 0:
        return 0
    import oracle

    p = WORKLOAD
    d = workloads.make(p)
    packed = oracle.pack(d["codes"], p.mode)
    threads = oracle.default_threads()
    # 128 token rows per step: the oracle converts each weight row it uses to
    # double once per call, which 16 rows would leave dominating the step
    rows, n_blk = 128, 128
    # size each step so that warm-up + timed steps end within ~2.5 minutes
    t0 = time.perf_counter()
    oracle.gemm(d["A"][:rows], packed[:n_blk], d["scales"][:n_blk], p.K, p.mode, threads=threads, want_acc=False)
    t_blk = time.perf_counter() - t0
    per_step = 150.0 / max(1, args.steps + args.warmup)
    n_blk = int(max(8, min(p.N, n_blk * per_step / max(t_blk, 1e-4))))
    n_tiles = max(1, p.N // n_blk)

    def step(i):
        m0 = (i * rows) % (p.M - rows)
        n0 = (i % n_tiles) * n_blk
        oracle.gemm(d["A"][m0:m0 + rows], packed[n0:n0 + n_blk], d["scales"][n0:n0 + n_blk], p.K, p.mode,
                    threads=threads, want_acc=False)

    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        step(args.warmup + i)
    dt = time.perf_counter() - t0
    value = 2 * rows * n_blk * p.K * args.steps / dt / 1e12
    sample = (f"each step: {rows} token rows x {n_blk} weight rows x K={p.K} of {p.name}, "
              f"C oracle with double accumulation on {threads} threads")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": p.name, "M": p.M, "N": p.N, "K": p.K, "mode": p.mode, "group": 128},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- bonsai
def make_sets(problem, count, torch, bw, distinct_weights=True):
    """`count` input sets on the device.  Each set has its own buffers; with
    distinct_weights the codes differ too (seed + i)."""
    sets = []
    base = None
    for i in range(count):
        if distinct_weights or base is None:
            d = workloads.make(mode=problem.mode, M=problem.M, N=problem.N, K=problem.K, seed=problem.seed + 100 * i)
            A = torch.from_numpy(d["A"].view(np.int16)).view(torch.float16).cuda()
            s = torch.from_numpy(d["scales"].view(np.int16)).view(torch.float16).cuda()
            packed = bw.pack(torch.from_numpy(d["codes"]).cuda(), problem.mode)
            base = (A, packed, s)
        else:
            A, packed, s = (t.clone() for t in base)
        out = torch.empty((problem.M, problem.N), dtype=torch.float16, device="cuda")
        sets.append((A, packed, s, out))
    torch.cuda.synchronize()
    return sets


def time_launches(torch, bw, problem, sets, steps, warmup, dist=None):
    """Device time of `steps` back-to-back launches, rotating over the input
    sets.  The launches are replayed from a captured CUDA graph (one pass
    over the sets per replay), as a serving loop would, so host-side call
    overhead does not show up as idle GPU time; CUDA events on the replay
    stream bracket the timed region."""
    def launch(i):
        A, p, s, o = sets[i % len(sets)]
        bw.lowbit_gemm(A, p, s, problem.mode, out=o)

    for i in range(max(warmup, 1)):  # also sets kernel attributes and caches before capture
        launch(i)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for i in range(len(sets)):
            launch(i)
    graph.replay()
    reps, rest = divmod(steps, len(sets))
    stream = torch.cuda.current_stream()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for _ in range(reps):
        graph.replay()
    for i in range(rest):
        launch(i)
    end.record(stream)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    del graph
    return start.elapsed_time(end) / 1e3  # seconds


def run_bonsai(args):
    import torch

    world, rank, local = dist_setup(args)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as tdist

        torch.cuda.set_device(local)
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local))
        dist = tdist
    else:
        torch.cuda.set_device(0)

    import bit_weight_gemm_b200 as bw

    bw.lib()
    peaks, peaks_kind = load_peaks()
    p = WORKLOAD

    cpu = None
    if rank == 0 and world == 1 and not args.no_extras and not args.small_only:
        cpu = cpu_baseline(p)  # before the first GPU work: the oracle runs threads, no fork

    result = {}
    if not args.small_only:
        sets = make_sets(p, args.sets, torch, bw)
        sampler = ClockSampler(local) if not args.no_extras else None
        if sampler:
            sampler.start()
        secs = time_launches(torch, bw, p, sets, args.steps, args.warmup, dist)
        clocks = sampler.stop() if sampler else None
        secs_max = max_over_ranks(torch, secs, dist)
        per_launch = secs_max / args.steps
        value = whole_job_rate(flops(p), args.steps, world, secs_max) / 1e12
        peak = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
        achieved = flops(p) / per_launch / 1e12
        result.update(value=value, ms_per_step=per_launch * 1e3, clocks=clocks, achieved=achieved, peak=peak)
        del sets

        e2e = None
        if not args.no_extras:
            e2e = time_e2e(torch, bw, p, min(args.steps, 50), 3, dist)
        result["e2e"] = e2e

    small = small_batch = None
    if not args.no_extras or args.small_only:
        small = [time_small(torch, bw, sp, args, dist, peaks, peaks_kind) for sp in SMALL]
        small_batch = time_small_batch(torch, bw, args, dist, peaks, peaks_kind)
    stack = None
    if not args.no_extras and not args.small_only:
        stack = [time_stack(torch, bw, m, "ternary", 20, 3) for m in (4608, 1024)]
        stack.append(time_stack(torch, bw, 4608, "ternary", 20, 3, split_qkv=True))
        stack += [time_stack(torch, bw, None, "ternary", 20, 3, streams=st) for st in ((4096, 512), (1024, 512))]
        stack += [time_stack(torch, bw, m, "binary", 20, 3) for m in (4608, 1024)]
    layers = None
    if not args.no_extras and not args.small_only:
        layers = time_layers(torch, bw, args, dist)
    cublas = None
    formats = None
    offline = None
    if not args.no_extras and not args.small_only:
        cublas = cublas_fp16_same_run(torch)
        formats = time_formats(torch, bw, args, dist, peaks, peaks_kind)
        offline = time_pack_dequant(torch, bw, p, peaks, peaks_kind)

    if dist is not None:
        dist.barrier()
    if rank == 0:
        if args.small_only:
            print(json.dumps({"small_m": small, "small_m_batch": small_batch}), flush=True)
        else:
            traffic = ncu_traffic(f"{p.mode}_M{p.M}_N{p.N}_K{p.K}")
            line = {
                "metric": METRIC, "value": result["value"], "unit": UNIT, "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": result["ms_per_step"], "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f16", "data": "synthetic",
                "config": {"workload": p.name, "M": p.M, "N": p.N, "K": p.K, "mode": p.mode, "group": 128,
                           "plan": bw.gemm_plan(p.M, p.N, p.K, p.mode), "parallelism": f"replicas{world}",
                           "l2": f"{args.sets} rotating input sets, {args.sets * (algorithmic_bytes(p)) / 1e6:.0f} MB "
                                 f"total > 126 MB L2"},
                "roofline": {"bound": "tensor", "achieved": result["achieved"], "peak": result["peak"],
                             "unit": "TFLOP/s", "frac": result["achieved"] / result["peak"],
                             "traffic": traffic, "peak_source": f"{peaks_kind} bf16 dense (fp16 same nominal rate)",
                             "cublas_fp16_same_run": cublas},
                "gpu_launches": args.steps,
                "timing": "CUDA graph replay of the launches, CUDA events on the replay stream",
                "clocks": result["clocks"],
                "e2e": result["e2e"],
                "cpu_baseline": cpu,
                "small_m": small,
                "small_m_batch": small_batch,
                "stack": stack,
                "layers": layers,
                "formats": formats,
                "pack_dequant": offline,
            }
            print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()
    return 0


def time_e2e(torch, bw, p, steps, warmup, dist):
    """Host buffers in, host buffers out, through the public API: per step one
    bonsai_lowbit_gemm_host call, which copies A in from pinned host memory,
    runs the GEMM and copies out back, chunked so that the copies in both
    directions overlap the GEMMs."""
    d = workloads.make(p)
    A_host = torch.from_numpy(d["A"].view(np.int16)).view(torch.float16).pin_memory()
    out_host = torch.empty((p.M, p.N), dtype=torch.float16).pin_memory()
    s = torch.from_numpy(d["scales"].view(np.int16)).view(torch.float16).cuda()
    packed = bw.pack(torch.from_numpy(d["codes"]).cuda(), p.mode)
    A_dev = torch.empty((p.M, p.K), dtype=torch.float16, device="cuda")
    out_dev = torch.empty((p.M, p.N), dtype=torch.float16, device="cuda")
    stream = torch.cuda.current_stream()

    def step():
        bw.lowbit_gemm_host(A_host, packed, s, p.mode, out_host=out_host, A_dev=A_dev, out_dev=out_dev)

    for _ in range(warmup):
        step()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for _ in range(steps):
        step()
    end.record(stream)
    torch.cuda.synchronize()
    secs = start.elapsed_time(end) / 1e3
    world = dist.get_world_size() if dist is not None else 1
    secs_max = max_over_ranks(torch, secs, dist)
    return {"value": whole_job_rate(flops(p), steps, world, secs_max) / 1e12, "unit": UNIT,
            "h2d_bytes_per_step": 2 * p.M * p.K, "d2h_bytes_per_step": 2 * p.M * p.N, "steps": steps,
            "api": "bonsai_lowbit_gemm_host, pinned host buffers, copies overlapped with the GEMMs in row chunks"}


def time_small(torch, bw, p, args, dist, peaks, peaks_kind):
    """Bandwidth-bound regime: M=16.  64 rotating copies of the inputs
    (about 500 MB, 4x L2) so that every launch reads its weights from HBM."""
    sets = make_sets(p, 64, torch, bw, distinct_weights=False)
    steps = max(args.steps, 200)
    secs = time_launches(torch, bw, p, sets, steps, max(args.warmup, 10), dist)
    per_launch = max_over_ranks(torch, secs, dist) / steps
    nbytes = algorithmic_bytes(p)
    achieved = nbytes / per_launch / 1e9
    peak = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    del sets
    return {"workload": p.name, "M": p.M, "N": p.N, "K": p.K, "plan": bw.gemm_plan(p.M, p.N, p.K, p.mode),
            "value": achieved, "unit": "GB/s",
            "us_per_launch": per_launch * 1e6, "tflops": flops(p) / per_launch / 1e12,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": ncu_traffic(f"{p.mode}_M{p.M}_N{p.N}_K{p.K}"),
                         "algorithmic_bytes_per_launch": nbytes, "peak_source": f"{peaks_kind} hbm copy"},
            "gpu_launches": steps}


BATCH_LAYERS = 80  # one denoise step's worth of linears per call


def time_small_batch(torch, bw, args, dist, peaks, peaks_kind):
    """The bandwidth-bound regime with many layers per call: 80 independent
    16-token GEMMs in one bonsai_lowbit_gemm_batch call (one persistent
    launch), each layer with its own buffers (633-752 MB in all, 5-6x L2, so
    every weight byte comes from HBM).  Three batches: 80 MLP-down layers
    (3072x9216), 80 fused-QKV layers (9216x3072), and the 80 linears of one
    denoise step; then the two repeated-layer batches with binary weights and
    MLP-down with base-3 ternary weights.  GB/s of algorithmic bytes (packed weights, scales,
    activations, outputs of all layers) per call; the call is replayed from a
    CUDA graph and timed with CUDA events on the replay stream."""
    out = []
    step_layers = [(n, k) for _, n, k in workloads.mmdit_stack_layers()]
    down = [(SMALL[0].N, SMALL[0].K)] * BATCH_LAYERS
    qkv = [(SMALL[1].N, SMALL[1].K)] * BATCH_LAYERS
    cases = [("ternary MLP-down M=16 x 80 layers", "ternary", down, SMALL[0].seed),
             ("ternary fused QKV M=16 x 80 layers", "ternary", qkv, SMALL[1].seed),
             ("ternary denoise-step linears M=16 (80 layers)", "ternary", step_layers, 3000),
             ("binary MLP-down M=16 x 80 layers", "binary", down, SMALL[0].seed),
             ("binary fused QKV M=16 x 80 layers", "binary", qkv, SMALL[1].seed),
             ("base-3 ternary MLP-down M=16 x 80 layers", "ternary_b3", down, SMALL[0].seed)]
    for name, mode, shapes, seed in cases:
        base = {}
        probs, nbytes = [], 0
        for j, (n, k) in enumerate(shapes):
            p = workloads.Problem(name, mode, 16, n, k, seed + j)
            if (n, k) not in base:
                d = workloads.make(p)
                base[(n, k)] = (torch.from_numpy(d["A"].view(np.int16)).view(torch.float16).cuda(),
                                bw.pack(torch.from_numpy(d["codes"]).cuda(), mode),
                                torch.from_numpy(d["scales"].view(np.int16)).view(torch.float16).cuda())
            A, packed, sc = (t.clone() for t in base[(n, k)])  # own buffers: every layer reads its own bytes
            probs.append((A, packed, sc))
            nbytes += algorithmic_bytes(p)
        outs = [torch.empty((16, n), dtype=torch.float16, device="cuda") for n, _ in shapes]
        torch.cuda.synchronize()

        def call():
            bw.lowbit_gemm_batch(probs, mode, outs=outs)

        for _ in range(max(args.warmup, 3)):
            call()
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            call()
        graph.replay()
        steps = 50
        stream = torch.cuda.current_stream()
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        start.record(stream)
        for _ in range(steps):
            graph.replay()
        end.record(stream)
        torch.cuda.synchronize()
        del graph
        per_call = max_over_ranks(torch, start.elapsed_time(end) / 1e3, dist) / steps
        achieved = nbytes / per_call / 1e9
        peak = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
        flop = sum(2 * 16 * n * k for n, k in shapes)
        # DRAM bytes: captured per layer on a 24-layer batch of one shape, times the layers
        per_layer = ncu_traffic(f"batch_{mode}_M16_N{shapes[0][0]}_K{shapes[0][1]}_per_layer") \
            if len(set(shapes)) == 1 else None
        out.append({"workload": name, "mode": mode, "M": 16, "layers": len(shapes), "value": achieved, "unit": "GB/s",
                    "us_per_call": per_call * 1e6, "us_per_layer": per_call * 1e6 / len(shapes),
                    "tflops": flop / per_call / 1e12, "api": "bonsai_lowbit_gemm_batch, one call per step",
                    "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                                 "frac": achieved / peak,
                                 "traffic": per_layer * len(shapes) if per_layer is not None else None,
                                 "algorithmic_bytes_per_call": nbytes, "peak_source": f"{peaks_kind} hbm copy"},
                    "gpu_launches": steps})
        del probs, outs, base
    return out


def time_formats(torch, bw, args, dist, peaks, peaks_kind):
    """The headline and the M=16 workloads with the same ternary codes stored
    in the base-3 format (1.75 bits per weight against INT2's 2): TFLOP/s at
    M=4608 and GB/s of algorithmic bytes (fewer packed bytes) at M=16."""
    out = []
    for base, sets_n, unit in ((WORKLOAD, args.sets, "TFLOP/s"), (SMALL[0], 64, "GB/s")):
        p = workloads.Problem("base-3 " + base.name, "ternary_b3", base.M, base.N, base.K, base.seed)
        sets = make_sets(p, sets_n, torch, bw, distinct_weights=False)
        steps = max(200, min(args.steps, 2000))
        secs = time_launches(torch, bw, p, sets, steps, max(args.warmup, 3), dist)
        t = max_over_ranks(torch, secs, dist) / steps
        del sets
        value = flops(p) / t / 1e12 if unit == "TFLOP/s" else algorithmic_bytes(p) / t / 1e9
        out.append({"workload": p.name, "mode": p.mode, "M": p.M, "N": p.N, "K": p.K, "value": value, "unit": unit,
                    "us_per_launch": t * 1e6, "packed_bytes": packed_weight_bytes(p.mode, p.N, p.K),
                    "int2_packed_bytes": packed_weight_bytes("ternary", p.N, p.K),
                    "plan": bw.gemm_plan(p.M, p.N, p.K, p.mode)})
    # 4-bit group-affine weights (the text encoder's format) on the headline shape and at M=16
    for p, unit in ((WORKLOAD, "TFLOP/s"), (SMALL[0], "GB/s")):
        out.append(time_hqq4(torch, bw, args, p, unit))
    return out


def time_hqq4(torch, bw, args, p, unit):
    """The 4-bit group-affine GEMM on problem p's shape: TFLOP/s, or GB/s of
    its algorithmic bytes (packed 4-bit words, FP16 scales and zeros per 64,
    activations in, output out)."""
    d = workloads.make_hqq4(1, p.N, p.K, seed=p.seed)
    packed = bw.hqq4_pack(torch.from_numpy(d["q"]).cuda())
    s = torch.from_numpy(d["scales"].view(np.int16)).view(torch.float16).cuda()
    z = torch.from_numpy(d["zeros"].view(np.int16)).view(torch.float16).cuda()
    rng = np.random.default_rng(p.seed)
    nsets = args.sets if unit == "TFLOP/s" else 32  # above L2 either way
    sets = [(torch.from_numpy(workloads.activations(rng, p.M, p.K).view(np.int16)).view(torch.float16).cuda(),
             packed.clone(), s.clone(), z.clone(), torch.empty((p.M, p.N), dtype=torch.float16, device="cuda"))
            for _ in range(nsets)]

    def launch(i):
        A, pk, sc, zc, o = sets[i % len(sets)]
        bw.hqq4_gemm(A, pk, sc, zc, out=o)

    for i in range(3):
        launch(i)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for i in range(len(sets)):
            launch(i)
    steps = max(200, min(args.steps, 2000)) // len(sets) * len(sets)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    graph.replay()
    torch.cuda.synchronize()
    e0.record()
    for _ in range(steps // len(sets)):
        graph.replay()
    e1.record()
    torch.cuda.synchronize()
    t = e0.elapsed_time(e1) / 1e3 / steps
    del graph, sets
    nbytes = p.N * p.K // 2 + 4 * p.N * (p.K // 64) + 2 * p.M * p.K + 2 * p.M * p.N
    return {"workload": "4-bit group-affine " + p.name, "mode": "hqq4", "M": p.M, "N": p.N, "K": p.K,
            "value": flops(p) / t / 1e12 if unit == "TFLOP/s" else nbytes / t / 1e9, "unit": unit,
            "us_per_launch": t * 1e6, "packed_bytes": p.N * p.K // 2, "algorithmic_bytes": nbytes,
            "plan": bw.gemm_plan(p.M, p.N, p.K, "hqq4")}


LAYER_SHAPES = ((18432, 3072, "single-stream fused QKV + MLP-up"), (3072, 12288, "single-stream out"))


def time_layers(torch, bw, args, dist):
    """The single-stream layers of the stack on their own, at the token counts
    of a 1024^2 image + text (4608), a 512^2 image + text (1536) and a 512^2
    image (1024): TFLOP/s of single launches (rotating inputs above L2,
    CUDA-graph replay) with the launch the planner chose."""
    out = []
    for n, k, name in LAYER_SHAPES:
        for m in (4608, 1536, 1024):
            p = workloads.Problem(f"{name} M={m}", "ternary", m, n, k, 5000 + m + n)
            count = int(min(16, max(2, -(-4 * 126 * 2 ** 20 // algorithmic_bytes(p)))))
            sets = make_sets(p, count, torch, bw, distinct_weights=False)
            steps = max(count * 8, 200) // count * count
            secs = time_launches(torch, bw, p, sets, steps, 3, dist)
            t = max_over_ranks(torch, secs, dist) / steps
            del sets
            out.append({"layer": name, "M": m, "N": n, "K": k, "us_per_launch": t * 1e6, "tflops": flops(p) / t / 1e12,
                        "plan": bw.gemm_plan(m, n, k, "ternary")})
    return out


def time_pack_dequant(torch, bw, p, peaks, peaks_kind, sets=5, reps=20):
    """The offline pack and the test-facing dequant on the headline weight
    shape, in GB/s of their algorithmic bytes (codes in + packed words out;
    packed words + scales in + FP16 weights out) against the measured HBM
    copy bandwidth.  bonsai_pack synchronises to read its bad-code flag, so
    its figure is per call (CUDA events around the call: flag reset, kernel,
    flag read-back), the median of `reps` calls over `sets` rotating inputs
    (larger than L2); dequant is timed as back-to-back launches replayed from
    a CUDA graph."""
    peak = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    out = []
    def call_time(codes, packed, mode):
        """Median per-call time of bonsai_pack over rotating inputs."""
        times = []
        for i in range(reps + 2):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            bw.pack(codes[i % len(codes)], mode, out=packed[i % len(codes)])
            e1.record()
            torch.cuda.synchronize()
            if i >= 2:
                times.append(e0.elapsed_time(e1) / 1e3)
        return statistics.median(times)

    for mode in ("ternary", "binary", "ternary_b3"):
        d = workloads.make(mode=mode, M=1, N=p.N, K=p.K, seed=p.seed)
        codes = [torch.from_numpy(d["codes"]).cuda() for _ in range(sets)]
        packed = [bw.pack(c, mode) for c in codes]
        t1 = call_time(codes, packed, mode)
        # Kernel time: one call on a weight 16 times as tall (453 MB of codes
        # for the headline shape, so the kernel dominates) minus the fixed
        # cost of a call (flag reset, read-back, synchronisation) measured on
        # a one-group weight, divided by 16.
        tiny = [torch.from_numpy(d["codes"][:8, :128].copy()).cuda() for _ in range(2)]
        t0 = call_time(tiny, [bw.pack(c, mode) for c in tiny], mode)
        big = [c.repeat(16, 1) for c in codes[:2]]
        big_packed = [bw.pack(c, mode) for c in big]
        t16 = call_time(big, big_packed, mode)
        del big, big_packed
        t = (t16 - t0) / 16
        nbytes = p.N * p.K + packed_weight_bytes(mode, p.N, p.K)
        out.append({"op": "pack", "mode": mode, "N": p.N, "K": p.K, "us_kernel": t * 1e6, "us_per_call": t1 * 1e6,
                    "value": nbytes / t / 1e9, "unit": "GB/s", "frac": nbytes / t / 1e9 / peak,
                    "algorithmic_bytes": nbytes,
                    "timing": "kernel time = (call on a 16x taller weight - call on one group) / 16; per call "
                              "incl. flag reset/read-back and synchronisation; CUDA events, medians"})
        if mode == "ternary_b3":
            continue
        scales = torch.from_numpy(d["scales"].view(np.int16)).view(torch.float16).cuda()
        sets_dq = [(packed[j], scales.clone(), torch.empty((p.N, p.K), dtype=torch.float16, device="cuda"))
                   for j in range(3)]
        for pk, sc, w in sets_dq:
            bw.dequant(pk, sc, p.K, mode, out=w)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for pk, sc, w in sets_dq:
                bw.dequant(pk, sc, p.K, mode, out=w)
        graph.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            graph.replay()
        e1.record()
        torch.cuda.synchronize()
        t = e0.elapsed_time(e1) / 1e3 / (reps * len(sets_dq))
        del graph, sets_dq
        nbytes = packed_weight_bytes(mode, p.N, p.K) + 2 * p.N * (p.K // 128) + 2 * p.N * p.K
        out.append({"op": "dequant", "mode": mode, "N": p.N, "K": p.K, "us_per_launch": t * 1e6,
                    "value": nbytes / t / 1e9, "unit": "GB/s", "frac": nbytes / t / 1e9 / peak,
                    "algorithmic_bytes": nbytes, "timing": "CUDA graph replay, CUDA events"})
        del codes, packed
    return out


def cublas_fp16_same_run(torch, n=8192, seconds=0.4):
    """Dense FP16 torch.matmul (cuBLAS) n^3 on this GPU in this run, for
    context beside the measured peaks: best of 10 single launches, and the
    mean over about `seconds` of back-to-back launches (the length of the
    headline's timed region, so under the same power cap)."""
    a = torch.randn((n, n), device="cuda", dtype=torch.float16)
    b = torch.randn((n, n), device="cuda", dtype=torch.float16)
    c = torch.empty((n, n), device="cuda", dtype=torch.float16)
    flop = 2.0 * n ** 3
    for _ in range(3):
        torch.matmul(a, b, out=c)
    torch.cuda.synchronize()
    best = float("inf")
    for _ in range(10):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        torch.matmul(a, b, out=c)
        e1.record()
        torch.cuda.synchronize()
        best = min(best, e0.elapsed_time(e1) / 1e3)
    reps = max(10, int(seconds / best))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        torch.matmul(a, b, out=c)
    e1.record()
    torch.cuda.synchronize()
    loop = e0.elapsed_time(e1) / 1e3 / reps
    del a, b, c
    return {"burst_tflops": flop / best / 1e12, "loop_tflops": flop / loop / 1e12, "loop_launches": reps,
            "shape": f"{n}^3 fp16"}


def time_stack(torch, bw, M, mode, steps, warmup, seed=2000, split_qkv=False, streams=None):
    """One denoise step of the 25-block MMDiT stack (80 launches = 100 linears
    with Q|K|V stacked, or 100 launches with split_qkv): every layer has its
    own weight buffers (cloned from one seeded set per distinct shape), the
    step is captured as one CUDA graph.  With streams = (image tokens, text
    tokens) the double-stream linears run on their own stream's rows and the
    single-stream ones on the joint sequence; otherwise every layer has M rows."""
    if streams is not None:
        layers = workloads.mmdit_stream_layers(*streams)
    else:
        layers = [(name, M, n, k) for name, n, k in workloads.mmdit_stack_layers(split_qkv=split_qkv)]
    shapes = sorted({(n, k) for _, _, n, k in layers})
    base = {}
    for j, (n, k) in enumerate(shapes):
        d = workloads.make(mode=mode, M=1, N=n, K=k, seed=seed + j)
        packed = bw.pack(torch.from_numpy(d["codes"]).cuda(), mode)
        scales = torch.from_numpy(d["scales"].view(np.int16)).view(torch.float16).cuda()
        base[(n, k)] = (packed, scales)
    weights = [tuple(t.clone() for t in base[(n, k)]) for _, _, n, k in layers]
    rng = np.random.default_rng(seed)
    acts = {(m, k): torch.from_numpy(workloads.activations(rng, m, k).view(np.int16)).view(torch.float16).cuda()
            for m, k in sorted({(m, k) for _, m, _, k in layers})}
    outs = {(m, n): torch.empty((m, n), dtype=torch.float16, device="cuda")
            for m, n in sorted({(m, n) for _, m, n, _ in layers})}

    def step():
        for (name, m, n, k), (packed, scales) in zip(layers, weights):
            bw.lowbit_gemm(acts[(m, k)], packed, scales, mode, out=outs[(m, n)])

    step()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    for _ in range(warmup):
        graph.replay()
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record()
    for _ in range(steps):
        graph.replay()
    end.record()
    torch.cuda.synchronize()
    ms = start.elapsed_time(end) / steps
    total_flops = sum(2 * m * n * k for _, m, n, k in layers)
    wbytes = sum(n * k // (8 if mode == "binary" else 4) + 2 * n * (k // 128) for _, _, n, k in layers)
    del graph
    rows = {"M": M} if streams is None else {"image_tokens": streams[0], "text_tokens": streams[1]}
    return {**rows, "mode": mode, "launches": len(layers), "ms_per_denoise_step": ms,
            "tflops": total_flops / (ms * 1e-3) / 1e12, "weight_bytes": wbytes,
            "weight_gbs": wbytes / (ms * 1e-3) / 1e9}


SWEEP_M = (16, 32, 64, 128, 192, 256, 384, 512, 768, 1024, 1536, 2048, 3072, 4096, 4608)
SWEEP_SHAPES = ((3072, 3072), (9216, 3072), (3072, 9216), (18432, 3072), (3072, 12288))


def run_m_sweep(args):
    """TFLOP/s and weight-stream GB/s of single launches over the token
    counts an MMDiT step meets (text stream 512, image 1024 / 4096, joint
    1536 / 4608) and the small-batch end, on the stack's layer shapes.
    Each point rotates over enough input sets to exceed L2 four times."""
    import torch

    torch.cuda.set_device(0)
    import bit_weight_gemm_b200 as bw

    mode = "ternary"
    points = []
    for j, (n, k) in enumerate(SWEEP_SHAPES):
        d = workloads.make(mode=mode, M=1, N=n, K=k, seed=3000 + j)
        packed = bw.pack(torch.from_numpy(d["codes"]).cuda(), mode)
        scales = torch.from_numpy(d["scales"].view(np.int16)).view(torch.float16).cuda()
        rng = np.random.default_rng(3100 + j)
        a_all = torch.from_numpy(workloads.activations(rng, max(SWEEP_M), k).view(np.int16)).view(torch.float16).cuda()
        for m in SWEEP_M:
            p = workloads.Problem(f"sweep M={m} N={n} K={k}", mode, m, n, k, 0)
            per_set = algorithmic_bytes(p)
            count = int(min(64, max(2, -(-4 * 126 * 2 ** 20 // per_set))))
            sets = [(a_all[:m].clone(), packed.clone(), scales.clone(),
                     torch.empty((m, n), dtype=torch.float16, device="cuda")) for _ in range(count)]
            est = max(flops(p) / 1.4e15, per_set / 6.0e12) + 3e-6
            steps = int(min(2000, max(4 * count, 0.03 / est)))
            steps -= steps % count
            secs = time_launches(torch, bw, p, sets, steps, 3)
            t = secs / steps
            wbytes = n * k // 4 + 2 * n * (k // 128)
            points.append({"M": m, "N": n, "K": k, "us": t * 1e6, "tflops": flops(p) / t / 1e12,
                           "gbs": per_set / t / 1e9, "weight_gbs": wbytes / t / 1e9,
                           "plan": bw.gemm_plan(m, n, k, mode)})
            del sets
        del packed, scales, a_all
    assert bw.get_device_error() == 0
    print(json.dumps({"m_sweep": points, "mode": mode, "timing": "CUDA graph replay, CUDA events"}), flush=True)
    return 0


def run_offline(args):
    """Pack and dequant alone (for profiling): one JSON line."""
    import torch

    torch.cuda.set_device(0)
    import bit_weight_gemm_b200 as bw

    peaks, peaks_kind = load_peaks()
    res = time_pack_dequant(torch, bw, WORKLOAD, peaks, peaks_kind)
    assert bw.get_device_error() == 0
    print(json.dumps({"pack_dequant": res, "peak_source": f"{peaks_kind} hbm copy"}), flush=True)
    return 0


def run_case(args):
    """One configuration of one kernel, launched --launches times on the
    seeded workload inputs: the command line the ncu summaries under
    profiles/ profile."""
    import torch

    torch.cuda.set_device(0)
    import bit_weight_gemm_b200 as bw

    op, _, rest = args.case.rpartition("-") if args.case.split(":")[0].startswith(("pack-", "dequant-", "batch-")) \
        else ("gemm", "", args.case)
    fields = rest.split(":")
    mode = fields[0]
    if op == "batch":
        # batch-MODE:M:N:K:L - L layers of one shape (own buffers each) in one bonsai_lowbit_gemm_batch call
        M, N, K, L = (int(x) for x in fields[1:5])
        d = workloads.make(mode=mode, M=M, N=N, K=K, seed=7)
        base = (torch.from_numpy(d["A"].view(np.int16)).view(torch.float16).cuda(),
                bw.pack(torch.from_numpy(d["codes"]).cuda(), mode),
                torch.from_numpy(d["scales"].view(np.int16)).view(torch.float16).cuda())
        probs = [tuple(t.clone() for t in base) for _ in range(L)]
        outs = [torch.empty((M, N), dtype=torch.float16, device="cuda") for _ in range(L)]
        torch.cuda.synchronize()
        for _ in range(args.launches):
            bw.lowbit_gemm_batch(probs, mode, outs=outs)
        torch.cuda.synchronize()
        assert bw.get_device_error() == 0
        print(json.dumps({"case": args.case, "launches": args.launches}), flush=True)
        return 0
    if op == "gemm":
        M, N, K = (int(x) for x in fields[1:4])
    else:
        M, (N, K) = 1, (int(x) for x in fields[1:3])
    if mode == "hqq4":
        d = workloads.make_hqq4(M, N, K, seed=7)
        packed = bw.hqq4_pack(torch.from_numpy(d["q"]).cuda())
        s = torch.from_numpy(d["scales"].view(np.int16)).view(torch.float16).cuda()
        z = torch.from_numpy(d["zeros"].view(np.int16)).view(torch.float16).cuda()
        A = torch.from_numpy(d["A"].view(np.int16)).view(torch.float16).cuda()
        run = {"gemm": lambda: bw.hqq4_gemm(A, packed, s, z),
               "dequant": lambda: bw.hqq4_dequant(packed, s, z, K),
               "pack": lambda: bw.hqq4_pack(torch.from_numpy(d["q"]).cuda())}[op]
    else:
        d = workloads.make(mode=mode, M=M, N=N, K=K, seed=7)
        codes = torch.from_numpy(d["codes"]).cuda()
        packed = bw.pack(codes, mode)
        s = torch.from_numpy(d["scales"].view(np.int16)).view(torch.float16).cuda()
        A = torch.from_numpy(d["A"].view(np.int16)).view(torch.float16).cuda()
        run = {"gemm": lambda: bw.lowbit_gemm(A, packed, s, mode),
               "dequant": lambda: bw.dequant(packed, s, K, mode),
               "pack": lambda: bw.pack(codes, mode, out=packed)}[op]
    torch.cuda.synchronize()
    for _ in range(args.launches):
        run()
    torch.cuda.synchronize()
    assert bw.get_device_error() == 0
    plan = bw.gemm_plan(M, N, K, mode) if op == "gemm" else None
    print(json.dumps({"case": args.case, "launches": args.launches, "plan": plan}), flush=True)
    return 0


def main():
    args = parse_args()
    if args.case:
        return run_case(args)
    if args.m_sweep:
        return run_m_sweep(args)
    if args.offline_only:
        return run_offline(args)
    if args.layers_only:
        import torch

        torch.cuda.set_device(0)
        import bit_weight_gemm_b200 as bw

        print(json.dumps({"layers": time_layers(torch, bw, args, None)}), flush=True)
        return 0
    if args.impl == "reference":
        return run_reference(args)
    return run_bonsai(args)


if __name__ == "__main__":
    sys.exit(main())
