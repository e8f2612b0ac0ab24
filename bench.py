#!/usr/bin/env python
"""Benchmark of the intra-expert sparse MoE layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload mixtral_decode] [--sparsity 0.7]

A step is one pass of the whole layer (router, permute, fused gate+up with
SwiGLU/threshold/compaction, union scan, sparse down projection, combine)
over each decode batch of the workload; for the Mixtral-8x7B-shaped layer
(bf16, d_model 4096, 8 experts top-2, d_ff 14336) that is the batches
T = 1, 8, 32, 64 (105 tokens per step). The metric is MoE-layer tokens/s,
measured on the device with CUDA events between a barrier and a
synchronize on both sides, max over ranks. The touched experts' weights
(>= 470 MB per forward) are larger than L2, so no flush is needed.

The same steps are run on the library's own dense path (no threshold, every
W_down row read) for the speedup, end to end through the Python API with
host buffers (e2e), and, on rank 0 at N=1, through the CPU oracle on the
host cores (cpu_baseline). ``--impl reference`` times only the oracle.
Multi-GPU runs are weak-scaling replicas: every rank runs the full workload
on its own GPU and copy of the weights; the path has no exchange step.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import threading
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from moe_inputs import WORKLOADS, make_tokens, make_weights  # noqa: E402

METRIC = "MoE-layer tokens/s and effective HBM GB/s vs own dense path, 0-90% sparsity"
FALLBACK_HBM_GBS = 6650.0
# DRAM traffic / algorithmic bytes of gate_up_tc_kernel from one ncu capture of a smaller
# launch of the same kernel (decode batch T=8, 7 experts touched): traffic grows with the
# touched experts, so a launch's traffic is this ratio times its algorithmic bytes. The
# ratio holds only for the kernel source it was captured on: SOURCE_SHA16 is the hash of
# those files (kernel_source_hash); when the sources differ the line reports traffic null.
GATE_UP_TRAFFIC = {"ratio": 1.0043, "source_sha16": "fa22b7db1f9b7c2e",
                   "files": ("gate_up_tc.cu", "common.cuh")}


def kernel_source_hash(files) -> str:
    """First 16 hex digits of the sha256 over the named kernel sources, in order."""
    import hashlib
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "intra_expert_activation_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def parse():
    ap = argparse.ArgumentParser(description="MoE-layer tokens/s of the sparse layer on B200")
    ap.add_argument("--gpus", type=int, default=1,
                    help="ranks (one per GPU, launched by torchrun for N > 1): replicas")
    ap.add_argument("--steps", type=int, default=20, help="timed steps")
    ap.add_argument("--warmup", type=int, default=5, help="untimed warm-up steps")
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours",
                    help="reference: time the CPU oracle on the host cores instead")
    ap.add_argument("--workload", default="mixtral_decode", choices=sorted(WORKLOADS),
                    help="synthetic workload (moe_inputs/workloads.py)")
    ap.add_argument("--sparsity", type=float, default=0.7,
                    help="target sparsity; tau comes from tests/golden/tau_calibration.json")
    ap.add_argument("--score", choices=("h", "gate"), default="h",
                    help="h: active iff |SiLU(g) u| > tau; gate: active iff |SiLU(g)| > tau with "
                         "the sparse up projection (the pages' own system)")
    ap.add_argument("--tokens", type=str, default="", help="comma list overriding the batches")
    ap.add_argument("--path", default="auto",
                    choices=("auto", "sparse_gemv", "sparse_tc", "sparse_tc_allrows"),
                    help="down-projection path of the sparse arm (default: the automatic "
                         "per-group choice; the others force one path, e.g. to profile it)")
    ap.add_argument("--no-dense", action="store_true", help="skip the dense-path comparison")
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the oracle timing")
    ap.add_argument("--no-e2e", action="store_true",
                    help="skip the end-to-end run with host buffers")
    ap.add_argument("--eager", action="store_true",
                    help="time eager API calls instead of replaying a captured CUDA graph")
    ap.add_argument("--reps", type=int, default=50,
                    help="graph replays timed one by one per latency point (median, p10, p90)")
    ap.add_argument("--no-sweep", action="store_true",
                    help="skip the sparsity sweep (Mixtral shape, sparse vs own dense path)")
    return ap.parse_args()


def load_tau(workload: str, q: float, score: str = "h"):
    with open(os.path.join(ROOT, "tests", "golden", "tau_calibration.json")) as f:
        e = json.load(f)[workload]["taus_gate" if score == "gate" else "taus"][f"{q:.2f}"]
    return e["tau"], e.get("tau_shared", 0.0), e["measured_sparsity"]


FALLBACK_BF16_TFLOPS = 1590.0


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def tensor_peak():
    """Dense bf16 TFLOP/s: the burst figure (the kernel is timed on its own)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    return FALLBACK_BF16_TFLOPS, "fallback"


class Clocks:
    """SM clock and clock-event reasons of this process's GPU, read through
    NVML every 5 ms by a background thread while the timed region runs
    (read-only queries; nothing is set)."""

    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4}

    def __init__(self, device: int):
        self.samples = []
        self.error = None
        self.max_mhz = None
        self._stop = threading.Event()
        self.thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(device).uuid)
            h = pynvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else f"GPU-{uuid}")
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
        except Exception as exc:  # no NVML on this machine
            self.error = f"NVML: {exc}"[:200]
            return

        def run():
            while not self._stop.is_set():
                try:
                    sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                    rs = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                except Exception as exc:
                    self.error = f"NVML: {exc}"[:200]
                    return
                self.samples.append((sm, rs))
                self._stop.wait(0.005)

        self.thread = threading.Thread(target=run, daemon=True)
        self.thread.start()

    def stop(self):
        if self.thread is not None:
            self._stop.set()
            self.thread.join(timeout=5)
        if not self.samples:
            return {"error": self.error or "no clock samples"}
        reasons = sorted(n for n, bit in self.REASONS.items()
                         if any(rs & bit for _, rs in self.samples))
        return {"sm_mhz": statistics.median(sm for sm, _ in self.samples),
                "sm_max_mhz": self.max_mhz, "reasons": reasons, "samples": len(self.samples),
                "source": "NVML, 5 ms"}


def dist_init(args=None, backend=None):
    """One process per GPU (torchrun env); NCCL on GPUs, gloo without."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    cuda = torch.cuda.is_available()
    if cuda:
        torch.cuda.set_device(local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = backend or ("nccl" if cuda else "gloo")
        kw = {"device_id": torch.device("cuda", local)} if backend == "nccl" else {}
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(world, v: float, local: int) -> float:
    """The slowest rank's time: every rank's number is all-reduced with MAX."""
    if world == 1:
        return v
    import torch.distributed as dist
    dev = "cpu" if dist.get_backend() == "gloo" else f"cuda:{local}"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_value(tokens_per_step: int, steps: int, world: int, ms: float) -> float:
    """Whole-job tokens/s of weak-scaling replicas: every rank runs the same
    steps on its own batch, the job takes the slowest rank's time."""
    return tokens_per_step * steps * world / (ms / 1e3)


def workload_config(args, wl, tokens, tau, calib_sparsity, world) -> dict:
    """The config block both arms print for a workload."""
    sh = wl.shape
    cfg = {"workload": args.workload, "score": args.score, "batches": tokens,
           "tokens_per_step": sum(tokens),
           "d_model": sh.d_model, "n_experts": sh.n_experts, "top_k": sh.top_k,
           "d_ff": sh.d_ff, "target_sparsity": args.sparsity, "tau": tau,
           "calibrated_sparsity": round(calib_sparsity, 4),
           "l2": "no flush: touched expert weights (>= 470 MB per forward) exceed L2",
           "parallelism": f"replicas x{world}"}
    if getattr(args, "path", "auto") != "auto":
        cfg["path"] = args.path
    return cfg


# ------------------------------------------------------------------ oracle arm

def oracle_step_time(wl, tokens, tau, tau_s, w_host, score="h"):
    from oracle import moe_oracle as om
    sh = wl.shape
    t0 = time.perf_counter()
    for T in tokens:
        x = make_tokens(sh.d_model, T, wl.token_seed, sh.dtype)
        om.layer_forward(x, w_host.W_router, w_host.W_gate, w_host.W_up, w_host.W_down, tau,
                         sh.top_k, sh.renormalize, router_bias=w_host.router_bias,
                         Ws_gate=w_host.Ws_gate, Ws_up=w_host.Ws_up, Ws_down=w_host.Ws_down,
                         tau_shared=tau_s, score=score)
    return time.perf_counter() - t0


def run_reference(args, world, rank):
    """The oracle arm: the fp64 CPU oracle timed on the host cores, on rank 0
    only; each step is the same step the GPU arm times (every batch of the
    workload), the same sample as the GPU arm's cpu_baseline."""
    if rank != 0:
        return 0
    wl = WORKLOADS[args.workload]
    tokens = [int(t) for t in args.tokens.split(",")] if args.tokens else list(wl.tokens)
    tau, tau_s, calib_sparsity = load_tau(args.workload, args.sparsity, args.score)
    w = make_weights(wl.shape, wl.weight_seed)
    sample = list(tokens)
    for _ in range(args.warmup):
        oracle_step_time(wl, sample, tau, tau_s, w, args.score)
    t = sum(oracle_step_time(wl, sample, tau, tau_s, w, args.score) for _ in range(args.steps))
    toks = sum(sample) * args.steps
    cores = len(os.sched_getaffinity(0))
    value = toks / t
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * t / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(args, wl, tokens, tau, calib_sparsity, world),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": f"each step: the decode batches T={sample} of "
                                   f"{args.workload}, as in the GPU arm's step (fp64 numpy "
                                   f"oracle on {cores} host threads)"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ latency points

def replay_stats(fwd, dev, warmup: int, reps: int) -> dict:
    """Layer latency of one forward: a CUDA graph of `fwd` replayed `reps`
    times, each replay between its own pair of CUDA events on the replaying
    stream; median, p10 and p90 in microseconds."""
    fwd()
    torch.cuda.synchronize(dev)
    stream = torch.cuda.current_stream(dev)
    side = torch.cuda.Stream(dev)
    side.wait_stream(stream)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        fwd()
    torch.cuda.synchronize(dev)
    for _ in range(warmup):
        g.replay()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(reps)]
    torch.cuda.synchronize(dev)
    for a, b in ev:
        a.record(stream)
        g.replay()
        b.record(stream)
    torch.cuda.synchronize(dev)
    us = np.array([1e3 * a.elapsed_time(b) for a, b in ev])
    del g
    return {"median": round(float(np.median(us)), 2), "p10": round(float(np.percentile(us, 10)), 2),
            "p90": round(float(np.percentile(us, 90)), 2), "reps": reps}


SWEEP_POINTS = {  # (T, target sparsity) per score
    "h": [(1, 0.0), (1, 0.5), (1, 0.7), (1, 0.9), (16, 0.0), (16, 0.5), (16, 0.7), (16, 0.9),
          (128, 0.0), (128, 0.9), (512, 0.0), (512, 0.9)],
    "gate": [(1, 0.0), (1, 0.5), (1, 0.7), (1, 0.9), (16, 0.0), (16, 0.5), (16, 0.7), (16, 0.9)],
}


def run_sweep(dev, local, warmup: int, reps: int, w_host=None) -> dict:
    """Sparsity sweep on the Mixtral-shaped layer (d_model 4096, 8 experts
    top-2, d_ff 14336, bf16, weights seed 4): tau calibrated on the 512-token
    batch at each target sparsity, the smaller batches its prefixes. Every
    point is the graph-replayed layer latency of the sparse path against the
    library's own dense path (same kernels, no threshold, every row) at the
    same T, for the |h| score and for the gate score."""
    from intra_expert_activation_b200 import MoESparseLayer
    wl = WORKLOADS["mixtral_sweep"]
    sh = wl.shape
    w_host = w_host or make_weights(sh, wl.weight_seed)
    W = {k: getattr(w_host, k).to(dev).contiguous() for k in ("W_router", "W_gate", "W_up",
                                                              "W_down")}
    xs = {T: make_tokens(sh.d_model, T, wl.token_seed, sh.dtype).to(dev)
          for T in sorted({T for pts in SWEEP_POINTS.values() for T, _ in pts})}

    def point(T, path, score, tau):
        L = MoESparseLayer(sh.d_model, sh.d_ff, sh.n_experts, sh.top_k, T,
                           renormalize=sh.renormalize, dtype=sh.dtype, path=path, device=local,
                           score=score)
        out = torch.empty((T, sh.d_model), dtype=torch.bfloat16, device=dev)

        def fwd():
            L.forward(xs[T], W["W_router"], W["W_gate"], W["W_up"], W["W_down"], tau,
                      sh.top_k, out=out)
        clk = Clocks(local)
        lat = replay_stats(fwd, dev, warmup, reps)
        c = clk.stop()
        lat["sm_mhz"] = c.get("sm_mhz")
        lat["clock_reasons"] = c.get("reasons")
        fwd()
        st = L.stats()
        assert L.status() == 0, "device status word set"
        L.close()
        return lat, st

    # batch by batch, smallest first (the large batches run the tensor cores
    # hardest and are measured last), each batch's dense point measured just
    # before and again just after its sparse points (the reference is the
    # mean of the two medians, so that a drift of the clock over the batch's
    # points shows in both); every point records the SM clock it ran at
    dense = {}
    points = []
    for T in sorted(xs):
        lat, st = point(T, "dense", "h", 0.0)
        dense[T] = {"us": lat, "rows": st["down_rows_read"]}
        first = len(points)
        for score, pts in SWEEP_POINTS.items():
            for T2, q in pts:
                if T2 != T:
                    continue
                tau, _, calib = load_tau("mixtral_sweep", q, score)
                lat, st = point(T, "auto", score, tau)
                meas = 1.0 - st["n_routed_active"] / max(st["n_routed_h"], 1)
                points.append({
                    "score": score, "T": T, "target_sparsity": q, "sparsity": round(meas, 4),
                    "tau": tau, "us": lat, "dense_us": dense[T]["us"],
                    "speedup": round(dense[T]["us"]["median"] / lat["median"], 3),
                    "down_rows_read": st["down_rows_read"], "up_rows_read": st["up_rows_read"],
                    "gate_up_rows_read": st["gate_up_rows_read"],
                    "down_rows_dense": dense[T]["rows"],
                    "groups": {"gemv": st["n_groups_gemv"], "tc_allrows": st["n_groups_tc_allrows"],
                               "tc_gather": st["n_groups_tc_gather"]},
                })
        lat2, _ = point(T, "dense", "h", 0.0)
        ref = 0.5 * (dense[T]["us"]["median"] + lat2["median"])
        dense[T]["us"] = dict(dense[T]["us"], median=round(ref, 2), before=dense[T]["us"]["median"],
                              after=lat2["median"])
        for pnt in points[first:]:
            pnt["dense_us"] = dense[T]["us"]
            pnt["speedup"] = round(ref / pnt["us"]["median"], 3)
    summary = {}
    for score in SWEEP_POINTS:
        for T in (1, 16):
            row = [p for p in points if p["score"] == score and p["T"] == T]
            summary[f"{score}_T{T}"] = {f"{p['target_sparsity']:.1f}": p["speedup"] for p in row}
    return {"workload": "mixtral_sweep", "reps": reps, "speedup_vs_dense": summary, "points": points,
            "timing": "graph replays, each between its own CUDA events; median/p10/p90 us; "
                      "touched expert weights exceed L2 (no flush)"}


# ------------------------------------------------------------------ GPU arm

def run_ours(args, world, rank, local):
    from intra_expert_activation_b200 import MoESparseLayer

    dev = torch.device("cuda", local)
    wl = WORKLOADS[args.workload]
    sh = wl.shape
    tokens = [int(t) for t in args.tokens.split(",")] if args.tokens else list(wl.tokens)
    tau, tau_s, calib_sparsity = load_tau(args.workload, args.sparsity, args.score)
    w_host = make_weights(sh, wl.weight_seed)
    mv = lambda t: None if t is None else t.to(dev).contiguous()
    W = {k: mv(getattr(w_host, k)) for k in ("W_router", "W_gate", "W_up", "W_down",
                                             "router_bias", "Ws_gate", "Ws_up", "Ws_down")}
    xs_host = [make_tokens(sh.d_model, T, wl.token_seed, sh.dtype) for T in tokens]
    xs = [x.to(dev) for x in xs_host]
    outs = [torch.empty((T, sh.d_model), dtype=x.dtype, device=dev) for T, x in zip(tokens, xs)]
    tmax = max(tokens)
    esize = 2 if sh.dtype == "bf16" else 4

    def make(path):
        L = MoESparseLayer(sh.d_model, sh.d_ff, sh.n_experts, sh.top_k, tmax,
                           renormalize=sh.renormalize, n_shared=sh.n_shared,
                           d_ff_shared=sh.d_ff_shared, dtype=sh.dtype, path=path, device=local,
                           score=args.score if path != "dense" else "h")
        if sh.n_shared:
            L.set_shared(W["Ws_gate"], W["Ws_up"], W["Ws_down"], tau_s)
        return L

    def step(L, out_list=outs, x_list=xs):
        for x, o in zip(x_list, out_list):
            L.forward(x, W["W_router"], W["W_gate"], W["W_up"], W["W_down"], tau, sh.top_k,
                      router_bias=W["router_bias"], out=o)

    stream = torch.cuda.current_stream(dev)

    def capture(L):
        """One step of forwards captured into a CUDA graph (the library's
        forward allocates nothing and never synchronises, so it captures)."""
        side = torch.cuda.Stream(dev)
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            step(L)
        stream.wait_stream(side)
        torch.cuda.synchronize(dev)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=side):
            step(L)
        torch.cuda.synchronize(dev)
        return g

    def timed(L, graph=None):
        """Pass A: K steps with nothing between the kernels (no events)."""
        for _ in range(args.warmup):
            graph.replay() if graph is not None else step(L)
        torch.cuda.synchronize(dev)
        barrier(world)
        torch.cuda.synchronize(dev)
        n0 = L.launch_count()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            graph.replay() if graph is not None else step(L)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        barrier(world)
        per_step = (L.launch_count() - n0) // args.steps if graph is None else None
        return e0.elapsed_time(e1), per_step

    def kernel_times(L):
        """Pass B: the same K steps, eager, with per-stage CUDA events recorded
        by the library on the forward's stream around every kernel."""
        L.set_timing(args.steps * len(tokens))
        torch.cuda.synchronize(dev)
        for _ in range(args.steps):
            step(L)
        torch.cuda.synchronize(dev)
        per = L.timing_all(args.steps * len(tokens))
        L.set_timing(0)
        return per

    def per_batch_us(L):
        """Layer latency per decode batch: --reps replays of a graph of one
        forward, each timed between its own events (median, p10, p90)."""
        res = []
        for x, o in zip(xs, outs):
            def one(x=x, o=o):
                L.forward(x, W["W_router"], W["W_gate"], W["W_up"], W["W_down"], tau,
                          sh.top_k, router_bias=W["router_bias"], out=o)
            res.append(replay_stats(one, dev, args.warmup, args.reps))
        return res

    sweep_on = (not args.no_sweep and world == 1 and args.workload == "mixtral_decode"
                and args.score == "h" and not args.tokens)

    sparse = make(args.path)
    for _ in range(args.warmup):
        step(sparse)
    torch.cuda.synchronize(dev)
    # launches per step, counted on an eager step
    n0 = sparse.launch_count()
    step(sparse)
    launches_per_step = sparse.launch_count() - n0
    g_sparse = None if args.eager else capture(sparse)
    clocks = Clocks(local)
    ms_sparse, _ = timed(sparse, g_sparse)
    clk = clocks.stop()
    ms_sparse = max_over_ranks(world, ms_sparse, local)
    launches = launches_per_step * args.steps
    per_fwd = kernel_times(sparse)
    lat_sparse = per_batch_us(sparse)
    tok_step = sum(tokens)
    value = replica_value(tok_step, args.steps, world, ms_sparse)

    # per-batch statistics of the sparse path (one extra forward each, untimed)
    stats = []
    for x, o in zip(xs, outs):
        sparse.forward(x, W["W_router"], W["W_gate"], W["W_up"], W["W_down"], tau, sh.top_k,
                       router_bias=W["router_bias"], out=o)
        stats.append(sparse.stats())
    assert sparse.status() == 0, "device status word set"

    dense_line = None
    per_dense = []
    lat_dense = [None] * len(tokens)
    if not args.no_dense:
        dense = make("dense")
        for _ in range(args.warmup):
            step(dense)
        g_dense = None if args.eager else capture(dense)
        ms_dense, _ = timed(dense, g_dense)
        ms_dense = max_over_ranks(world, ms_dense, local)
        per_dense = kernel_times(dense)
        lat_dense = per_batch_us(dense)
        dense_line = {"value": replica_value(tok_step, args.steps, world, ms_dense),
                      "ms_per_step": ms_dense / args.steps}
        del g_dense
        dense.close()

    # per-kernel times, grouped by batch (forwards cycle through `tokens`)
    nb = len(tokens)
    def avg_stage(per, i, stage):
        v = [f[stage] for j, f in enumerate(per) if j % nb == i]
        return sum(v) / len(v) if v else 0.0

    per_T = []
    gate_bytes_tot = gate_ms_tot = down_bytes_tot = down_ms_tot = 0.0
    up_bytes_tot = up_ms_tot = gate_flops_tot = gemv_bytes_tot = gemv_ms_tot = 0.0
    for i, T in enumerate(tokens):
        st = stats[i]
        P = T * sh.top_k
        touched = st["n_experts_touched"]
        if args.score == "gate":  # W_gate of every unit, W_up only where it ran densely
            g_bytes = st["gate_up_rows_read"] * sh.d_model * esize + P * sh.d_model * esize \
                + P * sh.d_ff * esize
        else:
            g_bytes = touched * 2 * sh.d_ff * sh.d_model * esize + P * sh.d_model * esize \
                + P * sh.d_ff * esize
            if sh.n_shared:
                g_bytes += sh.n_shared * 2 * sh.d_ff_shared * sh.d_model * esize
        rb = sh.d_model * esize
        # W_down rows the gate/up kernel read itself (fused down projection of
        # the groups of <= 4 tokens; with the gate score also the W_up rows of
        # its fused up + down) belong to that kernel's bytes
        fused_rows = st["down_rows_fused"]
        fused_up = st["up_rows_fused"]
        g_bytes += (fused_rows + fused_up) * rb
        u_bytes = (st["up_rows_read"] - fused_up) * rb
        u_ms = avg_stage(per_fwd, i, "updown_gemv")  # gate score: fused sparse up + down
        up_bytes_tot += u_bytes * args.steps
        up_ms_tot += u_ms * args.steps
        g_ms = avg_stage(per_fwd, i, "gate_up")
        # the down kernels, each counted only when it had rows to stream (a launch
        # that finds no group of its kind is not down-projection work): the row
        # stream (GEMV; with the gate score the fused kernel, which reads each
        # union row of W_up and of W_down) and the tensor-core path
        gemv_rows = st["down_rows_gemv"]
        tc_rows = st["down_rows_read"] - gemv_rows - fused_rows
        gemv_ms = avg_stage(per_fwd, i, "updown_gemv" if args.score == "gate" else "down_gemv")
        gemv_bytes = gemv_rows * rb * (2 if args.score == "gate" else 1)
        tc_ms = avg_stage(per_fwd, i, "down_tc")
        tc_bytes = tc_rows * rb
        d_ms = (gemv_ms if gemv_rows else 0.0) + (tc_ms if tc_rows else 0.0)
        d_bytes = (gemv_bytes if gemv_rows else 0) + (tc_bytes if tc_rows else 0)
        if gemv_rows:
            gemv_bytes_tot += gemv_bytes * args.steps
            gemv_ms_tot += gemv_ms * args.steps
        fwd_ms = sum(avg_stage(per_fwd, i, s) for s in per_fwd[0]) if per_fwd else 0.0
        fwd_dense = sum(avg_stage(per_dense, i, s) for s in per_dense[0]) if per_dense else None
        d_dense = (avg_stage(per_dense, i, "down_gemv") + avg_stage(per_dense, i, "down_tc")) \
            if per_dense else None
        # gate/up flops: 2 matrices (1 for gate-only rows) x 2 x tokens x d per loaded row
        g_flops = 2.0 * sh.d_model * (P * sh.d_ff * (1 if args.score == "gate" and
                                                      st["n_groups_tc_allrows"] == 0 else 2)
                                      + (sh.n_shared * T * sh.d_ff_shared * 2
                                         if sh.n_shared else 0))
        gate_flops_tot += g_flops * args.steps
        gate_bytes_tot += g_bytes * args.steps
        gate_ms_tot += g_ms * args.steps
        down_bytes_tot += d_bytes * args.steps
        down_ms_tot += d_ms * args.steps
        sp = 1.0 - st["n_routed_active"] / max(st["n_routed_h"], 1)
        per_T.append({
            "T": T, "sparsity": round(sp, 4), "experts_touched": touched,
            "layer_us_graph": lat_sparse[i]["median"],
            "layer_us_graph_p10_p90": [lat_sparse[i]["p10"], lat_sparse[i]["p90"]],
            "dense_layer_us_graph": None if lat_dense[i] is None else lat_dense[i]["median"],
            "dense_layer_us_graph_p10_p90": None if lat_dense[i] is None else
            [lat_dense[i]["p10"], lat_dense[i]["p90"]],
            "speedup_vs_dense_graph": None if lat_dense[i] is None else
            round(lat_dense[i]["median"] / lat_sparse[i]["median"], 3),
            "down_rows_gemv": gemv_rows,
            "down_rows_fused": fused_rows,
            "up_rows_fused": fused_up,
            "down_rows_read": st["down_rows_read"],
            "down_rows_dense": touched * sh.d_ff,
            "up_rows_read": st["up_rows_read"],
            "gate_up_rows_read": st["gate_up_rows_read"],
            "groups": {"gemv": st["n_groups_gemv"], "tc_gather": st["n_groups_tc_gather"],
                       "tc_allrows": st["n_groups_tc_allrows"]},
            "stage_us": {k: round(1e3 * avg_stage(per_fwd, i, k), 2) for k in
                         (per_fwd[0] if per_fwd else {})},
            "layer_us": round(1e3 * fwd_ms, 2),
            "dense_layer_us": None if fwd_dense is None else round(1e3 * fwd_dense, 2),
            "speedup_vs_dense": None if not fwd_dense else round(fwd_dense / fwd_ms, 3),
            "gate_up_GBps": round(g_bytes / (g_ms * 1e-3) / 1e9, 1) if g_ms else None,
            "down_GBps": round(d_bytes / (d_ms * 1e-3) / 1e9, 1) if d_ms else None,
            "down_gemv_GBps": round(gemv_bytes / (gemv_ms * 1e-3) / 1e9, 1)
            if gemv_rows and gemv_ms else None,
            "down_tc_GBps": round(tc_bytes / (tc_ms * 1e-3) / 1e9, 1) if tc_rows and tc_ms else None,
            # the fused kernel reads each active row of W_up and of W_down once
            "updown_GBps": round(2 * u_bytes / (u_ms * 1e-3) / 1e9, 1) if u_ms else None,
            "dense_down_us": None if d_dense is None else round(1e3 * d_dense, 2),
        })

    peak, peak_kind = peaks()
    g_ach = gate_bytes_tot / (gate_ms_tot * 1e-3) / 1e9 if gate_ms_tot else 0.0
    n_gate_launches = args.steps * len(tokens)
    traffic_ok = kernel_source_hash(GATE_UP_TRAFFIC["files"]) == GATE_UP_TRAFFIC["source_sha16"]
    g_traffic = None if not traffic_ok or args.score != "h" else \
        round(GATE_UP_TRAFFIC["ratio"] * gate_bytes_tot / n_gate_launches)
    d_ach = down_bytes_tot / (down_ms_tot * 1e-3) / 1e9 if down_ms_tot else 0.0
    gv_ach = gemv_bytes_tot / (gemv_ms_tot * 1e-3) / 1e9 if gemv_ms_tot else 0.0
    # the gate/up kernel is HBM-bound below the ridge (decode, few tokens per
    # expert) and tensor-bound above it (prefill): grade it on its own bound
    tpeak, tpeak_kind = tensor_peak()
    intensity = gate_flops_tot / max(gate_bytes_tot, 1.0)
    ridge = tpeak * 1e12 / (peak * 1e9)
    if intensity > ridge:
        g_tf = gate_flops_tot / (gate_ms_tot * 1e-3) / 1e12 if gate_ms_tot else 0.0
        roofline_gate = {"kernel": "gate_up_tc", "bound": "tensor", "achieved": round(g_tf, 1),
                         "peak": tpeak, "unit": "TFLOP/s", "frac": round(g_tf / tpeak, 4),
                         "traffic": None,
                         "algorithmic_flops": round(gate_flops_tot / n_gate_launches),
                         "flop_per_byte": round(intensity, 1), "peak_kind": tpeak_kind}
    else:
        roofline_gate = {"kernel": "gate_up_tc (W_gate + W_up tiles, and the W_down rows of "
                                   "the groups whose down projection it does)",
                         "bound": "hbm", "achieved": round(g_ach, 1),
                         "peak": peak, "unit": "GB/s", "frac": round(g_ach / peak, 4),
                         "traffic": g_traffic,
                         "algorithmic_bytes": round(gate_bytes_tot / n_gate_launches),
                         "flop_per_byte": round(intensity, 1), "peak_kind": peak_kind}
    u_ach = up_bytes_tot / (up_ms_tot * 1e-3) / 1e9 if up_ms_tot else 0.0
    steps_launches = launches

    # end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        xs_pin = [x.pin_memory() for x in xs_host]
        outs_pin = [torch.empty((T, sh.d_model), dtype=x.dtype).pin_memory()
                    for T, x in zip(tokens, xs_host)]
        xs_dev = [torch.empty_like(x, device=dev) for x in xs_host]

        # the copies go on a stream of their own: all of a step's inputs go up
        # while the first batches compute, each forward waits for its own
        # input only, and each output comes back while the next batch
        # computes; the step ends when the last output is on the host
        copy_stream = torch.cuda.Stream(dev)

        def e2e_step():
            copy_stream.wait_stream(stream)  # the previous step no longer reads xs_dev
            up = []
            with torch.cuda.stream(copy_stream):
                for xp, xd in zip(xs_pin, xs_dev):
                    xd.copy_(xp, non_blocking=True)
                    ev = torch.cuda.Event()
                    ev.record(copy_stream)
                    up.append(ev)
            for ev, xd, o, op in zip(up, xs_dev, outs, outs_pin):
                stream.wait_event(ev)
                sparse.forward(xd, W["W_router"], W["W_gate"], W["W_up"], W["W_down"], tau,
                               sh.top_k, router_bias=W["router_bias"], out=o, stream=stream)
                done = torch.cuda.Event()
                done.record(stream)
                copy_stream.wait_event(done)
                with torch.cuda.stream(copy_stream):
                    op.copy_(o, non_blocking=True)
            stream.wait_stream(copy_stream)  # outputs on the host before the step ends
        for _ in range(args.warmup):
            e2e_step()
        torch.cuda.synchronize(dev)
        barrier(world)
        torch.cuda.synchronize(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.steps):
            e2e_step()
        b.record(stream)
        torch.cuda.synchronize(dev)
        barrier(world)
        ms_e2e = max_over_ranks(world, a.elapsed_time(b), local)
        nbytes = sum(x.numel() * x.element_size() for x in xs_host)
        e2e = {"value": replica_value(tok_step, args.steps, world, ms_e2e), "unit": "tokens/s",
               "h2d_bytes_per_step": nbytes, "d2h_bytes_per_step": nbytes,
               "copies": "pinned host buffers; inputs up and outputs down on a second stream, "
                         "overlapped with the other batches' compute; eager forwards"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        t = oracle_step_time(wl, tokens, tau, tau_s, w_host, args.score)
        cores = len(os.sched_getaffinity(0))
        cpu = {"value": tok_step / t, "unit": "tokens/s", "cores": cores, "kind": "oracle",
               "sample": f"one step: decode batches T={tokens} of {args.workload} through the "
                         f"fp64 numpy oracle on {cores} host threads ({t:.1f} s)"}

    sweep = None
    if sweep_on:
        # after every headline pass, with the headline's layer, graph and device
        # tensors released first: the sweep's layers then run in the same clean
        # device memory state from point to point (its own weights are drawn on
        # the host now)
        del g_sparse
        sparse.close()
        sparse = g_sparse = None
        W.clear()
        xs.clear()
        outs.clear()
        torch.cuda.synchronize(dev)
        torch.cuda.empty_cache()
        sweep = run_sweep(dev, local, args.warmup, args.reps)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_sparse / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": sh.dtype,
            "data": "synthetic",
            "config": workload_config(args, wl, tokens, tau, calib_sparsity, world),
            "roofline": roofline_gate,
            "roofline_down": {"kernel": "down (GEMV / TC / fused up+down, rows actually read)",
                              "bound": "hbm",
                              "achieved": round(d_ach, 1), "peak": peak, "unit": "GB/s",
                              "frac": round(d_ach / peak, 4), "peak_kind": peak_kind},
            "roofline_down_gemv": None if not gemv_ms_tot else
            {"kernel": "updown_gemv" if args.score == "gate" else "down_gemv",
             "bound": "hbm", "achieved": round(gv_ach, 1), "peak": peak, "unit": "GB/s",
             "frac": round(gv_ach / peak, 4), "peak_kind": peak_kind,
             "bytes": "union rows streamed by the row stream (W_up and W_down rows with the "
                      "gate score), batches where it had rows"},
            "roofline_updown": None if args.score != "gate" else
            {"kernel": "updown_gemv (gate score: W_up + W_down rows actually read)",
             "bound": "hbm", "achieved": round(2 * u_ach, 1), "peak": peak, "unit": "GB/s",
             "frac": round(2 * u_ach / peak, 4), "peak_kind": peak_kind},
            "dense": dense_line,
            "speedup_vs_dense": None if not dense_line else
            round(dense_line["ms_per_step"] / (ms_sparse / args.steps), 4),
            "per_T": per_T,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": steps_launches,
            "launch": "eager" if args.eager else "cuda_graph",
            "kernel_times": "second timed pass of the same steps with per-stage CUDA events",
            "clocks": clk,
            "sweep": sweep,
        }
        print(json.dumps(line), flush=True)
    if sparse is not None:
        del g_sparse
        sparse.close()
    return 0


def main():
    args = parse()
    world, rank, local = dist_init(args) if args.impl == "ours" else (
        int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")), 0)
    try:
        if args.impl == "reference":
            return run_reference(args, world, rank)
        return run_ours(args, world, rank, local)
    finally:
        if args.impl == "ours" and world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
