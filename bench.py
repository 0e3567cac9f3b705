"""Benchmark of the activation-sparse linear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

(W below 3 is raised to 3; the JSON line reports the warm-up steps run.)

Workload (one step): one Llama-2-7B decoder layer's seven projections at
batch 1 (q, k, v, o 4096x4096; gate, up 4096->11008; down 11008->4096), fp16
weights ~ N(0, 0.02^2), Laplace activations, TEAL-style magnitude threshold
set at the 50 % quantile of |x|.  As in the model, q, k and v read one hidden
state and gate and up another, so the step is four fused
threshold -> compact -> split-K GEMV -> deterministic reduce launches:
(q|k|v), o, (gate|up), down; a shared input is read and masked once.

Metric: effective HBM GB/s = (kept weight rows + x + y bytes) / time, with
inputs resident in HBM; three copies of the layer's weights rotate so that
no step finds its weights in L2 (580 MB of kept rows per rotation, > 4x L2).
Steps are replayed CUDA graphs, timed with CUDA events on the launching stream.

The JSON line also carries the sparsity sweep, the top-k (Q-Sparse 70B), RaNA
gated-MLP, RaNA rank-adapter, per-token-mask batch, int8-weight and N:M GEMM rows, cuBLAS dense baselines at the same shapes, the
roofline of the sparse GEMV kernel, the oracle's CPU baseline and the SM
clocks sampled during the timed region.

Under torchrun (N > 1) every rank runs an independent replica (the method has
no exchange step); value = all ranks' bytes / max-over-ranks time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "sparse GEMV effective HBM GB/s (kept rows + x + y) at 50% sparsity, Llama-2-7B decode layer, batch 1"
UNIT = "GB/s"
HEADLINE_SPARSITY = 0.5
N_COPIES = 3


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--no-extras", action="store_true", help="skip the secondary rows")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--profile-case", default=None,
                    help="for ncu: run only this kernel case eagerly and exit "
                         "(a Llama-2-7B projection name or launch group such as 'q|k|v' or "
                         "'gate|up' at 50%%, 'topk70b', 'batchB' (B tokens, 4096->11008), "
                         "'q8up70b' / 'f8up70b' / 'q4up70b' (int8 / fp8 / int4 weights, "
                         "8192->28672), "
                         "'nmN:M' (N:M mask + GEMM, e.g. 'nm8:16'), 'nmsp2:4' (packed 2:4 "
                         "operand, sparse GEMM), 'nmex2:4', 'gemm:MxKxN' (dense "
                         "tensor-core GEMM) or 'gemmsp:MxKxN' (packed 2:4 GEMM)")
    ap.add_argument("--launches", type=int, default=8, help="launches in --profile-case mode")
    args = ap.parse_args()
    # at least three untimed warm-up steps; the JSON line reports the number run
    args.warmup = max(3, args.warmup)
    return args


# ---------------------------------------------------------------------------
# distributed plumbing
# ---------------------------------------------------------------------------

def dist_init(n_gpus):
    import torch
    import torch.distributed as dist
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v: float, world: int) -> float:
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate(units_per_rank: float, seconds_per_rank, world: int):
    """Whole-job throughput: all ranks' units over the slowest rank's time."""
    slow = max(seconds_per_rank)
    return units_per_rank * world / slow, slow


# ---------------------------------------------------------------------------
# clocks
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join(tempfile.gettempdir(), f"sig_clocks_rank{gpu_index}_{os.getpid()}.csv")

    def __enter__(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.fh, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.fh.close()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm, smax, reasons = [], None, set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for ln in open(self.path):
            f = [v.strip() for v in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        under_load = [v for v in sm if smax and v > 0.5 * smax] or sm
        return {"sm_mhz": float(np.median(under_load)) if under_load else None,
                "sm_max_mhz": smax, "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
# timing helpers
# ---------------------------------------------------------------------------

def capture(fn, stream):
    import torch
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        fn()
    return g


class StepGraphs:
    """CUDA graphs over a rotation of step callables.

    ``run(n)`` replays exactly ``n`` steps (step i uses fns[i % R]) as ONE
    graph of n steps when n <= ``cap``, so that no graph boundary falls inside
    the timed region and every launch can overlap its predecessor
    (programmatic dependent launch works inside a graph, not across two graph
    launches).  Longer runs replay a ``cap``-step graph (a multiple of R) and
    one graph of the remainder.  Graphs are captured on first use and cached
    by step count.  A graph's first launch also uploads it to the device, so
    ``warm(n)`` replays, untimed, every graph ``run(n)`` uses that has not run
    yet; ``warm_steps`` counts the untimed steps run.
    """

    def __init__(self, fns, stream, cap=600):
        import torch
        self.fns, self.R, self.stream = fns, len(fns), stream
        self.cap = max(self.R, (cap // self.R) * self.R)
        self.graphs = {}
        self.replayed = set()
        self.warm_steps = 0
        with torch.cuda.stream(stream):
            for f in fns:                      # one eager pass (kernel attributes)
                f()
        torch.cuda.synchronize()

    def _graph(self, n):
        g = self.graphs.get(n)
        if g is None:
            fns, R = self.fns, self.R

            def many():
                for i in range(n):
                    fns[i % R]()
            g = self.graphs[n] = capture(many, self.stream)
        return g

    def prepare(self, n):
        """Capture the graphs ``run(n)`` replays (outside any timed region)."""
        q, r = divmod(n, self.cap) if n > self.cap else (0, n)
        if q:
            self._graph(self.cap)
        if r:
            self._graph(r)

    def _replay(self, n):
        self._graph(n).replay()
        self.replayed.add(n)

    def run(self, n):
        q, r = divmod(n, self.cap) if n > self.cap else (0, n)
        for _ in range(q):
            self._replay(self.cap)
        if r:
            self._replay(r)

    def warm(self, n):
        """Replay once every graph that run(n) uses and that has not run yet."""
        q, r = divmod(n, self.cap) if n > self.cap else (0, n)
        for size in ([self.cap] if q else []) + ([r] if r else []):
            if size not in self.replayed:
                self._replay(size)
                self.warm_steps += size


def _queue_delay(stream, us=200.0):
    """Keep the device busy for ~``us`` microseconds before the start event, so
    that the host has queued the timed graph launches by the time the device
    reaches them (the wait for the host is then not inside the timed region)."""
    import torch
    with torch.cuda.stream(stream):
        torch.cuda._sleep(int(us * 2000))    # cycles at ~2 GHz


def time_steps(sg, steps, warmup, stream, world=1):
    """Warm up, then time exactly `steps` steps with CUDA events on `stream`."""
    import torch
    sg.prepare(warmup)
    sg.prepare(steps)
    with torch.cuda.stream(stream):
        sg.run(warmup)
        sg.warm_steps += warmup
        sg.warm(steps)            # the timed graphs' first launches (uploads), untimed
    barrier(world)
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    _queue_delay(stream)
    with torch.cuda.stream(stream):
        start.record(stream)
        sg.run(steps)
        end.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    return start.elapsed_time(end) / 1e3


def copy_peak_gbs(stream):
    """Read+write bytes / time of a 1 GiB device copy (best of 10)."""
    import torch
    a = torch.empty(1 << 29, dtype=torch.float16, device="cuda")
    b = torch.empty_like(a)
    a.fill_(1.0)
    best = float("inf")
    with torch.cuda.stream(stream):
        for _ in range(12):
            s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s.record(stream)
            b.copy_(a)
            e.record(stream)
            e.synchronize()
            best = min(best, s.elapsed_time(e) / 1e3)
    del a, b
    return 2 * (1 << 30) / best / 1e9


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d.get("hbm_gbs"), d.get("bf16_tflops"), "measured"
    return 6650.0, 1590.0, "fallback"


def kernel_source_hash():
    h = hashlib.sha256()
    for f in ("gemv.cu", "common.cuh", "internal.h"):
        h.update(open(os.path.join(ROOT, "sparse_input_gemv_threshold_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def ncu_traffic_per_launch():
    """DRAM bytes per GEMV launch from the committed ncu summary, valid only if
    the kernel source still hashes to what was profiled."""
    p = os.path.join(ROOT, "profiles", "sgemv_llama2_7b_layer_traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    if d.get("kernel_source_hash") != kernel_source_hash():
        return None
    return d.get("dram_bytes_per_launch_avg")


# ---------------------------------------------------------------------------
# our implementation
# ---------------------------------------------------------------------------

# Projections that read the same input, in launch order.
GROUPS = (("q", "k", "v"), ("o",), ("gate", "up"), ("down",))


def layer_groups(projs):
    by = {p.name: p for p in projs}
    return [[by[n] for n in g] for g in GROUPS]


def kept_count(p, sparsity):
    return int((np.abs(p.x.astype(np.float32)) >= p.thresholds[sparsity]).sum())


def kept_counts(projs, sparsity):
    return [kept_count(p, sparsity) for p in projs]


def group_bytes(group, nnz):
    """Kept rows of every weight in the group + the shared x once + each y."""
    dsum = sum(p.d_out for p in group)
    return nnz * 2 * dsum + 2 * group[0].d_in + 2 * dsum


def layer_bytes(groups, sparsity):
    return sum(group_bytes(g, kept_count(g[0], sparsity)) for g in groups)


def launch_group(sig, W, x, t, ys, ws, stream):
    """One launch for every projection that reads x."""
    if len(W) == 1:
        sig.sparse_gemv(W[0], x, t=t, y=ys[0], ws=ws, stream=stream)
    else:
        sig.sparse_gemv_multi(W, x, t=t, ys=ys, ws=ws, stream=stream)


def group_workspace(sig, group):
    import torch
    if len(group) == 1:
        n = sig.workspace_bytes(sig.OP_SPARSE_GEMV, group[0].d_in, group[0].d_out)
    else:
        n = sig.workspace_bytes_multi([p.d_out for p in group], group[0].d_in)
    return torch.zeros(max(n, 256), dtype=torch.uint8, device="cuda")


def run_ours(args, rank, world, local):
    import torch
    import sparse_input_gemv_threshold_b200 as sig

    stream = torch.cuda.Stream()
    projs = workloads.llama2_7b_layer(args.seed)
    groups = layer_groups(projs)
    gx = [torch.from_numpy(g[0].x).cuda() for g in groups]
    first = [[torch.from_numpy(p.WT).cuda() for p in g] for g in groups]
    copies = [first] + [[[w.clone() for w in g] for g in first] for _ in range(N_COPIES - 1)]
    gys = [[torch.empty(p.d_out, dtype=torch.float16, device="cuda") for p in g] for g in groups]
    gws = [group_workspace(sig, g) for g in groups]

    def step_fn(c, s):
        def f():
            for gi, g in enumerate(groups):
                launch_group(sig, copies[c][gi], gx[gi], g[0].thresholds[s], gys[gi], gws[gi],
                             stream)
        return f

    def graphs_for(s):
        return StepGraphs([step_fn(c, s) for c in range(N_COPIES)], stream)

    # ---- headline ----
    g50 = graphs_for(HEADLINE_SPARSITY)
    nnz50 = [kept_count(g[0], HEADLINE_SPARSITY) for g in groups]
    bytes_step = layer_bytes(groups, HEADLINE_SPARSITY)
    n_launch = len(groups)
    with ClockSampler(local) as clk:
        secs = time_steps(g50, args.steps, args.warmup, stream, world)
    clocks = clk.summary()
    slow = max_over_ranks(secs, world)
    value = bytes_step * args.steps * world / slow / 1e9
    ms_per_step = slow / args.steps * 1e3

    hbm_peak, bf16_peak, peak_kind = measured_peaks()
    result = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": g50.warm_steps, "ms_per_step": round(ms_per_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f16",
        "data": "synthetic",
        "config": {"workload": "llama2_7b_decode_layer_b1", "projections": "q,k,v,o 4096x4096; gate,up 4096->11008; down 11008->4096",
                   "launches": "(q|k|v) o (gate|up) down: q,k,v share one input and one mask, gate,up another",
                   "batch": 1, "sparsity": HEADLINE_SPARSITY, "mask": "threshold |x|>=t, t=50% quantile of |x|",
                   "weights": "fp16 N(0,0.02^2), transposed (d_in x d_out)", "x": "fp16 Laplace(0,1)",
                   "seed": args.seed, "parallelism": f"replicas x{world}",
                   "l2": f"inputs larger than L2: {N_COPIES} rotating weight copies, "
                         f"{N_COPIES * bytes_step / 1e6:.0f} MB of kept rows per rotation",
                   "bytes_per_step": bytes_step, "nnz_per_launch": nnz50},
        "gpu_launches": n_launch * args.steps,
        "clocks": clocks,
    }
    us_launch = slow / args.steps / n_launch * 1e6
    traffic = ncu_traffic_per_launch()
    result["roofline"] = {
        "kernel": "sgemv_kernel (fused threshold + split-K GEMV + reduce)", "bound": "hbm",
        "achieved": round(bytes_step / n_launch / (us_launch * 1e-6) / 1e9, 1), "peak": hbm_peak,
        "peak_kind": f"{peak_kind} hbm_gbs", "unit": "GB/s",
        "frac": round(bytes_step / n_launch / (us_launch * 1e-6) / 1e9 / hbm_peak, 4),
        "traffic": traffic, "algorithmic_bytes_per_launch": bytes_step // n_launch,
        "avg_launch_us": round(us_launch, 3),
    }

    # ---- e2e through the public API with host buffers ----
    result["e2e"] = e2e(args, groups, copies, gws, stream, sig, world, bytes_step)

    if not args.no_extras and rank == 0:
        extras = {}
        extras["copy_probe_gbs"] = round(copy_peak_gbs(stream), 1)
        steps_x = max(50, min(args.steps // 10, 2000))
        sweep = []
        for s in workloads.LLAMA2_SPARSITIES:
            gs = g50 if s == HEADLINE_SPARSITY else graphs_for(s)
            b = layer_bytes(groups, s)
            sec = time_steps(gs, steps_x, 24, stream)
            us = sec / steps_x * 1e6
            sweep.append({"sparsity": s, "us_per_step": round(us, 2),
                          "GBps": round(b / (us * 1e-6) / 1e9, 1),
                          "frac_of_peak": round(b / (us * 1e-6) / 1e9 / hbm_peak, 4)})
            if gs is not g50:
                del gs
        extras["sweep_llama2_7b_layer"] = sweep
        extras["per_launch_us_at_50"] = per_launch(groups, copies, gx, gys, gws, stream, sig,
                                                   steps_x)
        extras["seven_single_launches"] = seven_launches(groups, copies, gx, stream, sig, steps_x,
                                                         bytes_step)
        extras["cublas_dense_layer_us"] = cublas_dense(groups, copies, gx, stream, steps_x)
        del g50
        torch.cuda.synchronize()
        del copies[1:]
        torch.cuda.empty_cache()
        extras["topk_qsparse_70b"] = bench_topk(args, stream, sig, hbm_peak)
        extras["rana_gated_mlp"] = bench_rana(args, stream, sig, hbm_peak)
        extras["nm_gemm"] = bench_nm(args, stream, sig, bf16_peak)
        extras["teal_mlp"] = bench_teal_mlp(args, stream, sig, hbm_peak)
        extras["rana_rank_adapter"] = bench_rank_adapter(args, stream, sig, hbm_peak)
        extras["batched_per_token_masks"] = bench_batch(args, stream, sig, hbm_peak)
        extras["int8_weights"] = bench_q8(args, stream, sig, hbm_peak, "int8")
        extras["fp8_weights"] = bench_q8(args, stream, sig, hbm_peak, "fp8")
        extras["int4_weights"] = bench_q8(args, stream, sig, hbm_peak, "int4")
        result["extras"] = extras
        result["cpu_baseline"] = cpu_baseline(groups)
    return result


def per_launch(groups, copies, gx, gys, gws, stream, sig, steps):
    out = {}
    for gi, grp in enumerate(groups):
        def f(c, gi=gi, grp=grp):
            def g():
                launch_group(sig, copies[c][gi], gx[gi], grp[0].thresholds[HEADLINE_SPARSITY],
                             gys[gi], gws[gi], stream)
            return g
        sg = StepGraphs([f(c) for c in range(N_COPIES)], stream)
        sec = time_steps(sg, steps, 24, stream)
        us = sec / steps * 1e6
        b = group_bytes(grp, kept_count(grp[0], HEADLINE_SPARSITY))
        out["|".join(p.name for p in grp)] = {"us": round(us, 2),
                                              "GBps": round(b / (us * 1e-6) / 1e9, 1)}
    return out


def seven_launches(groups, copies, gx, stream, sig, steps, bytes_step):
    """The same layer as seven single-weight launches (each re-reads and
    re-masks its input), for comparison with the grouped launches."""
    import torch
    flat = [(gi, j, p) for gi, g in enumerate(groups) for j, p in enumerate(g)]
    ys = [torch.empty(p.d_out, dtype=torch.float16, device="cuda") for _, _, p in flat]
    wss = [torch.zeros(max(256, sig.workspace_bytes(sig.OP_SPARSE_GEMV, p.d_in, p.d_out)),
                       dtype=torch.uint8, device="cuda") for _, _, p in flat]

    def f(c):
        def g():
            for k, (gi, j, p) in enumerate(flat):
                sig.sparse_gemv(copies[c][gi][j], gx[gi], t=p.thresholds[HEADLINE_SPARSITY],
                                y=ys[k], ws=wss[k], stream=stream)
        return g
    sg = StepGraphs([f(c) for c in range(N_COPIES)], stream)
    sec = time_steps(sg, steps, 24, stream)
    us = sec / steps * 1e6
    return {"us_per_step": round(us, 2), "GBps_same_bytes": round(bytes_step / (us * 1e-6) / 1e9, 1)}


def cublas_dense(groups, copies, gx, stream, steps):
    """Dense fp16 GEMV through torch (cuBLAS), same shapes, same weight rotation."""
    import torch
    flat = [(gi, j, p) for gi, g in enumerate(groups) for j, p in enumerate(g)]
    outs = [torch.empty((1, p.d_out), dtype=torch.float16, device="cuda") for _, _, p in flat]

    def f(c):
        def g():
            for k, (gi, j, p) in enumerate(flat):
                torch.matmul(gx[gi].view(1, -1), copies[c][gi][j], out=outs[k])
        return g
    sg = StepGraphs([f(c) for c in range(N_COPIES)], stream)
    sec = time_steps(sg, steps, 24, stream)
    us = sec / steps * 1e6
    dense_bytes = sum(sum(p.d_in * p.d_out * 2 + 2 * p.d_out for p in g) + 2 * g[0].d_in
                      for g in groups)
    return {"us_per_step": round(us, 2), "GBps": round(dense_bytes / (us * 1e-6) / 1e9, 1)}


def bench_topk(args, stream, sig, hbm_peak):
    """Q-Sparse top-k then the index-list GEMV, both 70B MLP shapes, at the
    keep fractions 0.6, 0.5 and 0.4 of d_in."""
    import torch
    projs = workloads.qsparse_70b(args.seed)
    W = [torch.from_numpy(p.WT).cuda() for p in projs]
    Wc = [w.clone() for w in W]
    X = [torch.from_numpy(p.x).cuda() for p in projs]
    ys = [torch.empty(p.d_out, dtype=torch.float16, device="cuda") for p in projs]
    ws = [torch.zeros(sig.workspace_bytes(sig.OP_SPARSE_GEMV, p.d_in, p.d_out), dtype=torch.uint8,
                      device="cuda") for p in projs]
    bufs = [(torch.empty((p.d_in + 31) // 32, dtype=torch.int32, device="cuda"),
             torch.empty(p.d_in, dtype=torch.int32, device="cuda"),
             torch.empty(1, dtype=torch.int32, device="cuda")) for p in projs]
    steps = 200
    by_keep = {}
    for k_frac in (0.6, 0.5, 0.4):
        ks = [workloads.topk_count(k_frac, p.d_in) for p in projs]

        def f(ws_w, ks=ks):
            def g():
                for j, p in enumerate(projs):
                    mb, idx, nnz = bufs[j]
                    sig.sparsify_topk(X[j], ks[j], mask_bits=mb, idx=idx, nnz=nnz, stream=stream)
                    sig.sparse_gemv(ws_w[j], X[j], idx=idx, nnz=nnz, y=ys[j], ws=ws[j], stream=stream)
            return g
        sg = StepGraphs([f(W), f(Wc)], stream)
        sec = time_steps(sg, steps, 8, stream)
        us = sec / steps * 1e6
        b = sum(k * 2 * p.d_out + 2 * p.d_in + 2 * p.d_out for k, p in zip(ks, projs))

        def h(ks=ks):   # top-k alone
            for j, p in enumerate(projs):
                mb, idx, nnz = bufs[j]
                sig.sparsify_topk(X[j], ks[j], mask_bits=mb, idx=idx, nnz=nnz, stream=stream)
        st = StepGraphs([h], stream)
        sec_t = time_steps(st, steps, 8, stream)
        by_keep[k_frac] = {"keep": k_frac, "k": ks, "us_per_pair": round(us, 2),
                           "GBps": round(b / (us * 1e-6) / 1e9, 1),
                           "frac_of_peak": round(b / (us * 1e-6) / 1e9 / hbm_peak, 4),
                           "topk_select_us_per_pair": round(sec_t / steps * 1e6, 2)}
        del sg, st
    res = {"shapes": "8192->28672 and 28672->8192", **by_keep[0.5],
           "by_keep": [by_keep[k] for k in (0.6, 0.5, 0.4)],
           "l2": "2 rotating weight copies of 940 MB"}
    del W, Wc
    torch.cuda.empty_cache()
    return res


def bench_rana(args, stream, sig, hbm_peak):
    import torch
    mlp = workloads.rana_mlp(args.seed)
    x = torch.from_numpy(mlp.x).cuda()
    Ws = [tuple(torch.from_numpy(a).cuda() for a in (mlp.WgT, mlp.WuT, mlp.WdT))]
    Ws.append(tuple(w.clone() for w in Ws[0]))
    norms = sig.row_norms(Ws[0][2])
    h = torch.empty(mlp.WgT.shape[1], dtype=torch.float16, device="cuda")
    y = torch.empty(mlp.WgT.shape[0], dtype=torch.float16, device="cuda")
    mask = torch.empty((mlp.WgT.shape[1] + 31) // 32, dtype=torch.int32, device="cuda")
    ws = torch.zeros(sig.workspace_bytes(sig.OP_GATED_MLP, *mlp.WgT.shape), dtype=torch.uint8,
                     device="cuda")
    # threshold: 50 % quantile of this path's own scores (timing only)
    sig.gated_mlp_sparse(x, *Ws[0], norms, 0.0, y=y, h_out=h, ws=ws)
    s = (h.float().abs() * norms).cpu().numpy()
    t = float(np.sort(s)[len(s) // 2])

    def f(W):
        def g():
            sig.gated_mlp_sparse(x, *W, norms, t, y=y, h_out=h, mask_out=mask, ws=ws, stream=stream)
        return g
    nnz = int((s >= t).sum())
    sg = StepGraphs([f(W) for W in Ws], stream)
    steps = 300
    sec = time_steps(sg, steps, 8, stream)
    us = sec / steps * 1e6
    d_model, d_ff = mlp.WgT.shape
    b = 2 * d_model * d_ff * 2 + nnz * 2 * d_model + 2 * d_model + 2 * d_ff * 2 + 4 * d_ff
    res = {"shapes": "4096->11008 x2 dense, 11008->4096 sparse", "sparsity": round(1 - nnz / d_ff, 4),
           "us": round(us, 2), "GBps": round(b / (us * 1e-6) / 1e9, 1),
           "frac_of_peak": round(b / (us * 1e-6) / 1e9 / hbm_peak, 4),
           "l2": "2 rotating weight copies of 258 MB"}
    del Ws, sg
    torch.cuda.empty_cache()
    return res


def bench_teal_mlp(args, stream, sig, hbm_peak):
    """Gated MLP with the 50 % threshold on x (gate and up, one fused launch)
    and the 50 % threshold on h (down), Llama-2-7B MLP shapes."""
    import torch
    mlp = workloads.rana_mlp(args.seed)
    d_model, d_ff = mlp.WgT.shape
    xh = workloads.draw_vector(np.random.default_rng(args.seed), d_model, "laplace")
    t_x = workloads.quantile_threshold(xh, 0.5)
    x = torch.from_numpy(xh).cuda()
    Ws = [tuple(torch.from_numpy(a).cuda() for a in (mlp.WgT, mlp.WuT, mlp.WdT))]
    Ws += [tuple(w.clone() for w in Ws[0]) for _ in range(2)]
    h = torch.empty(d_ff, dtype=torch.float16, device="cuda")
    y = torch.empty(d_model, dtype=torch.float16, device="cuda")
    ws = torch.zeros(sig.workspace_bytes(sig.OP_GATED_MLP, d_model, d_ff), dtype=torch.uint8,
                     device="cuda")
    # t_h: 50 % quantile of this path's own h (timing only)
    sig.teal_mlp_sparse(x, *Ws[0], t_x, 0.0, y=y, h_out=h, ws=ws)
    hv = h.float().abs().cpu().numpy()
    t_h = float(np.sort(hv)[d_ff // 2])
    nnz_x = int((np.abs(xh.astype(np.float32)) >= t_x).sum())
    nnz_h = int((hv >= t_h).sum())

    def f(W):
        def g():
            sig.teal_mlp_sparse(x, *W, t_x, t_h, y=y, h_out=h, ws=ws, stream=stream)
        return g
    sg = StepGraphs([f(W) for W in Ws], stream)
    steps = 300
    us = time_steps(sg, steps, 12, stream) / steps * 1e6
    b = nnz_x * 2 * d_ff * 2 + nnz_h * 2 * d_model + 2 * d_model * 2 + 2 * d_ff * 2
    res = {"shapes": "4096->11008 x2 (threshold on x), 11008->4096 (threshold on h)",
           "sparsity_x": round(1 - nnz_x / d_model, 4), "sparsity_h": round(1 - nnz_h / d_ff, 4),
           "us": round(us, 2), "GBps": round(b / (us * 1e-6) / 1e9, 1),
           "frac_of_peak": round(b / (us * 1e-6) / 1e9 / hbm_peak, 4),
           "l2": "3 rotating weight copies of 271 MB"}
    del Ws, sg
    torch.cuda.empty_cache()
    return res


def bench_rank_adapter(args, stream, sig, hbm_peak):
    """RaNA rank adapter A (m . Bx) replacing one 4096 x 4096 projection, r = 2048."""
    import torch
    ra = workloads.rank_adapter(args.seed)
    d_in, r = ra.BT.shape
    d_out = ra.AT.shape[1]
    copies = 16                      # 16 x 33.6 MB of factors rotate, > 4x L2
    Bs = [torch.from_numpy(ra.BT).cuda()]
    As = [torch.from_numpy(ra.AT).cuda()]
    Bs += [Bs[0].clone() for _ in range(copies - 1)]
    As += [As[0].clone() for _ in range(copies - 1)]
    x = torch.from_numpy(ra.x).cuda()
    y = torch.empty(d_out, dtype=torch.float16, device="cuda")
    v = torch.empty(r, dtype=torch.float16, device="cuda")
    ws = torch.zeros(sig.workspace_bytes(sig.OP_RANK_ADAPTER, d_in, d_out, r), dtype=torch.uint8,
                     device="cuda")
    # threshold: 50 % quantile of this path's own scores v_i^2 (timing only)
    sig.rank_adapter_sparse(x, Bs[0], As[0], 0.0, y=y, v_out=v, ws=ws)
    sc = v.float().square().cpu().numpy()
    t = float(np.sort(sc)[r // 2])
    nnz = int((sc >= t).sum())

    def f(c):
        def g():
            sig.rank_adapter_sparse(x, Bs[c], As[c], t, y=y, v_out=v, ws=ws, stream=stream)
        return g
    sg = StepGraphs([f(c) for c in range(copies)], stream)
    steps = 320
    sec = time_steps(sg, steps, copies, stream)
    us = sec / steps * 1e6
    b = 2 * d_in * r + nnz * 2 * d_out + 2 * d_in + 4 * r + 2 * d_out
    # the dense projection the adapter stands in for, through torch (cuBLAS)
    W = [torch.empty((d_in, d_out), dtype=torch.float16, device="cuda").normal_(0, 0.02)
         for _ in range(copies)]
    yd = torch.empty((1, d_out), dtype=torch.float16, device="cuda")

    def dn(c):
        def g():
            torch.matmul(x.view(1, -1), W[c], out=yd)
        return g
    sd = StepGraphs([dn(c) for c in range(copies)], stream)
    us_dense = time_steps(sd, steps, copies, stream) / steps * 1e6
    res = {"shapes": f"B {r}x{d_in} dense, A {d_out}x{r} masked", "sparsity": round(1 - nnz / r, 4),
           "us": round(us, 2), "GBps": round(b / (us * 1e-6) / 1e9, 1),
           "frac_of_peak": round(b / (us * 1e-6) / 1e9 / hbm_peak, 4),
           "cublas_dense_4096x4096_us": round(us_dense, 2),
           "l2": f"{copies} rotating copies of the factors (538 MB)"}
    del Bs, As, W, sg, sd
    torch.cuda.empty_cache()
    return res


def bench_batch(args, stream, sig, hbm_peak):
    """A few tokens with their own 50 % threshold masks through the gate-shaped
    weight (4096 -> 11008): one batched launch that reads the union of the
    kept rows once, against one single-token launch per token."""
    import torch
    out = {"shape": "4096->11008", "l2": "6 rotating weight copies (541 MB)"}
    copies = 6
    for B in (2, 4, 8, 16):
        WT, X, t = workloads.batch_tokens(seed=args.seed + B, B=B)
        Ws = [torch.from_numpy(WT).cuda()]
        Ws += [Ws[0].clone() for _ in range(copies - 1)]
        Xd = torch.from_numpy(X).cuda()
        Y = torch.empty((B, WT.shape[1]), dtype=torch.float16, device="cuda")
        ws = torch.zeros(max(256, sig.workspace_bytes(sig.OP_SPARSE_GEMV_BATCH, WT.shape[0],
                                                      WT.shape[1], B)), dtype=torch.uint8, device="cuda")
        m = np.abs(X.astype(np.float32)) >= t
        union = int(m.any(axis=0).sum())

        def f(c, B=B):
            def g():
                sig.sparse_gemv_batch(Ws[c], Xd, t, Y=Y, ws=ws, stream=stream)
            return g
        sg = StepGraphs([f(c) for c in range(copies)], stream)
        steps = 240
        us = time_steps(sg, steps, copies, stream) / steps * 1e6
        d_in, d_out = WT.shape
        b = union * 2 * d_out + B * (2 * d_in + 2 * d_out)
        ys = [torch.empty(d_out, dtype=torch.float16, device="cuda") for _ in range(B)]
        wss = [torch.zeros(max(256, sig.workspace_bytes(sig.OP_SPARSE_GEMV, d_in, d_out)),
                           dtype=torch.uint8, device="cuda") for _ in range(B)]

        def h(c, B=B):
            def g():
                for j in range(B):
                    sig.sparse_gemv(Ws[c], Xd[j], t=t, y=ys[j], ws=wss[j], stream=stream)
            return g
        sh = StepGraphs([h(c) for c in range(copies)], stream)
        us_sep = time_steps(sh, steps, copies, stream) / steps * 1e6
        out[f"B={B}"] = {"union_density": round(union / d_in, 4), "us": round(us, 2),
                         "GBps": round(b / (us * 1e-6) / 1e9, 1),
                         "frac_of_peak": round(b / (us * 1e-6) / 1e9 / hbm_peak, 4),
                         "separate_single_token_launches_us": round(us_sep, 2)}
        del Ws, sg, sh
        torch.cuda.empty_cache()
    return out


def bench_q8(args, stream, sig, hbm_peak, fmt="int8"):
    """Quantised weights (int8, fp8 e4m3 or int4; one scale per column) at the
    Llama-2-7B shapes and a Llama-70B MLP shape, 50 % threshold, against the
    fp16 sparse GEMV on the same shapes."""
    import torch
    gen, call, op = {
        "int8": (workloads.q8_projection, sig.sparse_gemv_q8, sig.OP_SPARSE_GEMV_Q8),
        "fp8": (workloads.f8_projection, sig.sparse_gemv_f8, sig.OP_SPARSE_GEMV_F8),
        "int4": (workloads.q4_projection, sig.sparse_gemv_q4, sig.OP_SPARSE_GEMV_Q4)}[fmt]
    row_bytes = (lambda d_out: d_out // 2) if fmt == "int4" else (lambda d_out: d_out)
    out = {"note": f"{fmt} kept rows cost {'d_out / 2' if fmt == 'int4' else 'd_out'} bytes; "
                   "fp16 rows 2 d_out"}
    for name, d_in, d_out in (("q", 4096, 4096), ("gate", 4096, 11008), ("down", 11008, 4096),
                              ("70B up", 8192, 28672)):
        QT, scale, x, ts = gen(seed=args.seed + d_in + d_out, d_in=d_in, d_out=d_out)
        t = ts[0.5]
        copies = max(2, math.ceil(4 * 126e6 / (d_in * row_bytes(d_out))))
        Qs = [torch.from_numpy(QT).cuda()]
        Qs += [Qs[0].clone() for _ in range(copies - 1)]
        sd = torch.from_numpy(scale).cuda()
        xd = torch.from_numpy(x).cuda()
        y = torch.empty(d_out, dtype=torch.float16, device="cuda")
        ws = torch.zeros(max(256, sig.workspace_bytes(op, d_in, d_out)), dtype=torch.uint8,
                         device="cuda")

        def f(c):
            def g():
                call(Qs[c], sd, xd, t, y=y, ws=ws, stream=stream)
            return g
        sg = StepGraphs([f(c) for c in range(copies)], stream)
        steps = 400
        us = time_steps(sg, steps, copies, stream) / steps * 1e6
        nnz = int((np.abs(x.astype(np.float32)) >= t).sum())
        b = nnz * row_bytes(d_out) + 2 * d_in + 2 * d_out
        # the fp16 sparse GEMV on a weight of the same shape
        Ws = [torch.empty((d_in, d_out), dtype=torch.float16, device="cuda").normal_(0, 0.02)
              for _ in range(max(2, math.ceil(4 * 126e6 / (2 * d_in * d_out))))]
        ws16 = torch.zeros(max(256, sig.workspace_bytes(sig.OP_SPARSE_GEMV, d_in, d_out)),
                           dtype=torch.uint8, device="cuda")

        def h(c):
            def g():
                sig.sparse_gemv(Ws[c], xd, t=t, y=y, ws=ws16, stream=stream)
            return g
        sh = StepGraphs([h(c) for c in range(len(Ws))], stream)
        us16 = time_steps(sh, steps, len(Ws), stream) / steps * 1e6
        out[f"{name} {d_in}->{d_out}"] = {"us": round(us, 2), "GBps": round(b / (us * 1e-6) / 1e9, 1),
                                          "frac_of_peak": round(b / (us * 1e-6) / 1e9 / hbm_peak, 4),
                                          "fp16_sparse_us": round(us16, 2),
                                          "speedup_vs_fp16": round(us16 / us, 3)}
        del Qs, Ws, sg, sh
        torch.cuda.empty_cache()
    return out


def bench_nm(args, stream, sig, bf16_peak):
    import torch
    WT, X = workloads.nm_tokens(args.seed)
    rows, K = X.shape
    N = WT.shape[1]
    copies = 16
    Xs = [torch.from_numpy(X).cuda()]
    Xs += [Xs[0].clone() for _ in range(copies - 1)]
    Ws = [torch.from_numpy(WT).cuda()]
    Ws += [Ws[0].clone() for _ in range(copies - 1)]
    Y = torch.empty((rows, N), dtype=torch.float16, device="cuda")
    ws = torch.zeros(sig.workspace_bytes(sig.OP_NM_GEMM, K, N, rows), dtype=torch.uint8, device="cuda")
    flops_dense = 2.0 * rows * K * N
    out = {"shape": f"X {rows}x{K}, WT {K}x{N}", "l2": f"{copies} rotating input copies"}
    steps = 200
    for n, m in workloads.NM_PATTERNS:
        def f(c, n=n, m=m):
            def g():
                sig.nm_act_gemm(Xs[c], Ws[c], n, m, Y=Y, ws=ws, stream=stream)
            return g
        sg = StepGraphs([f(c) for c in range(copies)], stream)
        sec = time_steps(sg, steps, copies, stream)
        us = sec / steps * 1e6
        Xm = torch.empty_like(Xs[0])

        def mk(c, n=n, m=m):
            def g():
                sig.sparsify_nm(Xs[c], n, m, X_masked=Xm, want_bits=False, stream=stream)
            return g
        sm = StepGraphs([mk(c) for c in range(copies)], stream)
        us_mask = time_steps(sm, steps, copies, stream) / steps * 1e6
        row = {"us": round(us, 2),
               "TFLOPs_executed": round(flops_dense / (us * 1e-6) / 1e12, 1),
               "TFLOPs_algorithmic": round(flops_dense * n / m / (us * 1e-6) / 1e12, 1),
               "mask_only_us": round(us_mask, 2),
               "mask_GBps": round(2 * X.nbytes / (us_mask * 1e-6) / 1e9, 1)}
        if m == 4 and n <= 2:
            # the sparse tensor-core path: pack, then the 2:4 GEMM on the packed operand
            row["path"] = "packed 2:4 operand, tcgen05.mma.sp"
            row["TFLOPs_executed"] = round(flops_dense / 2 / (us * 1e-6) / 1e12, 1)
            row["TFLOPs_dense_equivalent"] = round(flops_dense / (us * 1e-6) / 1e12, 1)
            pk = [sig.sparsify_nm_packed(Xs[c], n) for c in range(2)]

            def fp(c, n=n):
                def g():
                    sig.sparsify_nm_packed(Xs[c], n, out=pk[c % 2], stream=stream)
                return g

            def fg(c):
                def g():
                    sig.nm_act_gemm_packed(pk[c % 2], rows, K, Ws[c], Y=Y, stream=stream)
                return g
            sp = StepGraphs([fp(c) for c in range(copies)], stream)
            us_pack = time_steps(sp, steps, copies, stream) / steps * 1e6
            sgm = StepGraphs([fg(c) for c in range(copies)], stream)
            us_gemm = time_steps(sgm, steps, copies, stream) / steps * 1e6
            pbytes = X.nbytes + sig.nm_packed_bytes(rows, K)
            row.update({"pack_only_us": round(us_pack, 2),
                        "pack_GBps": round(pbytes / (us_pack * 1e-6) / 1e9, 1),
                        "sparse_gemm_only_us": round(us_gemm, 2),
                        "sparse_gemm_TFLOPs_dense_equivalent":
                            round(flops_dense / (us_gemm * 1e-6) / 1e12, 1)})
            del pk, sp, sgm
        else:
            row["path"] = "masked X, dense tcgen05.mma"
        out[f"{n}:{m}"] = row
    Yd = torch.empty_like(Y)

    def d(c):
        def g():
            torch.matmul(Xs[c], Ws[c], out=Yd)
        return g
    sg = StepGraphs([d(c) for c in range(copies)], stream)
    sec = time_steps(sg, steps, copies, stream)
    us = sec / steps * 1e6
    out["cublas_dense"] = {"us": round(us, 2), "TFLOPs": round(flops_dense / (us * 1e-6) / 1e12, 1)}
    # the mitigation variants on 2:4: per-token shift (mean of the token), WT
    # scores with the weight's row norms, VAR; the shift added back in the GEMM
    shifts = [x.float().mean(dim=1).contiguous() for x in Xs[:2]]
    norms = sig.row_norms(Ws[0])
    csum = sig.col_sums_of(Ws[0])
    for label, kw in (("2:4 WT", {"norms": norms}), ("2:4 PTS+VAR", {"var": True}),
                      ("2:4 WT+PTS+VAR", {"norms": norms, "var": True})):
        use_shift = "PTS" in label

        def fv(c, kw=kw, use_shift=use_shift):
            def g():
                sig.nm_act_gemm_ex(Xs[c], Ws[c], 2, 4, shift=shifts[c % 2] if use_shift else None,
                                   col_sums=csum if use_shift else None, Y=Y, ws=ws, stream=stream, **kw)
            return g
        sv = StepGraphs([fv(c) for c in range(copies)], stream)
        usv = time_steps(sv, steps, copies, stream) / steps * 1e6
        out[label] = {"us": round(usv, 2), "TFLOPs_executed": round(flops_dense / (usv * 1e-6) / 1e12, 1)}
    out["tensor_peak_tflops"] = bf16_peak
    return out


def e2e(args, groups, copies, gws, stream, sig, world, bytes_step):
    """Public binding calls with host buffers.  Every step copies the layer's
    inputs in from pinned host memory (the four x vectors, one buffer, one
    copy), runs the four launches through the binding, and copies the seven y
    vectors (views of one device buffer) out to pinned host memory in one
    copy.  The copies run on their own streams with two buffers each way, so
    that step i+1's input copy and step i-1's output copy overlap step i's
    launches, as a serving loop would run them.  Timed two ways: the steps
    captured into CUDA graphs and replayed (how a decoding loop runs them),
    and the same calls issued eagerly from Python."""
    import torch
    d_ins = [g[0].d_in for g in groups]
    d_outs = [[p.d_out for p in g] for g in groups]
    xh = torch.from_numpy(np.concatenate([g[0].x for g in groups])).pin_memory()
    nx, ny = sum(d_ins), sum(sum(d) for d in d_outs)
    xd_all = [torch.empty(nx, dtype=torch.float16, device="cuda") for _ in range(2)]
    yd_all = [torch.empty(ny, dtype=torch.float16, device="cuda") for _ in range(2)]
    yh = [torch.empty(ny, dtype=torch.float16).pin_memory() for _ in range(2)]
    xd, ys = [], []
    for b in range(2):
        xs, o = [], 0
        for di in d_ins:
            xs.append(xd_all[b][o:o + di])
            o += di
        yb, o = [], 0
        for ds in d_outs:
            yb.append([])
            for dj in ds:
                yb[-1].append(yd_all[b][o:o + dj])
                o += dj
        xd.append(xs)
        ys.append(yb)
    cs_in, cs_out = torch.cuda.Stream(), torch.cuda.Stream()

    def steps(n, c0):
        """Enqueue n pipelined steps; returns after `stream` has joined both copy streams."""
        fork = torch.cuda.Event()
        fork.record(stream)
        cs_in.wait_event(fork)
        cs_out.wait_event(fork)
        comp, out = [None, None], [None, None]
        for i in range(n):
            b, c = i % 2, (c0 + i) % len(copies)
            with torch.cuda.stream(cs_in):
                if comp[b] is not None:        # step i-2 has finished reading x[b]
                    cs_in.wait_event(comp[b])
                xd_all[b].copy_(xh, non_blocking=True)
                ev_in = torch.cuda.Event()
                ev_in.record(cs_in)
            stream.wait_event(ev_in)
            if out[b] is not None:             # step i-2's y[b] has been copied out
                stream.wait_event(out[b])
            for gi, g in enumerate(groups):
                launch_group(sig, copies[c][gi], xd[b][gi], g[0].thresholds[HEADLINE_SPARSITY],
                             ys[b][gi], gws[gi], stream)
            comp[b] = torch.cuda.Event()
            comp[b].record(stream)
            with torch.cuda.stream(cs_out):
                cs_out.wait_event(comp[b])
                yh[b].copy_(yd_all[b], non_blocking=True)
                out[b] = torch.cuda.Event()
                out[b].record(cs_out)
        join = torch.cuda.Event()
        join.record(cs_in)
        stream.wait_event(join)
        for e in out:
            if e is not None:
                stream.wait_event(e)

    n_steps = max(200, min(args.steps, 1200))
    per = 600 if n_steps > 600 else n_steps
    chunks = [per] * (n_steps // per) + ([n_steps % per] if n_steps % per else [])
    with torch.cuda.stream(stream):
        steps(2 * len(copies), 0)             # eager warm-up
    torch.cuda.synchronize()
    graphs = {n: capture(lambda n=n: steps(n, 0), stream) for n in set(chunks)}

    def timed(run):
        torch.cuda.synchronize()
        barrier(world)
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        _queue_delay(stream)
        with torch.cuda.stream(stream):
            s.record(stream)
            run()
            e.record(stream)
        torch.cuda.synchronize()
        return max_over_ranks(s.elapsed_time(e) / 1e3, world)

    def replay_all():
        for n in chunks:
            graphs[n].replay()

    timed(replay_all)                                                 # warm-up
    sec = timed(replay_all)
    n_eager = max(50, min(args.steps, 400))

    def eager():
        # one stream, in order: copy in, the four binding calls, copy out
        for i in range(n_eager):
            b, c = i % 2, i % len(copies)
            xd_all[b].copy_(xh, non_blocking=True)
            for gi, g in enumerate(groups):
                launch_group(sig, copies[c][gi], xd[b][gi], g[0].thresholds[HEADLINE_SPARSITY],
                             ys[b][gi], gws[gi], stream)
            yh[b].copy_(yd_all[b], non_blocking=True)
    timed(eager)                                                      # warm-up
    sec_e = timed(eager)
    del graphs
    return {"value": round(bytes_step * n_steps * world / sec / 1e9, 1), "unit": UNIT,
            "steps": n_steps, "us_per_step": round(sec / n_steps * 1e6, 2),
            "h2d_bytes_per_step": 2 * nx, "d2h_bytes_per_step": 2 * ny,
            "eager_value": round(bytes_step * n_eager * world / sec_e / 1e9, 1),
            "eager_steps": n_eager, "eager_us_per_step": round(sec_e / n_eager * 1e6, 2),
            "note": "weights resident (model parameters, the same rotating copies as the device "
                    "timing); every step copies the layer's four x vectors in from pinned host "
                    "memory (one copy) and its seven y vectors out to pinned host memory (one "
                    "copy), on two copy streams with double buffers so the copies of steps i+1 "
                    "and i-1 overlap step i's launches; value: the steps' binding calls captured "
                    "in CUDA graphs and replayed; eager_value: the same calls and copies issued "
                    "from Python every step on one stream, in order (the binding's per-call host "
                    "cost is paid each step)"}


# ---------------------------------------------------------------------------
# CPU baseline / reference arm: the oracle as it stands
# ---------------------------------------------------------------------------

def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        return int(max(n)) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def cpu_model():
    """The host CPU's model name and logical core count (as nproc reports)."""
    name = None
    try:
        for ln in open("/proc/cpuinfo"):
            if ln.lower().startswith("model name"):
                name = ln.split(":", 1)[1].strip()
                break
    except OSError:
        pass
    try:
        nproc = len(os.sched_getaffinity(0))
    except AttributeError:
        nproc = os.cpu_count()
    return name or "unknown", nproc


def oracle_sample(groups, cols_per_proj, rng):
    """Run the oracle on `cols_per_proj` output columns of every projection,
    one mask per shared input; returns (algorithmic bytes of the sample, seconds)."""
    import oracle
    b = 0
    t0 = time.perf_counter()
    for g in groups:
        m = oracle.threshold_mask(g[0].x, g[0].thresholds[HEADLINE_SPARSITY])
        for p in g:
            cols = rng.choice(p.d_out, cols_per_proj, replace=False)
            oracle.sparse_linear(p.WT, p.x, m, cols=cols)
        b += int(m.sum()) * 2 * cols_per_proj * len(g) + 2 * g[0].d_in + 2 * cols_per_proj * len(g)
    return b, time.perf_counter() - t0


def _timed_oracle(groups, budget_s, rng):
    _, t1 = oracle_sample(groups, 256, rng)                      # warm-up and calibration
    reps = max(1, int(budget_s / max(t1, 1e-3)))
    tot_b, tot_t = 0, 0.0
    for _ in range(reps):
        b, t = oracle_sample(groups, 256, rng)
        tot_b += b
        tot_t += t
    return tot_b / tot_t / 1e9, reps, tot_t


def cpu_baseline(groups, budget_s=8.0):
    """The oracle as it stands on the host cores: once with the BLAS thread
    pool at its default (all cores) and once limited to one thread."""
    from threadpoolctl import threadpool_limits
    rng = np.random.default_rng(0)
    name, nproc = cpu_model()
    threads = _blas_threads()
    v_all, reps, tot = _timed_oracle(groups, budget_s, rng)
    with threadpool_limits(limits=1, user_api="blas"):
        v_one, reps1, tot1 = _timed_oracle(groups, budget_s, rng)
    return {"value": round(v_all, 4), "unit": UNIT, "cores": threads, "kind": "oracle",
            "cpu_model": name, "nproc": nproc,
            "single_thread": {"value": round(v_one, 4), "cores": 1,
                              "sample": f"{reps1} passes ({tot1:.1f} s)"},
            "sample": f"{reps} passes over the 7 projections, 256 random output columns each, "
                      f"one 50% threshold mask per shared input, numpy float64 ({tot:.1f} s, "
                      f"BLAS on {threads} threads); single_thread: the same with one BLAS thread"}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    groups = layer_groups(workloads.llama2_7b_layer(args.seed))
    rng = np.random.default_rng(1)
    # size the per-step sample so that warmup + steps stay within ~90 s
    _, t64 = oracle_sample(groups, 64, rng)
    per_step = 90.0 / max(1, args.steps + args.warmup)
    cols = int(max(1, min(4096, 64 * per_step / max(t64, 1e-6))))
    for _ in range(args.warmup):
        oracle_sample(groups, cols, rng)
    tot_b, tot_t = 0, 0.0
    for _ in range(args.steps):
        b, t = oracle_sample(groups, cols, rng)
        tot_b += b
        tot_t += t
    value = tot_b / tot_t / 1e9
    sample = (f"each step: the 7 projections' oracle product on {cols} random output columns "
              f"(one 50% threshold mask per shared input, numpy float64)")
    return {"metric": METRIC, "value": round(value, 4), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(tot_t / max(1, args.steps) * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": "llama2_7b_decode_layer_b1", "batch": 1,
                       "sparsity": HEADLINE_SPARSITY, "seed": args.seed, "parallelism": "cpu"},
            "cpu_baseline": {"value": round(value, 4), "unit": UNIT, "cores": _blas_threads(),
                             "kind": "oracle", "sample": sample, "cpu_model": cpu_model()[0],
                             "nproc": cpu_model()[1]},
            "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
            "gpu_launches": 0}


def profile_case(args):
    """A few eager launches of one kernel case, inputs larger than L2, for ncu."""
    import torch
    import sparse_input_gemv_threshold_b200 as sig
    torch.cuda.set_device(0)
    case = args.profile_case
    group_names = {"|".join(g): g for g in GROUPS}
    group_names.update({n: (n,) for n, _, _ in workloads.LLAMA2_7B_PROJECTIONS})
    if case in group_names:
        by = {p.name: p for p in workloads.llama2_7b_layer(args.seed)}
        grp = [by[n] for n in group_names[case]]
        wbytes = sum(p.d_in * p.d_out * 2 for p in grp)
        copies = max(2, math.ceil(4 * 126e6 / wbytes))
        W = [[torch.from_numpy(p.WT).cuda() for p in grp]]
        W += [[w.clone() for w in W[0]] for _ in range(copies - 1)]
        x = torch.from_numpy(grp[0].x).cuda()
        ys = [torch.empty(p.d_out, dtype=torch.float16, device="cuda") for p in grp]
        ws = group_workspace(sig, grp)
        for i in range(args.launches):
            launch_group(sig, W[i % copies], x, grp[0].thresholds[HEADLINE_SPARSITY], ys, ws, None)
        info = {"case": case, "launches": args.launches, "copies": copies,
                "algorithmic_bytes_per_launch": group_bytes(grp, kept_count(grp[0], HEADLINE_SPARSITY))}
    elif case.startswith("batch"):
        B = int(case[5:])
        WT, X, t = workloads.batch_tokens(seed=args.seed + B, B=B)
        copies = 6
        Ws = [torch.from_numpy(WT).cuda()]
        Ws += [Ws[0].clone() for _ in range(copies - 1)]
        Xd = torch.from_numpy(X).cuda()
        for i in range(args.launches):
            sig.sparse_gemv_batch(Ws[i % copies], Xd, t)
        union = int((np.abs(X.astype(np.float32)) >= t).any(axis=0).sum())
        info = {"case": case, "launches": args.launches, "copies": copies,
                "algorithmic_bytes_per_launch": union * 2 * WT.shape[1] + B * 2 * sum(WT.shape)}
    elif case in ("q8up70b", "f8up70b", "q4up70b"):
        make, run = {"q8up70b": (workloads.q8_projection, sig.sparse_gemv_q8),
                     "f8up70b": (workloads.f8_projection, sig.sparse_gemv_f8),
                     "q4up70b": (workloads.q4_projection, sig.sparse_gemv_q4)}[case]
        QT, scale, x, ts = make(seed=args.seed, d_in=8192, d_out=28672)
        copies = 3 if case != "q4up70b" else 5     # every copy larger than the L2
        Qs = [torch.from_numpy(QT).cuda()]
        Qs += [Qs[0].clone() for _ in range(copies - 1)]
        sd, xd = torch.from_numpy(scale).cuda(), torch.from_numpy(x).cuda()
        for i in range(args.launches):
            run(Qs[i % copies], sd, xd, ts[0.5])
        nnz = int((np.abs(x.astype(np.float32)) >= ts[0.5]).sum())
        info = {"case": case, "launches": args.launches, "copies": copies,
                "algorithmic_bytes_per_launch": nnz * QT.shape[1] + 2 * 8192 + 2 * 28672}
    elif case == "nmex2:4":
        WT, X = workloads.nm_tokens(args.seed)
        Xd, Wd = torch.from_numpy(X).cuda(), torch.from_numpy(WT).cuda()
        shift = Xd.float().mean(dim=1).contiguous()
        norms = sig.row_norms(Wd)
        for _ in range(args.launches):
            sig.sparsify_nm_ex(Xd, 2, 4, shift=shift, norms=norms, var=True, want_bits=False)
        info = {"case": case, "launches": args.launches}
    elif case in ("nmsp2:4", "nmsp1:4"):
        WT, X = workloads.nm_tokens(args.seed)
        n = int(case[4])
        copies = 8
        Xs = [torch.from_numpy(X).cuda() for _ in range(copies)]
        Wd = torch.from_numpy(WT).cuda()
        pk = [sig.sparsify_nm_packed(x, n) for x in Xs]
        for i in range(args.launches):
            sig.sparsify_nm_packed(Xs[i % copies], n, out=pk[i % copies])
            sig.nm_act_gemm_packed(pk[i % copies], X.shape[0], X.shape[1], Wd)
        info = {"case": case, "launches": args.launches}
    elif re.fullmatch(r"nm\d+:\d+", case):
        n, m = (int(v) for v in case[2:].split(":"))
        WT, X = workloads.nm_tokens(args.seed)
        Xd, Wd = torch.from_numpy(X).cuda(), torch.from_numpy(WT).cuda()
        for _ in range(args.launches):
            Y = sig.nm_act_gemm(Xd, Wd, n, m)
        info = {"case": case, "launches": args.launches}
    elif re.fullmatch(r"gemm(sp)?:\d+x\d+x\d+", case):
        # one large tensor-core GEMM: dense on X ('gemm:MxKxN') or the packed
        # 2:4 operand ('gemmsp:MxKxN'), for the CTA-pair kernels
        M, K, N = (int(v) for v in case.split(":")[1].split("x"))
        gen = torch.Generator(device="cpu").manual_seed(M + K + N)
        Xd = torch.randn(M, K, generator=gen).half().cuda()
        Wd = (torch.randn(K, N, generator=gen) * 0.02).half().cuda()
        if case.startswith("gemmsp"):
            pk = sig.sparsify_nm_packed(Xd, 2)
            for _ in range(args.launches):
                sig.nm_act_gemm_packed(pk, M, K, Wd)
        else:
            for _ in range(args.launches):
                sig.nm_act_gemm(Xd, Wd, 4, 4)
        info = {"case": case, "launches": args.launches}
    elif case == "topk70b":
        (p,) = workloads.qsparse_70b(args.seed, names=("down",))
        x = torch.from_numpy(p.x).cuda()
        for _ in range(args.launches):
            sig.sparsify_topk(x, workloads.topk_count(0.5, p.d_in))
        info = {"case": case, "launches": args.launches}
    else:
        raise SystemExit(f"unknown profile case {case!r}")
    torch.cuda.synchronize()
    print(json.dumps(info))
    return 0


def main():
    args = parse()
    if args.profile_case:
        return profile_case(args)
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        res = run_reference(args, rank, int(os.environ.get("WORLD_SIZE", "1")))
        if res is not None:
            print(json.dumps(res), flush=True)
        return 0
    rank, world, local = dist_init(args.gpus)
    res = run_ours(args, rank, world, local)
    if rank == 0:
        print(json.dumps(res), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
