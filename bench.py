#!/usr/bin/env python
"""POET-X linear forward + backward throughput on B200 (tokens/s), with roofline figures.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl poetx|reference]

One step is one pass of the whole path over one batch of synthetic tokens:
merge of the two permutations into W0' -> CNP forward (input and output blocks) ->
layer forward (gather, block product, W0' GEMM, block product, scatter) -> layer
backward (dG_R, dW, dV, dU, dG_P, dX) -> CNP backward (dtheta).

Workload: the Llama-1B-shaped attention projection, n = m = 2048, b = 256, k = 4,
T = 8192 tokens (4 x 2048), bf16 activations, fp32 theta / CNP.  Inputs rotate over three
seeded sets (192 MB of x and dy, larger than the 126 MB L2) between steps.

Under torchrun (N > 1) the step is data parallel (weak scaling): every rank takes its own
T tokens with theta, G and W0' replicated, and the step ends with one NCCL sum all-reduce
of dtheta; the step time is the maximum over ranks.  The outer-loop merge (once per inner
loop, outside the step) is timed separately after the timed region.  ``--impl reference``
times the float64 CPU oracle instead (rank 0 only) on a bounded token sample per step.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "POET-X linear fwd+bwd tokens/s at 1 B200; achieved % of HBM/tensor roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
SM_COUNT = 148
FP32_LANES_PER_SM = 128
SM_MAX_MHZ = 1965.0

# DRAM bytes (read + write) per launch of a family's kernel from one ncu capture of the
# current kernel (cold caches; mean over the family's launches in one step); families
# without a capture of their current kernel report null.
MEASURED_TRAFFIC = {"cnp_sgemm": (2.141e6 + 0.0008e6 + 16.829e6 + 0.504e6) / 2}


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["poetx", "reference"], default="poetx")
    ap.add_argument("--workload", default="llama1b-attn",
                    choices=["llama1b-attn", "llama8b-up", "fp32-small"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--oracle-budget", type=float, default=20.0,
                    help="seconds of CPU work for the oracle baseline")
    ap.add_argument("--e2e-steps", type=int, default=40)
    ap.add_argument("--no-graph", dest="graph", action="store_false",
                    help="launch every kernel from the host instead of replaying CUDA graphs")
    return ap.parse_args(argv)


def workload(name):
    from poetx_inputs import workload_llama1b_attn, workload_llama8b_up, workload_small_fp32
    return {"llama1b-attn": workload_llama1b_attn, "llama8b-up": workload_llama8b_up,
            "fp32-small": workload_small_fp32}[name]()


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------ clocks sampler
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ algorithmic work
def family_work(s, ksplit_R=1, ksplit_P=1):
    """Algorithmic FLOPs / bytes per step for each kernel family of the bf16 path."""
    T, n, m, b, k = s.T, s.n, s.m, s.b, s.k
    es = 2 if s.dtype == "bf16" else 4
    nP, nR = n // b, m // b
    d = (k + 1) // 2
    cnp_fwd = (d + 1) * b ** 3                        # d symmetric powers + G (half products)
    y_terms = 0 if d == 1 else (2 * b ** 3 + (d - 2) * 3 * b ** 3)
    # the backward reads S and F' kept by the forward: D, the Horner terms, A
    cnp_bwd = 2 * b ** 3 + y_terms + 4 * b ** 3
    return {
        "gemm_w0": {"bound": "tensor", "flops": 2 * (2.0 * T * n * m), "launches": 2},
        "gemm_blockdiag": {"bound": "hbm", "launches": 4,
                           "bytes": 2.0 * es * T * (2 * n + 2 * m) + 2.0 * es * (nP + nR) * b * b},
        "gemm_dG": {"bound": "hbm", "launches": 2,
                    "bytes": 2.0 * es * T * (n + m) + 4.0 * (nP + nR) * b * b},
        "permute": {"bound": "hbm", "launches": 5,
                    "bytes": 2.0 * es * (m * n + 2 * T * n + 2 * T * m)},
        "cnp_sgemm": {"bound": "alu", "flops": float(nP + nR) * (cnp_fwd + cnp_bwd)},
    }


# ------------------------------------------------------------------ oracle timing
def oracle_inputs(s, T_sample=None):
    from poetx_inputs import layer_inputs
    inp = layer_inputs(s)
    return inp


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        n = [i.get("num_threads", 0) for i in info if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def oracle_step_sampler(s, inp, perms, budget_per_step):
    """Returns (run_one_step, tokens_per_step): the oracle on a token window of T_s tokens
    plus the amortised share of the per-step CNP work (b x b blocks, forward + backward)."""
    from oracle import poetx_ref as ref
    pP, pR = perms
    nblk = s.n // s.b + s.m // s.b
    theta = np.concatenate([inp.theta_P, inp.theta_R])
    W0p = ref.merge_perm(inp.W0, pR, pP)
    G_P = ref.cnp_forward(inp.theta_P, s.b, s.k)
    G_R = ref.cnp_forward(inp.theta_R, s.b, s.k)
    # calibration: one CNP block forward + backward, and the layer on 64 tokens
    t0 = time.perf_counter()
    g1 = ref.cnp_forward(theta[:1], s.b, s.k)
    ref.cnp_backward(theta[:1], g1, s.b, s.k)
    t_blk = time.perf_counter() - t0
    t0 = time.perf_counter()
    Tc = min(64, s.T)
    ref.layer_forward(inp.x[:Tc], W0p, G_P, G_R, pP, pR)
    ref.layer_backward(inp.x[:Tc], inp.dy[:Tc], W0p, G_P, G_R, pP, pR)
    t_tok = (time.perf_counter() - t0) / Tc
    per_tok = t_tok + t_blk * nblk / s.T
    T_s = int(max(1, min(s.T, budget_per_step / per_tok)))
    state = {"credit": 0.0, "t0": 0}

    def run_one():
        a = state["t0"] % s.T
        e = min(s.T, a + T_s)
        x, dy = inp.x[a:e], inp.dy[a:e]
        state["t0"] = e % s.T
        W0p_ = ref.merge_perm(inp.W0, pR, pP)
        y, U, V, W = ref.layer_forward(x, W0p_, G_P, G_R, pP, pR)
        ref.layer_backward(x, dy, W0p_, G_P, G_R, pP, pR, U=U, W=W)
        state["credit"] += nblk * (e - a) / s.T
        while state["credit"] >= 1.0:
            j = int(state["credit"] * 7919) % nblk
            G = ref.cnp_forward(theta[j:j + 1], s.b, s.k)
            ref.cnp_backward(theta[j:j + 1], G, s.b, s.k)
            state["credit"] -= 1.0
        return e - a

    return run_one, T_s


def oracle_throughput(s, budget_s):
    """Oracle tokens/s on a bounded sample of the workload (about budget_s of CPU work)."""
    from oracle import poetx_ref as ref
    inp = oracle_inputs(s)
    pP, _ = ref.make_perm(inp.seed_P, s.n)
    pR, _ = ref.make_perm(inp.seed_R, s.m)
    run_one, T_s = oracle_step_sampler(s, inp, (pP, pR), budget_per_step=budget_s / 4)
    run_one()  # warm
    tokens, t0 = 0, time.perf_counter()
    while time.perf_counter() - t0 < budget_s * 0.75:
        tokens += run_one()
    dt = time.perf_counter() - t0
    return {"value": tokens / dt, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"{s.name}: float64 oracle on windows of {T_s} of {s.T} tokens (fwd+bwd, "
                      f"merge each window) plus the per-token share of the CNP forward+backward "
                      f"of the {s.n // s.b + s.m // s.b} b={s.b} blocks; {tokens} tokens in "
                      f"{dt:.1f} s"}


# ------------------------------------------------------------------ reference arm
def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    s = workload(args.workload)
    from oracle import poetx_ref as ref
    inp = oracle_inputs(s)
    pP, _ = ref.make_perm(inp.seed_P, s.n)
    pR, _ = ref.make_perm(inp.seed_R, s.m)
    budget_total = 150.0
    run_one, T_s = oracle_step_sampler(s, inp, (pP, pR),
                                       budget_per_step=budget_total / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        run_one()
    tokens, t0 = 0, time.perf_counter()
    for _ in range(args.steps):
        tokens += run_one()
    dt = time.perf_counter() - t0
    value = tokens / dt
    cores = blas_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * dt / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": s.name, "T": s.T, "n": s.n, "m": s.m, "b": s.b, "k": s.k,
                   "tokens_per_step": T_s},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": f"{T_s} of {s.T} tokens per step plus the per-token share of "
                                   f"the CNP work, {args.steps} steps"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ multi-rank timing
def max_over_ranks(local_ms: float, dist=None, device=None) -> float:
    """The step region's device time as the maximum over ranks (replicas run in lock-step
    between barriers; the slowest rank defines the job's time)."""
    if dist is None or not dist.is_available() or not dist.is_initialized() or \
            dist.get_world_size() == 1:
        return float(local_ms)
    import torch
    t = torch.tensor([float(local_ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(world: int, tokens_per_rank_step: int, steps: int, max_ms: float) -> float:
    """Whole-job throughput: tokens processed by all ranks / slowest rank's time."""
    return world * tokens_per_rank_step * steps / (max_ms / 1e3)


# ------------------------------------------------------------------ GPU arm
def run_poetx(args):
    import torch
    import torch.distributed as dist

    from orthogonal_reparameterized_cnp_b200 import poetx as P
    from poetx_inputs import layer_inputs

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        print(json.dumps({"metric": METRIC, "error": "no CUDA device"}))
        return 1
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    s = workload(args.workload)
    inp = layer_inputs(s)
    act = torch.bfloat16 if s.dtype == "bf16" else torch.float32
    to = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a)).to(dev, dt)  # noqa: E731
    pP, _ = P.make_perm(inp.seed_P, s.n)
    pR, _ = P.make_perm(inp.seed_R, s.m)
    layer = P.PoetxLinear(to(inp.W0, act), to(inp.theta_P, torch.float32),
                          to(inp.theta_R, torch.float32), pP, pR, s.b, s.k, s.T)
    nsets = 3
    xs = [to(inp.x, act)]
    dys = [to(inp.dy, act)]
    for i in range(1, nsets):  # further sets: the same values rolled by i tokens
        xs.append(torch.roll(xs[0], shifts=i, dims=0).contiguous())
        dys.append(torch.roll(dys[0], shifts=i, dims=0).contiguous())
    y = torch.empty((s.T, s.m), dtype=act, device=dev)
    dx = torch.empty((s.T, s.n), dtype=act, device=dev)
    stream = torch.cuda.current_stream(dev)

    from orthogonal_reparameterized_cnp_b200 import dp

    def exchange():  # the data-parallel step's one collective (a no-op on one rank)
        if world > 1:
            dp.allreduce_dtheta(layer.dtheta)

    def step(i):
        layer.step(xs[i % nsets], dys[i % nsets], y, dx, stream)
        exchange()

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local])

    # warm-up
    for i in range(max(3, args.warmup)):
        step(i)
    torch.cuda.synchronize(dev)
    if P.device_status(stream) != P.POETX_OK:
        raise RuntimeError("device status not OK after warm-up")

    # per-family breakdown (short profiled pass, outside the timed region)
    work = family_work(s)
    breakdown = {}
    for fam in ["gemm_w0", "gemm_blockdiag", "gemm_dG", "permute", "cnp_sgemm",
                "cnp_elementwise", "reduce"]:
        P.profile_begin(fam)
        nprof = 10
        for i in range(nprof):
            step(i)
        torch.cuda.synchronize(dev)
        launches, ms = P.profile_end()
        breakdown[fam] = {"launches_per_step": launches / nprof, "ms_per_step": ms / nprof}
    dominant = max(breakdown, key=lambda f: breakdown[f]["ms_per_step"])

    # timed region
    props = torch.cuda.get_device_properties(dev)
    uuid = str(getattr(props, "uuid", "") or "")
    gpu_id = (uuid if uuid.startswith("GPU-") else f"GPU-{uuid}") if uuid else str(local)
    sampler = ClockSampler(gpu_id)
    # the whole step captured once per input set and replayed (no per-kernel host work)
    graphs = None
    graph_launches = 0
    if args.graph:
        graphs = []
        for i in range(nsets):
            gr = torch.cuda.CUDAGraph()
            n0 = P.launch_count()
            with torch.cuda.graph(gr):
                layer.step(xs[i], dys[i], y, dx, torch.cuda.current_stream(dev))
            graph_launches = P.launch_count() - n0
            graphs.append(gr)
        for i in range(3):
            graphs[i % nsets].replay()
            exchange()
        torch.cuda.synchronize(dev)
        if P.device_status(stream) != P.POETX_OK:
            raise RuntimeError("device status not OK after graph warm-up")
    barrier()
    torch.cuda.synchronize(dev)
    sampler.start()
    time.sleep(0.3)
    launches0 = P.launch_count()
    if not graphs:
        P.profile_begin(dominant)
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for i in range(args.steps):
        if graphs:
            graphs[i % nsets].replay()  # the layer's kernels; the collective stays outside
            exchange()
        else:
            step(i)
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    if graphs:
        launches = graph_launches * args.steps  # libpoetx kernels in the replayed graphs
    else:
        dom_launches, dom_ms = P.profile_end()
        launches = P.launch_count() - launches0
    barrier()
    clocks = sampler.stop()
    elapsed_ms = ev0.elapsed_time(ev1)
    if graphs:
        # per-launch device time of the dominant family: eager steps right after the timed
        # region, each of its launches bracketed by CUDA events on the launch stream
        P.profile_begin(dominant)
        for i in range(min(args.steps, 300)):
            step(i)
        torch.cuda.synchronize(dev)
        dom_launches, dom_ms = P.profile_end()
    max_ms = max_over_ranks(elapsed_ms, dist if world > 1 else None, dev)
    if P.device_status(stream) != P.POETX_OK:
        raise RuntimeError("device status not OK after the timed region")
    ms_per_step = max_ms / args.steps
    value = job_tokens_per_s(world, s.T, args.steps, max_ms)

    # roofline of the dominant kernel family
    peaks, peak_src = load_peaks()
    avg_launch_ms = dom_ms / max(1, dom_launches)
    w = work.get(dominant)
    roof = None
    if w is not None:
        # launches of the family per step (exact, from the profiled pre-pass); the event
        # pool may bracket fewer launches than the timed region makes
        per_launch_steps = breakdown[dominant]["launches_per_step"]
        if w["bound"] == "tensor":
            achieved = w["flops"] / per_launch_steps / (avg_launch_ms / 1e3) / 1e12 \
                if per_launch_steps else 0.0
            peak = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
            unit = "TFLOP/s"
        elif w["bound"] == "hbm":
            achieved = w["bytes"] / per_launch_steps / (avg_launch_ms / 1e3) / 1e9
            peak = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
            unit = "GB/s"
        else:
            achieved = w["flops"] / per_launch_steps / (avg_launch_ms / 1e3) / 1e12
            peak = SM_COUNT * FP32_LANES_PER_SM * 2 * SM_MAX_MHZ * 1e6 / 1e12
            unit = "TFLOP/s"
        roof = {"kernel": dominant, "bound": w["bound"], "achieved": achieved, "peak": peak,
                "unit": unit, "frac": achieved / peak if peak else None,
                "traffic": MEASURED_TRAFFIC.get(dominant),
                "peak_source": peak_src if w["bound"] != "alu" else
                "derived: 148 SM x 128 FP32 lanes x 2 x 1965 MHz",
                "avg_launch_ms": avg_launch_ms, "launches": dom_launches}
    for fam, bd in breakdown.items():
        ww = work.get(fam)
        if ww and bd["ms_per_step"] > 0:
            if "flops" in ww:
                bd["achieved_tflops"] = ww["flops"] / (bd["ms_per_step"] / 1e3) / 1e12
            if "bytes" in ww:
                bd["achieved_gbs"] = ww["bytes"] / (bd["ms_per_step"] / 1e3) / 1e9

    # end to end through the public API with host buffers (pinned), copies timed: every
    # step uploads its x, dy, theta and downloads y, dx, dtheta; the host pipeline runs
    # the uploads of the next step and the downloads of the previous one on the two copy
    # engines while a step computes
    e2e = None
    if args.e2e_steps > 0:
        from orthogonal_reparameterized_cnp_b200.host_pipeline import HostPipeline
        hx = [xs[i].cpu().pin_memory() for i in range(nsets)]
        hdy = [dys[i].cpu().pin_memory() for i in range(nsets)]
        hth = layer.theta.cpu().pin_memory()
        hy = torch.empty(y.shape, dtype=act).pin_memory()
        hdx = torch.empty(dx.shape, dtype=act).pin_memory()
        hdth = torch.empty(layer.dtheta.shape, dtype=torch.float32).pin_memory()
        pipe = HostPipeline(layer, nbuf=2, exchange=exchange if world > 1 else None)

        def e2e_step(i):
            pipe.submit(i, hx[i % nsets], hdy[i % nsets], hth, hy, hdx, hdth)

        for i in range(3):
            e2e_step(i)
        pipe.synchronize()
        barrier()
        torch.cuda.synchronize(dev)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(pipe.h2d)  # every step's first operation (its upload) follows this
        for i in range(args.e2e_steps):
            e2e_step(i)
        e1.record(pipe.d2h)  # the last download is the last operation of the last step
        pipe.synchronize()
        torch.cuda.synchronize(dev)
        e_ms = max_over_ranks(e0.elapsed_time(e1), dist if world > 1 else None, dev)
        h2d = hx[0].numel() * hx[0].element_size() + hdy[0].numel() * hdy[0].element_size() + \
            hth.numel() * 4
        d2h = hy.numel() * hy.element_size() + hdx.numel() * hdx.element_size() + hdth.numel() * 4
        e2e = {"value": job_tokens_per_s(world, s.T, args.e2e_steps, e_ms), "unit": "tokens/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "steps": args.e2e_steps, "copies": "overlapped with compute (2 buffer sets)"}
        if P.device_status(stream) != P.POETX_OK:
            raise RuntimeError("device status not OK after the end-to-end steps")

    # outer-loop merge (once per inner loop, not part of the step): device time per call
    outer = None
    if s.dtype == "bf16":
        pP2, _ = P.make_perm(inp.seed_P + 1000003, s.n)
        pR2, _ = P.make_perm(inp.seed_R + 1000003, s.m)
        i32 = lambda a: torch.as_tensor(np.asarray(a, dtype=np.int32), device=dev)  # noqa: E731
        pP2d, pR2d = i32(pP2), i32(pR2)
        W0p_new = torch.empty_like(layer.W0p)
        mws = torch.empty(P.outer_merge_workspace(s.m, s.n, P.POETX_BF16), dtype=torch.uint8,
                          device=dev)
        GP, GR = layer.G_ops()

        def merge_call():
            P.outer_merge(layer.W0p, GP, GR, s.b, layer.inv_P, layer.inv_R, pP2d, pR2d,
                          W0p_new, mws, stream)

        for _ in range(3):
            merge_call()
        reps = 20
        m0 = torch.cuda.Event(enable_timing=True)
        m1 = torch.cuda.Event(enable_timing=True)
        m0.record(stream)
        for _ in range(reps):
            merge_call()
        m1.record(stream)
        torch.cuda.synchronize(dev)
        mms = m0.elapsed_time(m1) / reps
        # algorithmic: read W0' and write W0'_new (bf16), read both G; 2 b-wide products
        mbytes = 2 * s.m * s.n * 2 + (s.n + s.m) * s.b * 2
        outer = {"ms": mms, "achieved_gbs": mbytes / (mms / 1e3) / 1e9,
                 "achieved_tflops": 4.0 * s.m * s.n * s.b / (mms / 1e3) / 1e12,
                 "launches": 5}
        if P.device_status(stream) != P.POETX_OK:
            raise RuntimeError("device status not OK after the outer merge")

    # the same step with the int8 merged weight (POET-XQ reading), CUDA-graph replay
    xq = None
    if s.dtype == "bf16" and args.graph:
        lq = P.PoetxLinear(to(inp.W0, act), to(inp.theta_P, torch.float32),
                           to(inp.theta_R, torch.float32), pP, pR, s.b, s.k, s.T,
                           int8_weight=True)
        for i in range(3):
            lq.step(xs[i % nsets], dys[i % nsets], y, dx, stream)
        torch.cuda.synchronize(dev)
        gq = []
        for i in range(nsets):
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr):
                lq.step(xs[i], dys[i], y, dx, torch.cuda.current_stream(dev))
            gq.append(gr)
        for i in range(3):
            gq[i % nsets].replay()
        nq = min(args.steps, 500)
        q0 = torch.cuda.Event(enable_timing=True)
        q1 = torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        q0.record(stream)
        for i in range(nq):
            gq[i % nsets].replay()
        q1.record(stream)
        torch.cuda.synchronize(dev)
        if P.device_status(stream) != P.POETX_OK:
            raise RuntimeError("device status not OK after the int8-weight steps")
        qms = q0.elapsed_time(q1) / nq
        xq = {"ms_per_step": qms, "tokens_per_s": s.T / (qms / 1e3), "steps": nq,
              "weight": "int8 W0' (per-row scales), dequantised into scratch per call"}
        del gq

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = oracle_throughput(s, args.oracle_budget)

    nblk = s.n // s.b + s.m // s.b
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if s.dtype == "bf16" else "f32", "data": "synthetic",
        "config": {"workload": s.name, "T": s.T, "n": s.n, "m": s.m, "b": s.b, "k": s.k,
                   "cnp_blocks_per_step": nblk,
                   "l2": f"inputs rotate over {nsets} sets of x and dy "
                         f"({nsets * (s.T * (s.n + s.m) * (2 if s.dtype == 'bf16' else 4)) >> 20} MB"
                         f" > 126 MB L2)",
                   "parallelism": f"dp{world}" if world > 1 else "single",
                   "launch": "cuda_graph" if graphs else "eager",
                   "roofline_timing": ("eager steps after the timed region" if graphs
                                       else "inside the timed region")},
        "clocks": clocks,
        "e2e": e2e,
        "gpu_launches": int(launches),
        "roofline": roof,
        "cpu_baseline": cpu,
        "kernels": breakdown,
        "outer_merge": outer,
        "int8_weight_step": xq,
        "cnp_blocks_per_s": world * nblk * args.steps / (max_ms / 1e3),
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier(device_ids=[local])
        dist.destroy_process_group()
    return 0


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    return run_poetx(args)


if __name__ == "__main__":
    sys.exit(main())
