#!/usr/bin/env python
"""POET-X linear forward + backward throughput on B200 (tokens/s), with roofline figures.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl poetx|reference]
                    [--workload llama13b-block|llama8b-up|llama1b-attn|fp32-small]

One step is one pass of the per-step path over one batch of synthetic tokens: CNP forward
(every block of the workload, one call) -> every linear's forward (gather, block product,
W0' GEMM, block product, scatter) -> every linear's backward (dG_R, dW, dV, dU, dG_P, dX)
-> CNP backward (dtheta of every block, one call).  The permutations are drawn and merged
into W0' once per set of permutations (once per outer iteration), so that merge is not
part of the step; its time is reported separately.

Default workload: the Llama-13B-shaped decoder block, all 7 linears as POET-X layers
(q, k, v, o 5120 -> 5120; gate, up 5120 -> 13824; down 13824 -> 5120), b = 256, k = 4,
T = 8192 tokens, bf16 activations, fp32 theta / CNP, 382 CNP blocks.  The step touches
several GB, far more than the 126 MB L2, so consecutive steps never find their inputs in
L2; for workloads whose inputs fit in L2, a buffer of twice the L2 is written before every
timed step (outside that step's events), so each step starts from a cold L2.

Besides the headline line the run measures: the layer-only figure (forward + backward
without the CNP), CNP-only forward and backward (blocks/s), per-kernel-family device time
from CUDA-graph replays, the FP32 FMA peak of the device, and (default workload only, under
"also") the Llama-8B up-projection step, the fp32 small layer's CUDA-graph latency and the
CNP sweep over b in {64, 128, 256, 512} and k in {2, 4, 6}.

Under torchrun (N > 1) the step is data parallel (weak scaling): every rank takes its own
T tokens with theta, G and W0' replicated, and the step ends with one NCCL sum all-reduce
of dtheta; the step time is the maximum over ranks.  ``--impl reference`` times the float64
CPU oracle instead (rank 0 only) on a bounded token sample per step.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
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
L2_BYTES = 126 << 20
FAMILIES = ["gemm_w0", "gemm_blockdiag", "gemm_dG", "permute", "cnp_sgemm", "cnp_elementwise",
            "reduce"]
WORKLOADS = ["llama13b-block", "llama8b-up", "llama1b-attn", "fp32-small"]
# kernel source of each family: a committed DRAM-traffic figure applies only while the
# source it was captured from is unchanged
# the sources whose kernels a family's launches run (a committed traffic figure is used only
# while all of them are unchanged)
FAMILY_SOURCES = {
    "gemm_w0": ("kernels_umma2.cu", "kernels_umma.cu", "umma_ptx.cuh"),
    "gemm_blockdiag": ("kernels_umma.cu", "umma_ptx.cuh"),
    "gemm_dG": ("kernels_umma.cu", "umma_ptx.cuh"), "permute": ("kernels_perm.cu",),
    "cnp_sgemm": ("kernels_cnp_graph.cu",), "reduce": ("kernels_sgemm.cu",),
}
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "dram_traffic.md")


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["poetx", "reference"], default="poetx")
    ap.add_argument("--workload", default="llama13b-block", choices=WORKLOADS)
    ap.add_argument("--no-also", dest="also", action="store_false",
                    help="skip the secondary workloads of the default run")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--oracle-budget", type=float, default=20.0,
                    help="seconds of CPU work for the oracle baseline")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--no-graph", dest="graph", action="store_false",
                    help="launch every kernel from the host instead of replaying CUDA graphs")
    return ap.parse_args(argv)


def workload(name):
    """The linears of a named workload (LayerShape list; one entry except the 13B block)."""
    from poetx_inputs import (workload_llama13b_block, workload_llama1b_attn,
                              workload_llama8b_up, workload_small_fp32)
    if name == "llama13b-block":
        return workload_llama13b_block()
    return [{"llama8b-up": workload_llama8b_up, "llama1b-attn": workload_llama1b_attn,
             "fp32-small": workload_small_fp32}[name]()]


def workload_name(name, shapes):
    s = shapes[0]
    if name == "llama13b-block":
        return f"llama13b-block-7linears-d5120-ffn13824-b{s.b}-k{s.k}-T{s.T}"
    return s.name


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured (MEASURED_PEAKS.json)"
    return dict(FALLBACK_PEAKS), "fallback (no MEASURED_PEAKS.json on this box)"


def source_sha(fnames) -> str:
    """First 16 hex digits of the SHA-256 of the named kernel sources, concatenated."""
    h = hashlib.sha256()
    for fname in ((fnames,) if isinstance(fnames, str) else fnames):
        with open(os.path.join(ROOT, "orthogonal_reparameterized_cnp_b200", "csrc", fname),
                  "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def committed_traffic(family: str, workload_key: str):
    """DRAM bytes (read + write) per launch of `family` on `workload_key` from the committed
    ncu summary, or None when there is none or its kernel source has changed since."""
    if not os.path.exists(TRAFFIC_FILE) or family not in FAMILY_SOURCES:
        return None
    sha = source_sha(FAMILY_SOURCES[family])
    pat = re.compile(r"^\|\s*" + re.escape(family) + r"\s*\|\s*" + re.escape(workload_key) +
                     r"\s*\|\s*([0-9.eE+]+)\s*\|\s*([0-9a-f]{16})\s*\|")
    with open(TRAFFIC_FILE) as f:
        for line in f:
            m = pat.match(line.strip())
            if m and m.group(2) == sha:
                return float(m.group(1))
    return None


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
def cnp_flops_per_block(b: int, k: int):
    """(forward, backward) FLOPs of one block as the library computes it, counting a
    product whose result is symmetric (or symmetric + skew) as half a product: forward
    d + 1 half products (the d powers of S = Q^2, the last emitting E and F', then G);
    backward with Q, S and F' kept: D = Q dG (2 b^3), the Horner terms of the adjoint
    through S (d = 2: N_2 S, 2 b^3; d = 3: three more full products and one half
    product: 7 b^3 in all), A = f_0 dG + dG F' - Y Q (4 b^3)."""
    d = (k + 1) // 2
    fwd = (d + 1) * b ** 3
    horner = {1: 0, 2: 2, 3: 7}[d] * b ** 3
    return float(fwd), float(2 * b ** 3 + horner + 4 * b ** 3)


def family_work(shapes):
    """Algorithmic FLOPs / bytes per step (all linears of the workload) of each kernel
    family, and its launches per step."""
    es = 2 if shapes[0].dtype == "bf16" else 4
    T, b, k = shapes[0].T, shapes[0].b, shapes[0].k
    w0 = bd = dg = perm = 0.0
    nblk = 0
    for s in shapes:
        n, m = s.n, s.m
        nP, nR = n // b, m // b
        nblk += nP + nR
        w0 += 2 * (2.0 * T * n * m)
        # F1, F3, B1, B3: read and write one activation each, plus the G blocks
        bd += 2.0 * es * T * (2 * n + 2 * m) + 2.0 * es * (nP + nR) * b * b
        # dG_R, dG_P: read both activations, write the fp32 block gradients
        dg += 2.0 * es * T * (n + m) + 4.0 * (nP + nR) * b * b
        # gathers of x and dy, scatters of y and dx: one read and one write each
        perm += 2.0 * es * (2 * T * n + 2 * T * m)
    L = len(shapes)
    cf, cb = cnp_flops_per_block(b, k)
    return {
        "gemm_w0": {"bound": "tensor", "flops": w0, "launches": 2 * L},
        "gemm_blockdiag": {"bound": "hbm", "bytes": bd, "launches": 4 * L},
        "gemm_dG": {"bound": "hbm", "bytes": dg, "launches": 2 * L},
        "permute": {"bound": "hbm", "bytes": perm, "launches": 4 * L},
        "cnp_sgemm": {"bound": "alu", "flops": nblk * (cf + cb), "launches": 2,
                      "flops_fwd": nblk * cf, "flops_bwd": nblk * cb},
    }


# ------------------------------------------------------------------ oracle timing
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


class OracleSampler:
    """The float64 oracle on token windows of every linear of the workload, plus the
    per-token share of the per-step CNP work (forward + backward of each b x b block)."""

    def __init__(self, shapes, budget_per_step: float):
        from oracle import poetx_ref as ref
        from poetx_inputs import layer_inputs
        self.ref = ref
        self.shapes = shapes
        self.T = shapes[0].T
        self.b, self.k = shapes[0].b, shapes[0].k
        self.lin = []
        thetas = []
        for s in shapes:
            inp = layer_inputs(s)
            pP, _ = ref.make_perm(inp.seed_P, s.n)
            pR, _ = ref.make_perm(inp.seed_R, s.m)
            W0p = ref.merge_perm(inp.W0.astype(np.float64), pR, pP)
            G_P = ref.cnp_forward(inp.theta_P, s.b, s.k)
            G_R = ref.cnp_forward(inp.theta_R, s.b, s.k)
            self.lin.append((inp.x, inp.dy, W0p, G_P, G_R, pP, pR))
            thetas += [inp.theta_P, inp.theta_R]
        self.theta = np.concatenate(thetas)
        self.nblk = len(self.theta)
        # calibration: one CNP block forward + backward, and every linear on 32 tokens
        t0 = time.perf_counter()
        g1 = ref.cnp_forward(self.theta[:1], self.b, self.k)
        ref.cnp_backward(self.theta[:1], g1, self.b, self.k)
        t_blk = time.perf_counter() - t0
        Tc = min(32, self.T)
        t0 = time.perf_counter()
        self._layers(0, Tc)
        t_tok = (time.perf_counter() - t0) / Tc
        per_tok = t_tok + t_blk * self.nblk / self.T
        self.T_s = int(max(1, min(self.T, budget_per_step / per_tok)))
        self.credit = 0.0
        self.t0 = 0

    def _layers(self, a, e):
        ref = self.ref
        for x, dy, W0p, G_P, G_R, pP, pR in self.lin:
            y, U, V, W = ref.layer_forward(x[a:e], W0p, G_P, G_R, pP, pR)
            ref.layer_backward(x[a:e], dy[a:e], W0p, G_P, G_R, pP, pR, U=U, W=W)

    def run_one(self) -> int:
        ref = self.ref
        a = self.t0 % self.T
        e = min(self.T, a + self.T_s)
        self.t0 = e % self.T
        self._layers(a, e)
        self.credit += self.nblk * (e - a) / self.T
        while self.credit >= 1.0:
            j = int(self.credit * 7919) % self.nblk
            G = ref.cnp_forward(self.theta[j:j + 1], self.b, self.k)
            ref.cnp_backward(self.theta[j:j + 1], G, self.b, self.k)
            self.credit -= 1.0
        return e - a

    def describe(self, name):
        return (f"{name}: float64 oracle on windows of {self.T_s} of {self.T} tokens through "
                f"all {len(self.shapes)} linear(s) (forward + backward) plus the per-token "
                f"share of the CNP forward + backward of the {self.nblk} b={self.b} blocks")


def oracle_throughput(name, shapes, budget_s):
    """Oracle tokens/s on a bounded sample of the workload (about budget_s of CPU work)."""
    smp = OracleSampler(shapes, budget_per_step=budget_s / 4)
    smp.run_one()  # warm
    tokens, t0 = 0, time.perf_counter()
    while time.perf_counter() - t0 < budget_s * 0.75:
        tokens += smp.run_one()
    dt = time.perf_counter() - t0
    return {"value": tokens / dt, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
            "sample": smp.describe(name) + f"; {tokens} tokens in {dt:.1f} s"}


# ------------------------------------------------------------------ reference arm
def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    shapes = workload(args.workload)
    name = workload_name(args.workload, shapes)
    budget_total = 150.0
    smp = OracleSampler(shapes, budget_per_step=budget_total / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        smp.run_one()
    tokens, t0 = 0, time.perf_counter()
    for _ in range(args.steps):
        tokens += smp.run_one()
    dt = time.perf_counter() - t0
    value = tokens / dt
    cores = blas_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * dt / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(args.workload, shapes),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": smp.describe(name) + f"; {args.steps} steps"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_config(key, shapes):
    s = shapes[0]
    cfg = {"workload": workload_name(key, shapes), "T": s.T, "b": s.b, "k": s.k,
           "linears": [[x.n, x.m] for x in shapes],
           "cnp_blocks_per_step": sum(x.n // x.b + x.m // x.b for x in shapes)}
    return cfg


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


# ------------------------------------------------------------------ GPU helpers
def graph_of(fn, stream):
    """Captures fn(stream) into a CUDA graph (on the current device)."""
    import torch
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        fn(stream)
    return g


def time_graphs(graphs, reps, stream, flush=None):
    """Device time (ms) of `reps` back-to-back replays cycling over `graphs`.  With `flush`
    (a device buffer larger than L2) the buffer is overwritten before every replay and each
    replay is timed alone, so that no replay finds its data in L2."""
    import torch
    if flush is not None:
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(reps)]
        with torch.cuda.stream(stream):
            for i in range(reps):
                flush.fill_(i & 255)
                evs[i][0].record(stream)
                graphs[i % len(graphs)].replay()
                evs[i][1].record(stream)
        torch.cuda.synchronize()
        return sum(a.elapsed_time(b) for a, b in evs)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for i in range(reps):
            graphs[i % len(graphs)].replay()
        e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1)


def measure_fma_peak(P, dev):
    """FP32 FMA TFLOP/s of this device: the library's probe kernel, 2 CTAs of 512 threads
    per SM, best of 5 launches timed with events."""
    import torch
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    ctas, iters = 2 * sms, 20000
    out = torch.empty(ctas * 512, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    P.fma_probe(out, ctas, 200, stream)
    best = 0.0
    for _ in range(5):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        P.fma_probe(out, ctas, iters, stream)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        ms = e0.elapsed_time(e1)
        best = max(best, ctas * 512 * 16 * iters * 2 / (ms / 1e3) / 1e12)
    return best


class Workload:
    """Device state of one workload: the group of linears and its input sets."""

    def __init__(self, key, dev, int8=False, device_inputs=False, seed=0):
        import torch

        from orthogonal_reparameterized_cnp_b200 import poetx as P
        from poetx_inputs import layer_inputs
        self.key = key
        self.shapes = workload(key)
        s0 = self.shapes[0]
        self.T, self.b, self.k = s0.T, s0.b, s0.k
        self.bf16 = s0.dtype == "bf16"
        self.act = torch.bfloat16 if self.bf16 else torch.float32
        to = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a)).to(dev, dt)  # noqa: E731
        specs, xs, dys, self.host_inputs = [], [], [], []
        gen = torch.Generator(device=dev)
        for i, s in enumerate(self.shapes):
            pP, _ = P.make_perm((s.config_id << 32) | (s.linear_id << 8) | 0, s.n)
            pR, _ = P.make_perm((s.config_id << 32) | (s.linear_id << 8) | 1, s.m)
            if device_inputs:
                # seeded draws on the device at the workload's scales (timing-only runs)
                gen.manual_seed(seed * 1000 + i)
                rn = lambda shape, std, dt: (torch.randn(shape, generator=gen, device=dev)  # noqa: E731
                                             * std).to(dt)
                W0 = rn((s.m, s.n), 1.0 / np.sqrt(s.n), self.act)
                tP = rn((s.nblk_P, s.ntri), s.std_theta, torch.float32)
                tR = rn((s.nblk_R, s.ntri), s.std_theta, torch.float32)
                x = rn((s.T, s.n), 1.0, self.act)
                dy = rn((s.T, s.m), 1.0, self.act)
            else:
                inp = layer_inputs(s)
                W0, tP, tR = to(inp.W0, self.act), to(inp.theta_P, torch.float32), \
                    to(inp.theta_R, torch.float32)
                x, dy = to(inp.x, self.act), to(inp.dy, self.act)
            specs.append((W0, tP, tR, pP, pR))
            xs.append(x)
            dys.append(dy)
        self.group = P.PoetxLinearGroup(specs, self.b, self.k, self.T, int8_weight=int8)
        es = 2 if self.bf16 else 4
        in_bytes = sum(s.T * (s.n + s.m) * es for s in self.shapes)
        # inputs larger than L2 per step leave nothing useful in L2 for the next step; small
        # ones are evicted by writing a buffer of twice the L2 before every timed step
        self.nsets = 1
        self.flush = None
        if in_bytes <= 2 * L2_BYTES:
            self.flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)
        self.xs, self.dys = [xs], [dys]
        for r in range(1, self.nsets):
            self.xs.append([torch.roll(t, shifts=r, dims=0).contiguous() for t in xs])
            self.dys.append([torch.roll(t, shifts=r, dims=0).contiguous() for t in dys])
        self.ys = [torch.empty((s.T, s.m), dtype=self.act, device=dev) for s in self.shapes]
        self.dxs = [torch.empty((s.T, s.n), dtype=self.act, device=dev) for s in self.shapes]
        self.in_bytes = in_bytes
        self.nblk = self.group.cnp.nblk

    def step(self, i, stream):
        self.group.step(self.xs[i % self.nsets], self.dys[i % self.nsets], self.ys, self.dxs,
                        stream)

    def layer_only(self, i, stream):
        g = self.group
        xs, dys = self.xs[i % self.nsets], self.dys[i % self.nsets]
        g.forward(xs, self.ys, stream)
        g.backward(xs, dys, self.dxs, 0, stream)

    def l2_note(self):
        if self.flush is None:
            return (f"each step reads {self.in_bytes >> 20} MB of inputs and touches several "
                    f"times that (> 126 MB L2): no step finds its inputs in L2")
        return (f"inputs ({self.in_bytes >> 10} KB) fit in L2: L2 flushed before every timed "
                f"step by writing {self.flush.numel() >> 20} MB, each step timed alone")


def check_status(P, stream, where):
    if P.device_status(stream) != P.POETX_OK:
        raise RuntimeError(f"device status not OK after {where}")


def family_attribution(P, wl, stream, reps, families=None):
    """Per-family device time of one step from CUDA-graph replays: the step is captured
    once per family with CUDA events around that family's launches (event nodes of the
    graph), replayed `reps` times, and the bracketed times of each replay summed."""
    import torch
    out = {}
    for fam in families or FAMILIES:
        P.profile_begin(fam)
        g = graph_of(lambda st: wl.step(0, st), stream)
        P.profile_begin(None)
        tot, launches = 0.0, 0
        for i in range(reps):
            if wl.flush is not None:  # inputs that fit in L2: start every replay cold
                wl.flush.fill_(i & 255)
            g.replay()
            torch.cuda.synchronize()
            n, ms = P.profile_end()
            tot += ms
            launches = n
        out[fam] = {"launches_per_step": launches, "ms_per_step": tot / reps,
                    "avg_launch_ms": (tot / reps / launches) if launches else None}
        del g
    check_status(P, stream, "the attribution replays")
    return out


def single_cta(P, wl, stream, reps, families=("gemm_w0",)):
    """The merged-weight GEMMs of one step on single CTAs instead of CTA pairs, from
    CUDA-graph replays with events around each launch (for comparison)."""
    import torch
    out = {}
    prev = P.set_gemm_pairs(False)
    try:
        for fam in families:
            P.profile_begin(fam)
            g = graph_of(lambda st: wl.step(0, st), stream)
            P.profile_begin(None)
            tot, launches = 0.0, 0
            for i in range(reps):
                if wl.flush is not None:
                    wl.flush.fill_(i & 255)
                g.replay()
                torch.cuda.synchronize()
                n, ms = P.profile_end()
                tot += ms
                launches = n
            del g
            out[fam] = {"launches_per_step": launches, "ms_per_step": tot / reps}
    finally:
        P.set_gemm_pairs(prev)
    check_status(P, stream, "the single-CTA replays")
    return out


def cnp_only(P, wl, stream, reps):
    """CNP forward and backward alone (one call each over every block), CUDA-graph replay."""
    c = wl.group.cnp
    gf = graph_of(lambda st: c.forward(st), stream)
    gb = graph_of(lambda st: c.backward(st), stream)
    time_graphs([gf, gb], 2, stream)
    fms = time_graphs([gf], reps, stream, wl.flush) / reps
    bms = time_graphs([gb], reps, stream, wl.flush) / reps
    check_status(P, stream, "the CNP-only replays")
    cf, cb = cnp_flops_per_block(wl.b, wl.k)
    return {"blocks": c.nblk, "b": wl.b, "k": wl.k, "fwd_ms": fms, "bwd_ms": bms,
            "fwd_blocks_per_s": c.nblk / (fms / 1e3), "bwd_blocks_per_s": c.nblk / (bms / 1e3),
            "fwd_tflops": c.nblk * cf / (fms / 1e3) / 1e12,
            "bwd_tflops": c.nblk * cb / (bms / 1e3) / 1e12}


def cnp_sweep(P, dev, stream, fma_peak):
    """The CNP-only sweep: b in {64, 128, 256, 512}, k in {2, 4, 6}; block count = both
    sides of all 7 linears x 32 layers of Llama-8B shapes; seeded device inputs at the
    sweep's scales (theta ~ N(0, 0.01^2), dG ~ N(0, 1))."""
    import torch

    from orthogonal_reparameterized_cnp_b200 import poetx as P_
    from poetx_inputs import cnp_sweep_blocks
    res = []
    gen = torch.Generator(device=dev)
    for b in (64, 128, 256, 512):
        nblk = cnp_sweep_blocks(b)
        gen.manual_seed(b)
        c = P_.CnpBuffers(nblk, b, 2, dev)
        c.theta.copy_(torch.randn(c.theta.shape, generator=gen, device=dev) * 0.01)
        c.dG.copy_(torch.randn(c.dG.shape, generator=gen, device=dev))
        for k in (2, 4, 6):
            c.set_order(k)
            c.forward(stream)
            c.backward(stream)
            gf = graph_of(lambda st: c.forward(st), stream)
            gb = graph_of(lambda st: c.backward(st), stream)
            time_graphs([gf, gb], 1, stream)
            reps = 3
            fms = time_graphs([gf], reps, stream) / reps
            bms = time_graphs([gb], reps, stream) / reps
            cf, cb = cnp_flops_per_block(b, k)
            res.append({"b": b, "k": k, "blocks": nblk,
                        "fwd_blocks_per_s": nblk / (fms / 1e3),
                        "bwd_blocks_per_s": nblk / (bms / 1e3),
                        "fwd_frac_fma": nblk * cf / (fms / 1e3) / 1e12 / fma_peak,
                        "bwd_frac_fma": nblk * cb / (bms / 1e3) / 1e12 / fma_peak})
            del gf, gb
        del c
        torch.cuda.empty_cache()
    check_status(P, stream, "the CNP sweep")
    return res


def secondary_step(P, key, dev, stream, reps):
    """Step and layer-only throughput of a secondary workload, CUDA-graph replay, seeded
    device inputs (timing only; parity of these shapes is checked by the tests)."""
    import torch
    wl = Workload(key, dev, device_inputs=True, seed=7)
    for i in range(3):
        wl.step(i, stream)
    torch.cuda.synchronize()
    gs = [graph_of(lambda st, i=i: wl.step(i, st), stream) for i in range(wl.nsets)]
    gl = [graph_of(lambda st, i=i: wl.layer_only(i, st), stream) for i in range(wl.nsets)]
    time_graphs(gs, 3, stream)
    ms = time_graphs(gs, reps, stream, wl.flush) / reps
    lms = time_graphs(gl, reps, stream, wl.flush) / reps
    check_status(P, stream, f"the {key} replays")
    out = {"workload": workload_name(key, wl.shapes), "ms_per_step": ms,
           "tokens_per_s": wl.T / (ms / 1e3), "layer_only_tokens_per_s": wl.T / (lms / 1e3),
           "launch": "cuda_graph", "l2": wl.l2_note(), "steps": reps}
    del gs, gl, wl
    torch.cuda.empty_cache()
    return out


# ------------------------------------------------------------------ GPU arm
def run_poetx(args):
    import torch
    import torch.distributed as dist

    from orthogonal_reparameterized_cnp_b200 import dp
    from orthogonal_reparameterized_cnp_b200 import poetx as P

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
    stream = torch.cuda.Stream(dev)
    torch.cuda.set_stream(stream)
    fma_peak = measure_fma_peak(P, dev)

    wl = Workload(args.workload, dev)
    shapes = wl.shapes
    T = wl.T

    def exchange():  # the data-parallel step's one collective (a no-op on one rank)
        if world > 1:
            dp.allreduce_dtheta(wl.group.cnp.dtheta)

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local])

    # warm-up (eager), then the step captured once per input set
    for i in range(max(3, args.warmup)):
        wl.step(i, stream)
        exchange()
    torch.cuda.synchronize(dev)
    check_status(P, stream, "warm-up")
    graphs = None
    graph_launches = 0
    if args.graph:
        graphs = []
        for i in range(wl.nsets):
            n0 = P.launch_count()
            graphs.append(graph_of(lambda st, i=i: wl.step(i, st), stream))
            graph_launches = P.launch_count() - n0
        for i in range(3):
            with torch.cuda.stream(stream):
                graphs[i % wl.nsets].replay()
            exchange()
        torch.cuda.synchronize(dev)
        check_status(P, stream, "graph warm-up")

    # timed region
    props = torch.cuda.get_device_properties(dev)
    uuid = str(getattr(props, "uuid", "") or "")
    gpu_id = (uuid if uuid.startswith("GPU-") else f"GPU-{uuid}") if uuid else str(local)
    sampler = ClockSampler(gpu_id)
    barrier()
    torch.cuda.synchronize(dev)
    sampler.start()
    time.sleep(0.3)
    launches0 = P.launch_count()
    # one event pair around all steps; with an L2 flush between steps (inputs that fit in
    # L2), one pair per step with the flush outside it
    nev = args.steps if wl.flush is not None else 1
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(nev)]
    with torch.cuda.stream(stream):
        for i in range(args.steps):
            if wl.flush is not None:
                wl.flush.fill_(i & 255)
            if wl.flush is not None or i == 0:
                evs[min(i, nev - 1)][0].record(stream)
            if graphs:
                graphs[i % wl.nsets].replay()  # the layers' kernels; the collective outside
            else:
                wl.step(i, stream)
            exchange()
            if wl.flush is not None or i == args.steps - 1:
                evs[min(i, nev - 1)][1].record(stream)
    torch.cuda.synchronize(dev)
    launches = graph_launches * args.steps if graphs else P.launch_count() - launches0
    barrier()
    clocks = sampler.stop()
    elapsed_ms = sum(a.elapsed_time(b) for a, b in evs)
    max_ms = max_over_ranks(elapsed_ms, dist if world > 1 else None, dev)
    check_status(P, stream, "the timed region")
    ms_per_step = max_ms / args.steps
    value = job_tokens_per_s(world, T, args.steps, max_ms)

    reps = max(10, min(args.steps, 50))
    # layer-only figure: forward + backward of every linear without the CNP
    gl = [graph_of(lambda st, i=i: wl.layer_only(i, st), stream) for i in range(wl.nsets)]
    time_graphs(gl, 3, stream)
    lms = time_graphs(gl, reps, stream, wl.flush) / reps
    check_status(P, stream, "the layer-only replays")
    del gl
    cnp = cnp_only(P, wl, stream, reps)

    # per-family device time and the roofline of the dominant family
    work = family_work(shapes)
    breakdown = family_attribution(P, wl, stream, reps=min(reps, 20))
    if wl.bf16:
        fw = family_work(shapes)
        for fam, alt in single_cta(P, wl, stream, reps=min(reps, 20)).items():
            if "flops" in fw[fam]:
                alt["achieved_tflops"] = fw[fam]["flops"] / (alt["ms_per_step"] / 1e3) / 1e12
            if "bytes" in fw[fam]:
                alt["achieved_gbs"] = fw[fam]["bytes"] / (alt["ms_per_step"] / 1e3) / 1e9
            breakdown[fam + "_single_cta"] = alt
    dominant = max(FAMILIES, key=lambda f: breakdown[f]["ms_per_step"])
    peaks, peak_src = load_peaks()
    wkey = workload_name(args.workload, shapes)
    for fam in FAMILIES:
        bd = breakdown[fam]
        ww = work.get(fam)
        if ww and bd["ms_per_step"] > 0:
            if "flops" in ww:
                bd["achieved_tflops"] = ww["flops"] / (bd["ms_per_step"] / 1e3) / 1e12
            if "bytes" in ww:
                bd["achieved_gbs"] = ww["bytes"] / (bd["ms_per_step"] / 1e3) / 1e9
    roof = None
    w = work.get(dominant)
    bd = breakdown[dominant]
    if w is not None and bd["launches_per_step"]:
        per_launch_s = bd["avg_launch_ms"] / 1e3
        nl = bd["launches_per_step"]
        if w["bound"] == "tensor":
            achieved = w["flops"] / nl / per_launch_s / 1e12
            peak = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
            unit, psrc = "TFLOP/s", peak_src + ", bf16 burst"
        elif w["bound"] == "hbm":
            achieved = w["bytes"] / nl / per_launch_s / 1e9
            peak = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
            unit, psrc = "GB/s", peak_src
        else:
            achieved = w["flops"] / nl / per_launch_s / 1e12
            peak = fma_peak
            unit, psrc = "TFLOP/s", "measured: FP32 FMA probe kernel on this device"
        roof = {"kernel": dominant, "bound": w["bound"], "achieved": achieved, "peak": peak,
                "unit": unit, "frac": achieved / peak if peak else None,
                "traffic": committed_traffic(dominant, wkey),
                "peak_source": psrc, "avg_launch_ms": bd["avg_launch_ms"],
                "launches_per_step": nl,
                "timing": "CUDA events around each launch of the family, as event nodes of "
                          "the captured step graph, averaged over replays"}
        if w["bound"] == "tensor":
            sus = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
            roof["frac_of_sustained"] = achieved / sus

    # end to end through the public API with host buffers (pinned), copies timed: every
    # step uploads every linear's x and dy and theta and downloads the step's result,
    # dtheta (y and dx stay on the device, as for layers that feed other layers); the host
    # pipeline overlaps the uploads of the next step and the downloads of the previous one
    # with the step's kernels (two copy engines)
    e2e = None
    if args.e2e_steps > 0:
        from orthogonal_reparameterized_cnp_b200.host_pipeline import HostPipeline
        g = wl.group
        hx = [t.cpu().pin_memory() for t in wl.xs[0]]
        hdy = [t.cpu().pin_memory() for t in wl.dys[0]]
        hth = g.cnp.theta.cpu().pin_memory()
        hy = hdx = None  # the step's result is dtheta
        hdth = torch.empty(g.cnp.dtheta.shape, dtype=torch.float32).pin_memory()
        pipe = HostPipeline(g, nbuf=2, exchange=exchange if world > 1 else None)
        for i in range(3):
            pipe.submit(i, hx, hdy, hth, hy, hdx, hdth)
        pipe.synchronize()
        barrier()
        torch.cuda.synchronize(dev)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(pipe.h2d)  # every step's first operation (its upload) follows this
        for i in range(args.e2e_steps):
            pipe.submit(i, hx, hdy, hth, hy, hdx, hdth)
        e1.record(pipe.d2h)  # the last download is the last operation of the last step
        pipe.synchronize()
        torch.cuda.synchronize(dev)
        e_ms = max_over_ranks(e0.elapsed_time(e1), dist if world > 1 else None, dev)
        nbytes = lambda ts: sum(t.numel() * t.element_size() for t in ts)  # noqa: E731
        h2d = nbytes(hx) + nbytes(hdy) + hth.numel() * 4
        d2h = hdth.numel() * 4
        e2e = {"value": job_tokens_per_s(world, T, args.e2e_steps, e_ms), "unit": "tokens/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "steps": args.e2e_steps, "copies": "overlapped with compute (2 buffer sets)",
               "downloaded": "dtheta (the step's result); y and dx stay on the device"}
        check_status(P, stream, "the end-to-end steps")
        del pipe, hx, hdy

    # the merge of the permutations into W0' (S1: once per set of permutations, every
    # linear of the workload), and the outer-loop merge of the first linear (once per
    # inner loop); device time per call
    merge = None
    gm = graph_of(lambda st: wl.group.merge(st), stream)
    time_graphs([gm], 2, stream)
    mms = time_graphs([gm], 10, stream, wl.flush) / 10
    mbytes = sum(2.0 * s.m * s.n * (2 if wl.bf16 else 4) for s in shapes)
    merge = {"ms": mms, "achieved_gbs": mbytes / (mms / 1e3) / 1e9}
    del gm
    outer = None
    if wl.bf16:
        L0 = wl.group.layers[0]
        s = shapes[0]
        pP2, _ = P.make_perm(12345 + 1000003, s.n)
        pR2, _ = P.make_perm(12346 + 1000003, s.m)
        i32 = lambda a: torch.as_tensor(np.asarray(a, dtype=np.int32), device=dev)  # noqa: E731
        pP2d, pR2d = i32(pP2), i32(pR2)
        W0p_new = torch.empty_like(L0.W0p)
        mws = torch.empty(P.outer_merge_workspace(s.m, s.n, P.POETX_BF16), dtype=torch.uint8,
                          device=dev)
        GP, GR = L0.G_ops()
        go = graph_of(lambda st: P.outer_merge(L0.W0p, GP, GR, s.b, L0.inv_P, L0.inv_R, pP2d,
                                               pR2d, W0p_new, mws, st), stream)
        time_graphs([go], 2, stream)
        oms = time_graphs([go], 10, stream, wl.flush) / 10
        mb = 2 * s.m * s.n * 2 + (s.n + s.m) * s.b * 2
        outer = {"linear": [s.n, s.m], "ms": oms, "achieved_gbs": mb / (oms / 1e3) / 1e9,
                 "achieved_tflops": 4.0 * s.m * s.n * s.b / (oms / 1e3) / 1e12}
        check_status(P, stream, "the outer merge")
        del go, W0p_new, mws

    # the same step with the int8 merged weight (POET-XQ reading), CUDA-graph replay
    xq = None
    if wl.bf16 and args.graph:
        wq = Workload(args.workload, dev, int8=True, device_inputs=True, seed=3)
        for i in range(3):
            wq.step(i, stream)
        torch.cuda.synchronize(dev)
        gq = [graph_of(lambda st, i=i: wq.step(i, st), stream) for i in range(wq.nsets)]
        time_graphs(gq, 3, stream)
        qms = time_graphs(gq, reps, stream, wq.flush) / reps
        check_status(P, stream, "the int8-weight steps")
        qfam = family_attribution(P, wq, stream, min(reps, 20), families=("gemm_w0",))
        xq = {"ms_per_step": qms, "tokens_per_s": T / (qms / 1e3), "steps": reps,
              "weight": "int8 W0' (per-row scales), converted to bf16 in shared memory "
                        "inside the W0' GEMMs",
              "gemm_w0_ms_per_step": qfam["gemm_w0"]["ms_per_step"]}
        del gq, wq
        torch.cuda.empty_cache()

    also = None
    if args.also and args.workload == "llama13b-block" and world == 1:
        also = {}
        del graphs
        graphs = None
        torch.cuda.empty_cache()
        for key in ("llama8b-up", "fp32-small"):
            try:
                also[key] = secondary_step(P, key, dev, stream,
                                           reps=20 if key == "llama8b-up" else 200)
            except Exception as exc:  # reported in the line; the headline stands on its own
                also[key] = {"error": f"{type(exc).__name__}: {exc}"}
        if "ms_per_step" in also.get("fp32-small", {}):
            also["fp32-small"]["latency_us"] = 1e3 * also["fp32-small"]["ms_per_step"]
        try:
            also["cnp_sweep"] = cnp_sweep(P, dev, stream, fma_peak)
        except Exception as exc:
            also["cnp_sweep"] = {"error": f"{type(exc).__name__}: {exc}"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = oracle_throughput(wkey, shapes, args.oracle_budget)

    cfg = workload_config(args.workload, shapes)
    cfg.update({
        "l2": wl.l2_note(), "parallelism": f"dp{world}" if world > 1 else "single",
        "launch": "cuda_graph" if args.graph else "eager",
        "step": "CNP forward (one call, every block) + every linear's forward + every "
                "linear's backward + CNP backward (one call); the merge of the "
                "permutations is once per set of permutations, reported under 'merge'"})
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if wl.bf16 else "f32", "data": "synthetic",
        "config": cfg,
        "clocks": clocks,
        "e2e": e2e,
        "gpu_launches": int(launches),
        "roofline": roof,
        "cpu_baseline": cpu,
        "layer_only": {"tokens_per_s": world * T / (lms / 1e3), "ms_per_step": lms,
                       "what": "every linear's forward + backward, no CNP (CUDA graph)"},
        "cnp": cnp,
        "fma_peak_tflops": fma_peak,
        "kernels": breakdown,
        "merge": merge,
        "outer_merge": outer,
        "int8_weight_step": xq,
        "also": also,
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
