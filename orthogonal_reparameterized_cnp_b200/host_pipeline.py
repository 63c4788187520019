"""Steps of a PoetxLinear fed from, and drained to, host (pinned) memory with the copies
overlapped with the GPU work.

A training loop that holds its batches in host memory pays, every step, one upload of
x, dy and theta and one download of y, dx and dtheta.  Done in line they add the PCIe
time of both directions to the kernels' time.  Here three CUDA streams run them
concurrently: the upload of step i+1 (copy engine, host -> device), the step i kernels,
and the download of step i-1 (the other copy engine, device -> host).  Each of `nbuf`
device buffer sets cycles through upload -> compute -> download; events order the three
streams so that a set is refilled only after its results have left the device.
Every step still makes its full upload and download.
"""
from __future__ import annotations


class HostPipeline:
    """Runs ``layer.step`` on host tensors with copies and compute overlapped.

    submit(i, ...) enqueues step i (nothing blocks on the host); synchronize() waits for
    every submitted step.  The host tensors must be pinned and must stay untouched until
    synchronize() (or until the step's results have been waited for).
    """

    def __init__(self, layer, nbuf: int = 2, exchange=None):
        """exchange: optional callable run on the compute stream after each step, before
        dtheta is copied out (the data-parallel all-reduce of dtheta)."""
        import torch
        dev = layer.W0.device
        act = layer.W0.dtype
        self.layer = layer
        self.nbuf = nbuf
        self.exchange = exchange
        self.h2d = torch.cuda.Stream(dev)
        self.comp = torch.cuda.Stream(dev)
        self.d2h = torch.cuda.Stream(dev)
        T, n, m = layer.T, layer.n, layer.m
        mk = lambda shape, dt: [torch.empty(shape, dtype=dt, device=dev) for _ in range(nbuf)]  # noqa: E731
        self.x, self.dy = mk((T, n), act), mk((T, m), act)
        self.y, self.dx = mk((T, m), act), mk((T, n), act)
        self.theta = mk(tuple(layer.theta.shape), torch.float32)
        self.dtheta = mk(tuple(layer.dtheta.shape), torch.float32)
        ev = lambda: [torch.cuda.Event() for _ in range(nbuf)]  # noqa: E731
        self.in_ready, self.computed, self.out_done = ev(), ev(), ev()
        self.used = [False] * nbuf

    def submit(self, i: int, hx, hdy, htheta, hy, hdx, hdtheta) -> None:
        import torch
        s = i % self.nbuf
        L = self.layer
        with torch.cuda.stream(self.h2d):
            if self.used[s]:
                self.h2d.wait_event(self.computed[s])  # the set's inputs are consumed
            self.x[s].copy_(hx, non_blocking=True)
            self.dy[s].copy_(hdy, non_blocking=True)
            self.theta[s].copy_(htheta, non_blocking=True)
            self.in_ready[s].record(self.h2d)
        with torch.cuda.stream(self.comp):
            self.comp.wait_event(self.in_ready[s])
            if self.used[s]:
                self.comp.wait_event(self.out_done[s])  # the set's results have left
            L.theta.copy_(self.theta[s])
            L.step(self.x[s], self.dy[s], self.y[s], self.dx[s], self.comp)
            if self.exchange is not None:
                self.exchange()
            self.dtheta[s].copy_(L.dtheta)
            self.computed[s].record(self.comp)
        with torch.cuda.stream(self.d2h):
            self.d2h.wait_event(self.computed[s])
            hy.copy_(self.y[s], non_blocking=True)
            hdx.copy_(self.dx[s], non_blocking=True)
            hdtheta.copy_(self.dtheta[s], non_blocking=True)
            self.out_done[s].record(self.d2h)
        self.used[s] = True

    def synchronize(self) -> None:
        for st in (self.h2d, self.comp, self.d2h):
            st.synchronize()
