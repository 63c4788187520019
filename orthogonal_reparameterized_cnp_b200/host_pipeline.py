"""Steps of a PoetxLinear (or a PoetxLinearGroup) fed from, and drained to, host (pinned)
memory with the copies overlapped with the GPU work.

A training loop that holds its batches in host memory pays, every step, one upload of
x, dy and theta and one download of y, dx and dtheta.  Done in line they add the PCIe
time of both directions to the kernels' time.  Here three CUDA streams run them
concurrently: the upload of step i+1 (copy engine, host -> device), the step i kernels,
and the download of step i-1 (the other copy engine, device -> host).  Each of `nbuf`
device buffer sets cycles through upload -> compute -> download; events order the three
streams so that a set is refilled only after its results have left the device.
Every step still makes its full upload and its download of dtheta.  The downloads of y
and dx may be left out (pass None): a training loop whose next layers run on the device
needs only the step's result, dtheta, on the host.
"""
from __future__ import annotations


def _as_list(t):
    return list(t) if isinstance(t, (list, tuple)) else [t]


class HostPipeline:
    """Runs ``model.step`` on host tensors with copies and compute overlapped.

    ``model`` is a PoetxLinear (host tensors passed as single tensors) or a
    PoetxLinearGroup (host tensors passed as lists, one per linear).  submit(i, ...)
    enqueues step i (nothing blocks on the host); synchronize() waits for every submitted
    step.  The host tensors must be pinned and must stay untouched until synchronize() (or
    until the step's results have been waited for).
    """

    def __init__(self, model, nbuf: int = 2, exchange=None):
        """exchange: optional callable run on the compute stream after each step, before
        dtheta is copied out (the data-parallel all-reduce of dtheta)."""
        import torch
        self.group = hasattr(model, "layers")
        layers = model.layers if self.group else [model]
        dev = layers[0].W0.device
        act = layers[0].W0.dtype
        self.model = model
        self.nbuf = nbuf
        self.exchange = exchange
        self.theta_dev = model.cnp.theta if self.group else model.theta
        self.dtheta_dev = model.cnp.dtheta if self.group else model.dtheta
        self.h2d = torch.cuda.Stream(dev)
        self.comp = torch.cuda.Stream(dev)
        self.d2h = torch.cuda.Stream(dev)

        def mk(shapes, dt):
            return [[torch.empty(sh, dtype=dt, device=dev) for sh in shapes] for _ in range(nbuf)]

        self.x = mk([(L.T, L.n) for L in layers], act)
        self.dy = mk([(L.T, L.m) for L in layers], act)
        self.y = mk([(L.T, L.m) for L in layers], act)
        self.dx = mk([(L.T, L.n) for L in layers], act)
        self.theta = [torch.empty_like(self.theta_dev) for _ in range(nbuf)]
        self.dtheta = [torch.empty_like(self.dtheta_dev) for _ in range(nbuf)]
        ev = lambda: [torch.cuda.Event() for _ in range(nbuf)]  # noqa: E731
        self.in_ready, self.computed, self.out_done = ev(), ev(), ev()
        self.used = [False] * nbuf

    def submit(self, i: int, hx, hdy, htheta, hy, hdx, hdtheta) -> None:
        """hy, hdx: host outputs, or None to keep y and dx on the device only."""
        import torch
        s = i % self.nbuf
        hx, hdy = _as_list(hx), _as_list(hdy)
        hy = _as_list(hy) if hy is not None else []
        hdx = _as_list(hdx) if hdx is not None else []
        with torch.cuda.stream(self.h2d):
            if self.used[s]:
                self.h2d.wait_event(self.computed[s])  # the set's inputs are consumed
            for d, h in zip(self.x[s], hx):
                d.copy_(h, non_blocking=True)
            for d, h in zip(self.dy[s], hdy):
                d.copy_(h, non_blocking=True)
            self.theta[s].copy_(htheta, non_blocking=True)
            self.in_ready[s].record(self.h2d)
        with torch.cuda.stream(self.comp):
            self.comp.wait_event(self.in_ready[s])
            if self.used[s]:
                self.comp.wait_event(self.out_done[s])  # the set's results have left
            self.theta_dev.copy_(self.theta[s])
            if self.group:
                self.model.step(self.x[s], self.dy[s], self.y[s], self.dx[s], self.comp)
            else:
                self.model.step(self.x[s][0], self.dy[s][0], self.y[s][0], self.dx[s][0],
                                self.comp)
            if self.exchange is not None:
                self.exchange()
            self.dtheta[s].copy_(self.dtheta_dev)
            self.computed[s].record(self.comp)
        with torch.cuda.stream(self.d2h):
            self.d2h.wait_event(self.computed[s])
            for h, d in zip(hy, self.y[s]):
                h.copy_(d, non_blocking=True)
            for h, d in zip(hdx, self.dx[s]):
                h.copy_(d, non_blocking=True)
            hdtheta.copy_(self.dtheta[s], non_blocking=True)
            self.out_done[s].record(self.d2h)
        self.used[s] = True

    def synchronize(self) -> None:
        for st in (self.h2d, self.comp, self.d2h):
            st.synchronize()
