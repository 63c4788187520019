"""Single kernel families on named cases, for profiler captures (ncu) and quick timing.

    python -m orthogonal_reparameterized_cnp_b200.kernel_cases <case> [args]

Cases (all on cuda:0, seeded random inputs, a few GB of device memory at most):

    gemm T N K int8    one PoetxLinear (n = K, m = N, b = 256, k = 4), bf16 or int8 merged
                       weight: forward + backward 3 times, then 10 forwards and 10 backwards
                       timed per W0' GEMM launch (family gemm_w0)
    layer T n m int8   one PoetxLinear, forward + backward 5 times (every layer kernel)
    layer32            the small fp32 linear: n = m = 256, b = 32, k = 4, T = 512, 5 steps
    cnp nblk b k       CnpBuffers: forward + backward 4 times, the last timed
    q8merge m n        merge_perm_q8 of an m x n bf16 weight, 4 times

Every case ends by checking the library's device status.  Kernel order per step, for
ncu's --launch-skip: see the docstring of each function.
"""
import sys

import torch

from . import poetx as P


def _dev():
    return torch.device("cuda", 0)


def _linear(T, n, m, int8, dtype=torch.bfloat16, b=256, std=0.01):
    dev = _dev()
    W0 = (torch.randn(m, n, device=dev) / n ** 0.5).to(dtype)
    tP = torch.randn(n // b, b * (b - 1) // 2, device=dev) * std
    tR = torch.randn(m // b, b * (b - 1) // 2, device=dev) * std
    pP, _ = P.make_perm(1, n)
    pR, _ = P.make_perm(2, m)
    L = P.PoetxLinear(W0, tP, tR, pP, pR, b, 4, T, int8_weight=bool(int8))
    x = torch.randn(T, n, device=dev).to(dtype)
    dy = torch.randn(T, m, device=dev).to(dtype)
    y = torch.empty(T, m, device=dev, dtype=dtype)
    dx = torch.empty(T, n, device=dev, dtype=dtype)
    L.cnp_forward()
    return L, x, dy, y, dx


def _check():
    torch.cuda.synchronize()
    if P.device_status() != P.POETX_OK:
        raise RuntimeError("device status not OK")


def gemm(T, N, K, int8):
    """Per step: the forward's W0' GEMM (B K-major), then the backward's (B MN-major); the
    3 warm-up steps are 6 `k_umma_gemm_pair` launches, then 10 forward ones, 10 backward."""
    L, x, dy, y, dx = _linear(T, K, N, int8)
    for _ in range(3):
        L.forward(x, y)
        L.backward(x, dy, dx)
    _check()
    flops = 2.0 * T * N * K
    out = []
    for name, fn in (("fwd", lambda: L.forward(x, y)), ("bwd", lambda: L.backward(x, dy, dx))):
        P.profile_begin("gemm_w0")
        for _ in range(10):
            fn()
        torch.cuda.synchronize()
        n, ms = P.profile_end()
        out.append(f"{name} {ms / n:.4f} ms ({flops / (ms / n / 1e3) / 1e12:.0f} TFLOP/s)")
    _check()
    print(f"gemm T={T} N={N} K={K} int8={int8}: " + ", ".join(out))


def layer(T, n, m, int8):
    """Per step (b = 256): forward = gather x, block product (G_P), W0' GEMM, block product
    (G_R), scatter y; backward = gather dy, block product, dG, reduce, W0' GEMM, block
    product, dG, reduce, scatter dx."""
    L, x, dy, y, dx = _linear(T, n, m, int8)
    for _ in range(5):
        L.forward(x, y)
        L.backward(x, dy, dx)
    _check()
    print("layer ok")


def layer32():
    L, x, dy, y, dx = _linear(512, 256, 256, 0, dtype=torch.float32, b=32, std=0.02)
    for _ in range(5):
        L.step(x, dy, y, dx)
    _check()
    print("layer32 ok")


def cnp(nblk, b, k):
    """Per call: k_zero_ints then k_cnp_graph (forward, then backward); for b = 32 or 64 one
    k_cnp_fused_fwd / k_cnp_fused_bwd launch per call instead."""
    dev = _dev()
    c = P.CnpBuffers(nblk, b, k, dev, torch.bfloat16)
    c.theta.copy_(torch.randn(c.theta.shape, device=dev) * 0.01)
    c.dG.copy_(torch.randn(c.dG.shape, device=dev))
    for _ in range(3):
        c.forward()
        c.backward()
    _check()
    e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    e[0].record()
    c.forward()
    e[1].record()
    c.backward()
    e[2].record()
    _check()
    print(f"cnp nblk={nblk} b={b} k={k}: fwd {e[0].elapsed_time(e[1]):.3f} ms "
          f"bwd {e[1].elapsed_time(e[2]):.3f} ms")


def q8merge(m, n):
    dev = _dev()
    W0 = (torch.randn(m, n, device=dev) / n ** 0.5).to(torch.bfloat16)
    q = torch.empty(m, n, dtype=torch.int8, device=dev)
    s = torch.empty(m, device=dev)
    pP, _ = P.make_perm(1, n)
    pR, _ = P.make_perm(2, m)
    pPd, pRd = torch.from_numpy(pP).to(dev), torch.from_numpy(pR).to(dev)
    for _ in range(4):
        P.merge_perm_q8(W0, q, s, pRd, pPd)
    _check()
    print("q8merge ok")


CASES = {"gemm": gemm, "layer": layer, "layer32": layer32, "cnp": cnp, "q8merge": q8merge}


def main(argv=None):
    argv = sys.argv[1:] if argv is None else argv
    if not argv or argv[0] not in CASES:
        print(__doc__)
        return 2
    torch.manual_seed(0)
    CASES[argv[0]](*[int(a) for a in argv[1:]])
    return 0


if __name__ == "__main__":
    sys.exit(main())
