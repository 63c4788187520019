"""The bench's algorithmic work per step (what roofline.achieved divides by time) against
the formulas stated for each kernel family, on the bench workload (no GPU)."""
import pytest


def test_family_work_of_the_bench_workload():
    import bench
    s = bench.workload("llama1b-attn")
    assert (s.T, s.n, s.m, s.b, s.k) == (8192, 2048, 2048, 256, 4)
    w = bench.family_work(s)
    T, n, m, b = s.T, s.n, s.m, s.b
    nblk = n // b + m // b
    # two W0' GEMMs of 2 T n m FLOPs each
    assert w["gemm_w0"]["flops"] == pytest.approx(2 * 2.0 * T * n * m)
    # four block-diagonal products: each reads and writes its bf16 activation, plus G
    assert w["gemm_blockdiag"]["bytes"] == pytest.approx(2.0 * 2 * T * (2 * n + 2 * m)
                                                         + 2.0 * 2 * nblk * b * b)
    # CNP per block with k = 4 (d = 2): forward 3 b^3 (half products by symmetry),
    # backward with Q, S, F' kept 2 b^3 (D) + 2 b^3 (Pm) + 4 b^3 (A)
    assert w["cnp_sgemm"]["flops"] == pytest.approx(nblk * (3 + 8) * b ** 3)
    assert w["cnp_sgemm"]["bound"] == "alu"
    assert w["gemm_w0"]["bound"] == "tensor"
    assert w["permute"]["bound"] == "hbm"


def test_derived_fma_peak():
    import bench
    peak = bench.SM_COUNT * bench.FP32_LANES_PER_SM * 2 * bench.SM_MAX_MHZ * 1e6 / 1e12
    assert peak == pytest.approx(74.44992)
