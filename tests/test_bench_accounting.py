"""The bench's algorithmic work per step (what roofline.achieved divides by time) against
the formulas stated for each kernel family, on the bench workloads (no GPU)."""
import pytest


def test_default_workload_is_the_13b_block():
    import bench
    a = bench.parse_args([])
    assert a.workload == "llama13b-block"
    shapes = bench.workload(a.workload)
    assert [(s.n, s.m) for s in shapes] == [(5120, 5120)] * 4 + [(5120, 13824)] * 2 + \
        [(13824, 5120)]
    assert {(s.T, s.b, s.k, s.dtype) for s in shapes} == {(8192, 256, 4, "bf16")}
    cfg = bench.workload_config(a.workload, shapes)
    assert cfg["cnp_blocks_per_step"] == 382


def test_family_work_of_the_single_layer_workload():
    import bench
    shapes = bench.workload("llama1b-attn")
    s = shapes[0]
    assert (s.T, s.n, s.m, s.b, s.k) == (8192, 2048, 2048, 256, 4)
    w = bench.family_work(shapes)
    T, n, m, b = s.T, s.n, s.m, s.b
    nblk = n // b + m // b
    # two W0' GEMMs of 2 T n m FLOPs each
    assert w["gemm_w0"]["flops"] == pytest.approx(2 * 2.0 * T * n * m)
    # four block-diagonal products: each reads and writes its bf16 activation, plus G
    assert w["gemm_blockdiag"]["bytes"] == pytest.approx(2.0 * 2 * T * (2 * n + 2 * m)
                                                         + 2.0 * 2 * nblk * b * b)
    # four activation gathers / scatters (x, y, dy, dx), one read and one write each
    assert w["permute"]["bytes"] == pytest.approx(2.0 * 2 * (2 * T * n + 2 * T * m))
    # CNP per block with k = 4 (d = 2): forward 3 b^3 (half products by symmetry),
    # backward with Q, S, F' kept 2 b^3 (D) + 2 b^3 (Pm) + 4 b^3 (A)
    assert w["cnp_sgemm"]["flops"] == pytest.approx(nblk * (3 + 8) * b ** 3)
    assert w["cnp_sgemm"]["bound"] == "alu"
    assert w["gemm_w0"]["bound"] == "tensor"
    assert w["permute"]["bound"] == "hbm"


def test_family_work_sums_over_the_linears():
    import bench
    shapes = bench.workload("llama13b-block")
    w = bench.family_work(shapes)
    T = 8192
    assert w["gemm_w0"]["flops"] == pytest.approx(sum(4.0 * T * s.n * s.m for s in shapes))
    assert w["gemm_w0"]["launches"] == 14 and w["permute"]["launches"] == 28
    assert w["cnp_sgemm"]["flops"] == pytest.approx(382 * 11 * 256 ** 3)


@pytest.mark.parametrize("k,fwd,bwd", [(1, 2, 6), (2, 2, 6), (4, 3, 8), (6, 4, 13)])
def test_cnp_flops_per_block(k, fwd, bwd):
    # d = floor((k+1)/2): forward (d + 1) half products; backward D (2) + Horner terms
    # (d = 2: N_2 S, 2; d = 3: N_3 S, S N_3, S R_1 full and T_1 S half, 7) + A (4)
    import bench
    f, b_ = bench.cnp_flops_per_block(64, k)
    assert (f, b_) == (fwd * 64 ** 3, bwd * 64 ** 3)


def test_committed_traffic_is_tied_to_the_kernel_source(tmp_path, monkeypatch):
    import bench
    sha = bench.source_sha(bench.FAMILY_SOURCES["gemm_w0"])
    # a change in any source of the family makes the row stale
    assert sha != bench.source_sha(bench.FAMILY_SOURCES["gemm_w0"][:1])
    f = tmp_path / "t.md"
    f.write_text(f"| gemm_w0 | wl-a | 1.5e9 | {sha} | note |\n"
                 f"| gemm_w0 | wl-b | 2.0e9 | {'0' * 16} | stale |\n")
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(f))
    assert bench.committed_traffic("gemm_w0", "wl-a") == pytest.approx(1.5e9)
    assert bench.committed_traffic("gemm_w0", "wl-b") is None   # the kernel changed since
    assert bench.committed_traffic("cnp_elementwise", "wl-a") is None
