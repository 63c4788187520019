"""The case runner behind the ncu summaries (kernel_cases) runs every case cleanly on small
shapes, so the profiling commands stay valid."""
import pytest

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("argv", [["gemm", "512", "512", "512", "0"],
                                  ["gemm", "512", "512", "512", "1"],
                                  ["layer", "300", "512", "768", "0"],
                                  ["layer32"],
                                  ["cnp", "5", "64", "4"],
                                  ["cnp", "5", "256", "4"],
                                  ["q8merge", "256", "512"]])
def test_kernel_case_runs(argv, capsys):
    from orthogonal_reparameterized_cnp_b200 import kernel_cases
    assert kernel_cases.main(argv) == 0
    out = capsys.readouterr().out
    assert argv[0] in out or "ok" in out


def test_kernel_cases_usage():
    from orthogonal_reparameterized_cnp_b200 import kernel_cases
    assert kernel_cases.main([]) == 2
