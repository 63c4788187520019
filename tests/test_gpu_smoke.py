"""The entry point's smoke check (one small bf16 and one small fp32 layer step through the
library, compared with the oracle) runs as part of the GPU suite."""
import pytest


@pytest.mark.gpu
def test_smoke_entry_point():
    import __graft_entry__ as entry
    entry.smoke()
