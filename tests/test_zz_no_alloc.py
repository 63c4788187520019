"""poetx_cnp_fwd_static: the Cayley-Neumann forward for callers that cannot allocate
device memory (their device memory belongs to a host framework's pool they cannot reach
from the call site, or the call sits in a loop where cudaMalloc would synchronise the
device).  Its scratch is a fixed array of the library's own device memory instead of a
caller buffer.  Checked through the C ABI against poetx_cnp_fwd on two calls in a row.

This file is collected last on purpose (the name sorts after the others).
"""
import ctypes

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

CNP_ABS = 1e-5  # the CNP parity bar used by the other GPU tests


@pytest.fixture(scope="module")
def P():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from orthogonal_reparameterized_cnp_b200 import poetx
    poetx.lib()
    return poetx


def _buffered(P, theta, nblk, b, k):
    import torch
    G = torch.empty((nblk, b, b), dtype=torch.float32, device="cuda")
    Gb = torch.empty((nblk, b, b), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(max(P.cnp_workspace(nblk, b, k), 16), dtype=torch.uint8, device="cuda")
    P.cnp_fwd(theta, G, Gb, b, k, ws)
    return G, Gb


def test_static_scratch_forward_matches_buffered_forward(P):
    import torch
    lib = P.lib()
    stream = torch.cuda.current_stream().cuda_stream
    # first call: 40 blocks of 256 need two passes through the 32 MiB array;
    # second call: other sizes, reusing the array the first call left behind
    for nblk, b, k, seed in [(40, 256, 4, 1), (7, 64, 6, 2)]:
        rng = np.random.default_rng(seed)
        theta = torch.from_numpy(
            (rng.standard_normal((nblk, b * (b - 1) // 2)) * 0.01).astype(np.float32)).cuda()
        G_ref, Gb_ref = _buffered(P, theta, nblk, b, k)
        G = torch.full((nblk, b, b), float("nan"), dtype=torch.float32, device="cuda")
        Gb = torch.zeros((nblk, b, b), dtype=torch.bfloat16, device="cuda")
        st = lib.poetx_cnp_fwd_static(theta.data_ptr(), G.data_ptr(), Gb.data_ptr(), nblk, b, k,
                                      stream)
        assert st == P.POETX_OK, lib.poetx_last_error()
        torch.cuda.synchronize()
        assert P.device_status() == P.POETX_OK
        assert (G - G_ref).abs().max().item() <= CNP_ABS
        assert (Gb.float() - Gb_ref.float()).abs().max().item() <= 2 ** -7


def test_static_scratch_rejects_blocks_above_its_size(P):
    lib = P.lib()
    fake = ctypes.c_void_p(0x10000)
    assert lib.poetx_cnp_fwd_static(fake, fake, None, 1, 1024, 4, None) == P.POETX_ERR_WORKSPACE
    assert b"fixed" in lib.poetx_last_error()
