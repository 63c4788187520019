"""poetx_cnp_fwd_static: the Cayley-Neumann forward for callers that cannot allocate
device memory (their device memory belongs to a host framework's pool they cannot reach
from the call site, or the call sits in a loop where cudaMalloc would synchronise the
device).  Its scratch is a fixed array of the library's own device memory instead of a
caller buffer.  Checked through the C ABI on two calls in a row: bit for bit against
poetx_cnp_fwd (the same kernels on the same chunks of blocks) and against the float64
oracle within the CNP bar.

This file is collected last on purpose (the name sorts after the others).
"""
import ctypes

import numpy as np
import pytest

from oracle import poetx_ref as ref

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
    # second call: other sizes, reusing the array the first call left behind;
    # third call: b = 1024, one block per pass (its forward scratch is 16 MiB + counters)
    for nblk, b, k, seed in [(40, 256, 4, 1), (7, 64, 6, 2), (2, 1024, 4, 3)]:
        rng = np.random.default_rng(seed)
        th_np = (rng.standard_normal((nblk, b * (b - 1) // 2)) * 0.01).astype(np.float32)
        theta = torch.from_numpy(th_np).cuda()
        G_ref, Gb_ref = _buffered(P, theta, nblk, b, k)
        G = torch.full((nblk, b, b), float("nan"), dtype=torch.float32, device="cuda")
        Gb = torch.zeros((nblk, b, b), dtype=torch.bfloat16, device="cuda")
        st = lib.poetx_cnp_fwd_static(theta.data_ptr(), G.data_ptr(), Gb.data_ptr(), nblk, b, k,
                                      stream)
        assert st == P.POETX_OK, lib.poetx_last_error()
        torch.cuda.synchronize()
        assert P.device_status() == P.POETX_OK
        assert torch.equal(G, G_ref)
        assert torch.equal(Gb, Gb_ref)
        # the oracle on the first and the last block
        for j in (0, nblk - 1):
            G_o = ref.cnp_forward(th_np[j:j + 1], b, k)[0]
            assert np.abs(G[j].double().cpu().numpy() - G_o).max() <= CNP_ABS


def test_static_scratch_rejects_blocks_above_its_size(P):
    # Only shapes the host check rejects are passed here: the placeholder pointers must never
    # reach a launch.  b = 1024: a forward block needs d + 2 matrices of 4 MiB (d = (k+1)//2);
    # k = 16 (10 matrices) and k = 11 (8 matrices, plus the counters) exceed the 32 MiB array.
    lib = P.lib()
    fake = ctypes.c_void_p(0x10000)
    for k in (16, 11):
        assert lib.poetx_cnp_fwd_static(fake, fake, None, 1, 1024, k, None) == \
            P.POETX_ERR_WORKSPACE
        assert b"fixed" in lib.poetx_last_error()
