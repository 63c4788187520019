"""The bounded waits give up without a fault: the CNP task graph is launched with a
dependency that can never be met (poetx_selftest_wait_timeout), under a short wait limit.
The launch must return, poetx_device_status must report POETX_ERR_TIMEOUT once (and clear
it), and the next normal calls must be correct.  Nothing here faults, traps or waits
without a bound."""
import time

import numpy as np
import pytest

from oracle import poetx_ref as ref

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def P():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from orthogonal_reparameterized_cnp_b200 import poetx
    poetx.lib()
    return poetx


@pytest.mark.parametrize("nblk,b,k", [(3, 64, 4), (20, 128, 6)])
def test_unreachable_dependency_times_out_and_the_library_recovers(P, nblk, b, k):
    import torch
    rng = np.random.default_rng(nblk + b)
    th_np = (rng.standard_normal((nblk, b * (b - 1) // 2)) * 0.01).astype(np.float32)
    theta = torch.from_numpy(th_np).cuda()
    G = torch.empty((nblk, b, b), dtype=torch.float32, device="cuda")
    ws = torch.empty(P.cnp_workspace(nblk, b, k), dtype=torch.uint8, device="cuda")
    assert P.device_status() == P.POETX_OK
    prev = P.set_wait_limit(50_000_000)  # 50 ms
    try:
        t0 = time.perf_counter()
        P.selftest_wait_timeout(theta, G, b, k, ws)
        st = P.device_status()           # synchronises the stream: the launch has returned
        dt = time.perf_counter() - t0
    finally:
        P.set_wait_limit(prev)
    assert st == P.POETX_ERR_TIMEOUT
    assert dt < 10.0                      # the wait gave up long before any outer limit
    assert P.device_status() == P.POETX_OK  # the flag was cleared
    # a normal forward and backward afterwards are correct
    dG_np = rng.standard_normal((nblk, b, b)).astype(np.float32)
    P.cnp_fwd(theta, G, None, b, k, ws)
    dth = torch.empty_like(theta)
    P.cnp_bwd(theta, torch.from_numpy(dG_np).cuda(), dth, b, k, ws)
    torch.cuda.synchronize()
    assert P.device_status() == P.POETX_OK
    assert np.abs(G.double().cpu().numpy() - ref.cnp_forward(th_np, b, k)).max() <= 1e-5
    assert np.abs(dth.double().cpu().numpy() - ref.cnp_backward(th_np, dG_np, b, k)).max() <= 1e-5
