"""GPU parity of the outer-loop merge (W <- R W0 P, then the merged weight under new
permutations) against the float64 oracle, through the C ABI.

Each side builds its own permutations and its own G from the same seeded theta (the GPU
through its CNP forward, the oracle through its own), so no expected value depends on the
CUDA path.  Bars: bf16 normalised max error <= 2e-2, fp32 <= 1e-5; theta = 0 bit-exact.
"""
import numpy as np
import pytest

from oracle import poetx_ref as ref
from poetx_inputs import round_to_bf16

from .gpu_harness import host, norm_max_err, tensor

pytestmark = pytest.mark.gpu

F32_NORM = 1e-5
BF16_NORM = 2e-2


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from orthogonal_reparameterized_cnp_b200 import poetx as P
    P.lib()  # fails loudly if the library is missing
    yield


def _inputs(m, n, b, dtype, seed, theta_scale):
    rng = np.random.default_rng(seed)
    W0 = rng.standard_normal((m, n)) / np.sqrt(n)
    W0 = round_to_bf16(W0) if dtype == "bf16" else W0.astype(np.float32).astype(np.float64)
    tP = (rng.standard_normal((n // b, b * (b - 1) // 2)) * theta_scale).astype(np.float32)
    tR = (rng.standard_normal((m // b, b * (b - 1) // 2)) * theta_scale).astype(np.float32)
    seeds = [seed * 8 + i for i in range(4)]  # old P, old R, new P, new R
    return W0, tP, tR, seeds


def _gpu_merge(W0, tP, tR, seeds, m, n, b, k, dtype):
    import torch
    from orthogonal_reparameterized_cnp_b200 import poetx as P
    act = torch.bfloat16 if dtype == "bf16" else torch.float32
    pP, iP = P.make_perm(seeds[0], n)
    pR, iR = P.make_perm(seeds[1], m)
    pP2, _ = P.make_perm(seeds[2], n)
    pR2, _ = P.make_perm(seeds[3], m)
    i32 = lambda a: tensor(a, torch.int32)
    W0d = tensor(W0, act)
    W0p = torch.empty_like(W0d)
    P.merge_perm(W0d, W0p, i32(pR), i32(pP))
    Gs = []
    for th, nb in [(tP, n // b), (tR, m // b)]:
        thd = tensor(th, torch.float32)
        G = torch.empty((nb, b, b), dtype=torch.float32, device="cuda")
        Gb = torch.empty((nb, b, b), dtype=torch.bfloat16, device="cuda")
        ws = torch.empty(P.cnp_workspace(nb, b, k), dtype=torch.uint8, device="cuda")
        P.cnp_fwd(thd, G, Gb, b, k, ws)
        Gs.append(Gb if dtype == "bf16" else G)
    out = torch.empty_like(W0p)
    ws = torch.empty(P.outer_merge_workspace(m, n, P.POETX_BF16 if dtype == "bf16" else P.POETX_F32),
                     dtype=torch.uint8, device="cuda")
    P.outer_merge(W0p, Gs[0], Gs[1], b, i32(iP), i32(iR), i32(pP2), i32(pR2), out, ws)
    torch.cuda.synchronize()
    assert P.device_status() == 0
    return host(out)


def _oracle_merge(W0, tP, tR, seeds, m, n, b, k):
    pP, _ = ref.make_perm(seeds[0], n)
    pR, _ = ref.make_perm(seeds[1], m)
    pP2, _ = ref.make_perm(seeds[2], n)
    pR2, _ = ref.make_perm(seeds[3], m)
    GP, GR = ref.cnp_forward(tP, b, k), ref.cnp_forward(tR, b, k)
    return ref.outer_merge(W0, GP, GR, pP, pR, pP2, pR2)[1], (pP2, pR2)


@pytest.mark.parametrize("m,n,b,k,dtype", [(512, 384, 128, 4, "bf16"), (2048, 2048, 256, 4, "bf16"),
                                           (1024, 512, 512, 2, "bf16"), (96, 64, 32, 4, "f32"),
                                           (256, 192, 64, 3, "f32")])
def test_outer_merge_matches_oracle(m, n, b, k, dtype):
    W0, tP, tR, seeds = _inputs(m, n, b, dtype, m + n + b, 0.01)
    got = _gpu_merge(W0, tP, tR, seeds, m, n, b, k, dtype)
    want, _ = _oracle_merge(W0, tP, tR, seeds, m, n, b, k)
    err = norm_max_err(got, want)
    assert err <= (BF16_NORM if dtype == "bf16" else F32_NORM), err


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_outer_merge_at_zero_theta_is_bit_exact(dtype):
    # G = I exactly (also in bf16), so the products are exact and the result is the
    # plain gather of W0 under the new permutations
    m, n, b, k = 512, 256, 128, 4
    W0, tP, tR, seeds = _inputs(m, n, b, dtype, 77, 0.0)
    got = _gpu_merge(W0, tP, tR, seeds, m, n, b, k, dtype)
    _, (pP2, pR2) = _oracle_merge(W0, tP, tR, seeds, m, n, b, k)
    assert np.array_equal(got, W0[np.ix_(pR2, pP2)])
