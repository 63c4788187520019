"""GPU parity of the int8 base weight (POET-XQ reading): codes and scales bit-exact with
the oracle's fp32 decision, and the bf16 layer run on the int8 merged weight against the
float64 oracle layer on the dequantised weight (normalised max error <= 2e-2)."""
import numpy as np
import pytest

from oracle import poetx_ref as ref
from poetx_inputs import LayerShape, layer_inputs, round_to_bf16

from .gpu_harness import host, norm_max_err, tensor

pytestmark = pytest.mark.gpu

BF16_NORM = 2e-2


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from orthogonal_reparameterized_cnp_b200 import poetx as P
    P.lib()  # fails loudly if the library is missing
    yield


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("m,n", [(1, 16), (300, 520), (64, 2048), (7, 33)])
def test_quantize_rows_bit_exact(dtype, m, n):
    import torch
    from orthogonal_reparameterized_cnp_b200 import poetx as P
    rng = np.random.default_rng(m * 31 + n)
    W = rng.standard_normal((m, n)) * rng.uniform(1e-3, 5.0, (m, 1))
    if m > 3:
        W[3] = 0.0
    W = round_to_bf16(W) if dtype == "bf16" else W.astype(np.float32).astype(np.float64)
    Wd = tensor(W, torch.bfloat16 if dtype == "bf16" else torch.float32)
    q = torch.empty((m, n), dtype=torch.int8, device="cuda")
    s = torch.empty((m,), dtype=torch.float32, device="cuda")
    P.quantize_rows(Wd, q, s)
    torch.cuda.synchronize()
    q_ref, s_ref = ref.quantize_rows_int8(W)
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(s.cpu().numpy(), s_ref)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("m,n", [(1, 16), (300, 520), (13824, 5120), (77, 13824), (5, 33)])
def test_merge_perm_q8_bit_exact(dtype, m, n):
    """Codes and scales of the merged weight straight from W0 equal the oracle's quantiser
    applied to the oracle's merged weight W0[p_R][:, p_P] (zero rows included)."""
    import torch
    from orthogonal_reparameterized_cnp_b200 import poetx as P
    rng = np.random.default_rng(m * 7 + n)
    W = rng.standard_normal((m, n)) * rng.uniform(1e-3, 5.0, (m, 1))
    W[min(2, m - 1)] = 0.0
    W = round_to_bf16(W) if dtype == "bf16" else W.astype(np.float32).astype(np.float64)
    Wd = tensor(W, torch.bfloat16 if dtype == "bf16" else torch.float32)
    pR, _ = P.make_perm(m + 1, m)
    pP, _ = P.make_perm(n + 2, n)
    q = torch.empty((m, n), dtype=torch.int8, device="cuda")
    s = torch.empty((m,), dtype=torch.float32, device="cuda")
    P.merge_perm_q8(Wd, q, s, tensor(pR, torch.int32), tensor(pP, torch.int32))
    torch.cuda.synchronize()
    oR, _ = ref.make_perm(m + 1, m)
    oP, _ = ref.make_perm(n + 2, n)
    q_ref, s_ref = ref.quantize_rows_int8(ref.merge_perm(W, oR, oP))
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(s.cpu().numpy(), s_ref)


@pytest.mark.parametrize("T,n,m,pairs", [(300, 512, 384, True), (600, 1024, 2048, True),
                                         (1000, 2048, 1024, True), (600, 1024, 2048, False)])
def test_int8_layer_equals_bf16_layer_on_the_dequantised_weight(T, n, m, pairs):
    """The int8 entry points give exactly what the bf16 entry points give on bf16(s * q) as a
    whole weight: the CTA-pair kernel converting int8 tiles in shared memory (both operand
    layouts, ragged token counts), and the panel-by-panel form that other shapes take (m =
    384 forward, and every GEMM with pairs switched off: several panels per GEMM)."""
    import torch
    from orthogonal_reparameterized_cnp_b200 import poetx as P
    prev = P.set_gemm_pairs(pairs)
    try:
        _int8_equals_bf16(T, n, m)
    finally:
        P.set_gemm_pairs(prev)


def _int8_equals_bf16(T, n, m):
    import torch
    from orthogonal_reparameterized_cnp_b200 import poetx as P
    b = 256 if n % 256 == 0 and m % 256 == 0 else 128
    s = LayerShape(f"xqeq-{n}x{m}", T=T, n=n, m=m, b=b, k=4, dtype="bf16", config_id=12,
                   std_theta=0.01)
    inp = layer_inputs(s)
    pP, _ = P.make_perm(inp.seed_P, n)
    pR, _ = P.make_perm(inp.seed_R, m)
    L = P.PoetxLinear(tensor(inp.W0, torch.bfloat16), tensor(inp.theta_P, torch.float32),
                      tensor(inp.theta_R, torch.float32), pP, pR, b, 4, T, int8_weight=True)
    x = tensor(inp.x, torch.bfloat16)
    dy = tensor(inp.dy, torch.bfloat16)
    L.cnp_forward()
    y8 = torch.empty((T, m), dtype=torch.bfloat16, device="cuda")
    dx8 = torch.empty((T, n), dtype=torch.bfloat16, device="cuda")
    L.forward(x, y8)
    L.backward(x, dy, dx8)
    dG8 = L.dG.clone()
    # the same layer on the dequantised weight through the bf16 entry points
    Wdq = (L.scales[:, None] * L.W0q.float()).to(torch.bfloat16).contiguous()
    GP, GR = L.G_ops()
    ws = torch.empty(max(P.linear_fwd_workspace(L.desc), P.linear_bwd_workspace(L.desc)),
                     dtype=torch.uint8, device="cuda")
    y = torch.empty_like(y8)
    dx = torch.empty_like(dx8)
    U = torch.empty_like(L.U)
    Ws = torch.empty_like(L.Wsave)
    dG_P = torch.empty_like(L.dG[: L.nP])
    dG_R = torch.empty_like(L.dG[L.nP:])
    P.linear_fwd(L.desc, x, GP, GR, Wdq, y, U, Ws, ws)
    P.linear_bwd(L.desc, x, dy, GP, GR, Wdq, U, Ws, dx, dG_P, dG_R, 0, ws)
    torch.cuda.synchronize()
    assert P.device_status() == P.POETX_OK
    assert torch.equal(y8, y)
    assert torch.equal(dx8, dx)
    assert torch.equal(dG8[: L.nP], dG_P) and torch.equal(dG8[L.nP:], dG_R)


@pytest.mark.parametrize("T,n,m,b", [(256, 512, 384, 128), (320, 512, 768, 256)])
def test_int8_layer_matches_oracle(T, n, m, b):
    import torch
    from orthogonal_reparameterized_cnp_b200 import poetx as P
    s = LayerShape(f"xq-{n}x{m}-b{b}", T=T, n=n, m=m, b=b, k=4, dtype="bf16", config_id=11,
                   std_theta=0.01)
    inp = layer_inputs(s)
    dev = torch.device("cuda")
    pP, _ = P.make_perm(inp.seed_P, n)
    pR, _ = P.make_perm(inp.seed_R, m)
    layer = P.PoetxLinear(tensor(inp.W0, torch.bfloat16), tensor(inp.theta_P, torch.float32),
                          tensor(inp.theta_R, torch.float32), pP, pR, b, 4, T, int8_weight=True)
    x = tensor(inp.x, torch.bfloat16)
    dy = tensor(inp.dy, torch.bfloat16)
    y = torch.empty((T, m), dtype=torch.bfloat16, device=dev)
    dx = torch.empty((T, n), dtype=torch.bfloat16, device=dev)
    layer.step(x, dy, y, dx)
    torch.cuda.synchronize()
    assert P.device_status() == P.POETX_OK
    # oracle: its own permutations, merge, quantisation and CNP; layer on s * q
    oP, _ = ref.make_perm(inp.seed_P, n)
    oR, _ = ref.make_perm(inp.seed_R, m)
    W0p = ref.merge_perm(inp.W0, oR, oP)
    q, sc = ref.quantize_rows_int8(W0p)
    assert np.array_equal(layer.W0q.cpu().numpy(), q) and np.array_equal(layer.scales.cpu().numpy(), sc)
    Wdq = ref.dequantize_rows(q, sc)
    G_P, G_R = ref.cnp_forward(inp.theta_P, b, 4), ref.cnp_forward(inp.theta_R, b, 4)
    x64, dy64 = inp.x.astype(np.float64), inp.dy.astype(np.float64)
    Y, U, V, W = ref.layer_forward(x64, Wdq, G_P, G_R, oP, oR)
    dX, dG_P, dG_R = ref.layer_backward(x64, dy64, Wdq, G_P, G_R, oP, oR, U=U, W=W)
    dth = np.concatenate([ref.cnp_backward(inp.theta_P, dG_P, b, 4),
                          ref.cnp_backward(inp.theta_R, dG_R, b, 4)])
    errs = {"y": norm_max_err(host(y), Y), "dx": norm_max_err(host(dx), dX),
            "dG_P": norm_max_err(host(layer.dG[: n // b]), dG_P),
            "dG_R": norm_max_err(host(layer.dG[n // b:]), dG_R),
            "dtheta": norm_max_err(host(layer.dtheta), dth)}
    assert all(v <= BF16_NORM for v in errs.values()), errs
