"""GPU parity: libpoetx (through its C ABI) against the float64 oracle on the same seeded
inputs.

Bars: permutations / index maps / merged weight bit-exact; CNP fp32 max-abs <= 1e-5 on G
and dtheta; fp32 layer normalised max error <= 1e-5; bf16 layer outputs and gradients
normalised max error <= 2e-2 (normalised = max|gpu - ref| / max|ref| per tensor).
"""
import numpy as np
import pytest

from oracle import poetx_ref as ref
from poetx_inputs import (LayerShape, cnp_inputs, cnp_sweep_blocks, layer_inputs,
                          workload_llama13b_block, workload_llama1b_attn, workload_llama8b_up,
                          workload_small_fp32)

from .gpu_harness import host, norm_max_err, run_group, run_layer, tensor

pytestmark = pytest.mark.gpu

CNP_ABS = 1e-5
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


def _P():
    from orthogonal_reparameterized_cnp_b200 import poetx as P
    return P


# ------------------------------------------------------------------ index maps
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("rows,cols", [(1, 8), (7, 24), (300, 2048), (9, 2056), (3, 2560),
                                       (6, 2568), (17, 3072), (11, 4096), (33, 14336),
                                       (5, 13824)])
def test_permute_cols_bit_exact(dtype, rows, cols):
    import torch
    P = _P()
    tdt = torch.float32 if dtype == "f32" else torch.bfloat16
    rng = np.random.default_rng(rows * 7 + cols)
    a = rng.standard_normal((rows, cols)).astype(np.float32)
    perm, inv = P.make_perm(rows * 1000 + cols, cols)
    x = tensor(a, tdt)
    out = torch.empty_like(x)
    back = torch.empty_like(x)
    P.permute_cols(x, out, tensor(perm, torch.int32))
    P.permute_cols(out, back, tensor(inv, torch.int32))
    torch.cuda.synchronize()
    xs = x.cpu()
    assert torch.equal(out.cpu(), xs[:, torch.from_numpy(perm.astype(np.int64))])
    assert torch.equal(back.cpu(), xs)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("m,n", [(12, 8), (2048, 2048), (14336, 4096)])
def test_merge_perm_bit_exact(dtype, m, n):
    import torch
    P = _P()
    tdt = torch.float32 if dtype == "f32" else torch.bfloat16
    W0 = tensor(np.random.default_rng(m + n).standard_normal((m, n)).astype(np.float32), tdt)
    pR, _ = P.make_perm(11 + m, m)
    pP, _ = P.make_perm(13 + n, n)
    W0p = torch.empty_like(W0)
    P.merge_perm(W0, W0p, tensor(pR, torch.int32), tensor(pP, torch.int32))
    torch.cuda.synchronize()
    expect = ref.merge_perm(W0.cpu().float().numpy(), pR.astype(np.int64), pP.astype(np.int64))
    assert np.array_equal(W0p.cpu().float().numpy(), expect)


# ------------------------------------------------------------------ CNP
def _cnp_gpu(theta, dG, b, k, with_bf16=False, ws_blocks=None):
    import torch
    P = _P()
    nblk = theta.shape[0]
    th = tensor(theta, torch.float32)
    G = torch.empty((nblk, b, b), dtype=torch.float32, device="cuda")
    Gb = torch.empty((nblk, b, b), dtype=torch.bfloat16, device="cuda") if with_bf16 else None
    ws_bytes = P.cnp_workspace(nblk if ws_blocks is None else ws_blocks, b, k)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device="cuda")
    P.cnp_fwd(th, G, Gb, b, k, ws)
    dth = None
    if dG is not None:
        dth_t = torch.empty_like(th)
        P.cnp_bwd(th, tensor(dG, torch.float32), dth_t, b, k, ws)
        dth = dth_t
    torch.cuda.synchronize()
    assert P.device_status() == P.POETX_OK
    return G, Gb, dth


@pytest.mark.parametrize("b,k", [(2, 1), (2, 4), (3, 2), (5, 3), (8, 4), (17, 5), (32, 4),
                                 (64, 2), (64, 6), (100, 4), (128, 4), (256, 4), (256, 7),
                                 (512, 4), (1024, 2)])
def test_cnp_matches_oracle(b, k):
    nblk = 3 if b <= 256 else 2
    rng = np.random.default_rng(b * 31 + k)
    theta = (rng.standard_normal((nblk, b * (b - 1) // 2)) * 0.01).astype(np.float32)
    dG = rng.standard_normal((nblk, b, b)).astype(np.float32)
    G, Gb, dth = _cnp_gpu(theta, dG, b, k, with_bf16=True)
    G_ref = ref.cnp_forward(theta, b, k)
    assert np.abs(host(G) - G_ref).max() <= CNP_ABS
    dth_ref = ref.cnp_backward(theta, dG, b, k)
    assert np.abs(host(dth) - dth_ref).max() <= CNP_ABS
    # the bf16 copy is the round-to-nearest-even of the fp32 G
    import torch
    assert torch.equal(Gb.cpu(), G.cpu().to(torch.bfloat16))


@pytest.mark.parametrize("b,k,nblk", [(64, 6, 3), (100, 4, 3), (256, 4, 3), (128, 1, 3),
                                      (256, 4, 200), (128, 6, 700)])
def test_cnp_saved_pair_is_bit_identical(b, k, nblk):
    # the forward keeps Q, S = Q^2 and F'; the backward that reads them must give exactly
    # the dtheta of the recomputing backward (task graph: b % 64 == 0; b = 100 takes the
    # per-step path; 200 blocks of 256 and 700 of 128 take the 128 x 128 product items),
    # and S must be Q^2
    import torch
    P = _P()
    rng = np.random.default_rng(b * 7 + k)
    theta = (rng.standard_normal((nblk, b * (b - 1) // 2)) * 0.01).astype(np.float32)
    dG = rng.standard_normal((nblk, b, b)).astype(np.float32)
    G, _, dth = _cnp_gpu(theta, dG, b, k)
    th = tensor(theta, torch.float32)
    G2 = torch.empty_like(G)
    Qs = torch.empty_like(G)
    S = torch.empty_like(G)
    F = torch.empty_like(G)
    dth2 = torch.empty_like(th)
    ws = torch.empty(max(P.cnp_workspace(nblk, b, k), 16), dtype=torch.uint8, device="cuda")
    P.cnp_fwd_save(th, G2, None, Qs, S, F, b, k, ws)
    P.cnp_bwd_saved(th, tensor(dG, torch.float32), Qs, S, F, dth2, b, k, ws)
    torch.cuda.synchronize()
    assert P.device_status() == P.POETX_OK
    assert torch.equal(G2, G)
    assert torch.equal(dth2, dth)
    sel = [0, nblk // 2, nblk - 1]
    Q = np.stack([ref.theta_to_Q(t, b) for t in theta[sel].astype(np.float64)])
    # the packing, bit-exact (fp32 theta is exact in fp64)
    assert np.array_equal(host(Qs[sel]), Q)
    assert np.abs(host(S[sel]) - Q @ Q).max() <= CNP_ABS
    # G and dtheta of those blocks against the oracle
    assert np.abs(host(G[sel]) - ref.cnp_forward(theta[sel], b, k)).max() <= CNP_ABS
    assert np.abs(host(dth[sel]) - ref.cnp_backward(theta[sel], dG[sel], b, k)).max() <= CNP_ABS


def test_cnp_zero_theta_is_exact_identity():
    import torch
    for b in [4, 64, 256]:
        theta = np.zeros((3, b * (b - 1) // 2), dtype=np.float32)
        G, Gb, _ = _cnp_gpu(theta, None, b, 4, with_bf16=True)
        eye = torch.eye(b).expand(3, b, b)
        assert torch.equal(G.cpu(), eye)
        assert torch.equal(Gb.cpu(), eye.to(torch.bfloat16))


def test_cnp_small_workspace_chunks_blocks():
    # one block's worth of scratch forces a chunk per block; results must not change
    b, k, nblk = 64, 4, 5
    rng = np.random.default_rng(5)
    theta = (rng.standard_normal((nblk, b * (b - 1) // 2)) * 0.01).astype(np.float32)
    dG = rng.standard_normal((nblk, b, b)).astype(np.float32)
    G1, _, d1 = _cnp_gpu(theta, dG, b, k)
    G2, _, d2 = _cnp_gpu(theta, dG, b, k, ws_blocks=1)
    import torch
    assert torch.equal(G1.cpu(), G2.cpu()) and torch.equal(d1.cpu(), d2.cpu())


@pytest.mark.parametrize("b", [64, 128, 256, 512])
@pytest.mark.parametrize("k", [2, 4, 6])
def test_cnp_sweep_sampled(b, k):
    """CNP sweep: all 7 linears x 32 layers of Llama-8B shapes on both sides (full block
    count); the oracle checks the first, the last and randomly chosen blocks."""
    nblk = cnp_sweep_blocks(b)
    theta, dG = cnp_inputs(4, b * 10 + k, nblk, b)
    G, _, dth = _cnp_gpu(theta, dG, b, k)
    nsamp = {64: 24, 128: 12, 256: 6, 512: 3}[b]
    rng = np.random.default_rng(b + k)
    idx = sorted({0, nblk - 1, *rng.choice(nblk, nsamp, replace=False).tolist()})
    G_h = G[idx].cpu().double().numpy()
    d_h = dth[idx].cpu().double().numpy()
    G_ref = ref.cnp_forward(theta[idx], b, k)
    d_ref = ref.cnp_backward(theta[idx], dG[idx], b, k)
    assert np.abs(G_h - G_ref).max() <= CNP_ABS
    assert np.abs(d_h - d_ref).max() <= CNP_ABS


# ------------------------------------------------------------------ layer, fp32
def _check_full(out, s, inp, tol):
    W0p = ref.merge_perm(inp.W0, out["perm_R"].astype(np.int64), out["perm_P"].astype(np.int64))
    assert np.array_equal(out["W0p"], W0p)
    o = ref.full_step(inp.x, inp.W0, inp.theta_P, inp.theta_R, inp.dy,
                      out["perm_P"].astype(np.int64), out["perm_R"].astype(np.int64), s.b, s.k)
    errs = {key: norm_max_err(out[key], o[key])
            for key in ["y", "dx", "dG_P", "dG_R", "dtheta_P", "dtheta_R"]}
    bad = {kk: v for kk, v in errs.items() if not v <= tol}
    assert not bad, f"normalised max errors above {tol}: {errs}"
    G_ref = np.concatenate([o["G_P"], o["G_R"]])
    assert np.abs(out["G"] - G_ref).max() <= CNP_ABS
    return errs


def test_layer_fp32_small_config():
    s = workload_small_fp32()
    inp = layer_inputs(s)
    out = run_layer(inp)
    _check_full(out, s, inp, F32_NORM)


@pytest.mark.parametrize("n,m,b,k,T", [(8, 12, 2, 1, 5), (12, 8, 4, 3, 3), (16, 24, 8, 4, 70),
                                       (96, 64, 32, 2, 129), (256, 128, 64, 4, 1)])
def test_layer_fp32_small_shapes(n, m, b, k, T):
    s = LayerShape(f"fp32-{n}x{m}", T=T, n=n, m=m, b=b, k=k, dtype="f32", config_id=100 + b,
                   std_theta=0.05)
    inp = layer_inputs(s)
    out = run_layer(inp)
    _check_full(out, s, inp, F32_NORM)


# ------------------------------------------------------------------ layer, bf16
@pytest.mark.parametrize("n,m,b,T", [(256, 256, 128, 300), (512, 256, 256, 129), (256, 768, 128, 1),
                                     (1024, 512, 512, 200), (384, 640, 128, 513)])
def test_layer_bf16_small_shapes(n, m, b, T):
    s = LayerShape(f"bf16-{n}x{m}", T=T, n=n, m=m, b=b, k=4, dtype="bf16", config_id=200 + b)
    inp = layer_inputs(s)
    out = run_layer(inp)
    _check_full(out, s, inp, BF16_NORM)


def test_layer_bf16_llama1b_full():
    """n = m = 2048, b = 256, k = 4, T = 8192: every output against the full oracle."""
    s = workload_llama1b_attn()
    inp = layer_inputs(s)
    out = run_layer(inp)
    _check_full(out, s, inp, BF16_NORM)


@pytest.mark.parametrize("n,m,T", [(1024, 1024, 1000), (512, 1536, 300), (1536, 512, 257)])
def test_gemm_pairs_and_single_ctas_agree_with_the_oracle(n, m, T):
    """The merged-weight GEMMs on CTA pairs (256 x 256 tiles over two SMs) and on single CTAs
    both meet the bar against the oracle, with ragged token counts (M tails)."""
    P = _P()
    s = LayerShape(f"pairs-{n}x{m}", T=T, n=n, m=m, b=256, k=4, dtype="bf16", config_id=500)
    inp = layer_inputs(s)
    outs = {}
    prev = P.set_gemm_pairs(True)
    try:
        for pairs in (True, False):
            P.set_gemm_pairs(pairs)
            out = run_layer(inp)
            out.pop("layer")
            outs[pairs] = out
            _check_full(out, s, inp, BF16_NORM)
    finally:
        P.set_gemm_pairs(prev)
    for key in ["y", "dx", "dG_P", "dG_R"]:
        assert norm_max_err(outs[True][key], outs[False][key]) <= 1e-2, key


def test_recompute_mode_matches_saved_mode():
    s = LayerShape("bf16-recompute", T=777, n=512, m=768, b=256, k=4, dtype="bf16", config_id=300)
    inp = layer_inputs(s)
    a = run_layer(inp, save=True)
    b_ = run_layer(inp, save=False)
    for key in ["y", "dx", "dG_P", "dG_R", "dtheta_P", "dtheta_R"]:
        assert np.array_equal(a[key], b_[key]), key


def test_runs_are_deterministic():
    s = LayerShape("bf16-det", T=1000, n=512, m=512, b=128, k=4, dtype="bf16", config_id=301)
    inp = layer_inputs(s)
    a = run_layer(inp)
    b_ = run_layer(inp)
    for key in ["y", "dx", "dG_P", "dG_R", "dtheta_P", "dtheta_R"]:
        assert np.array_equal(a[key], b_[key]), key


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_micro_batch_accumulation(dtype):
    import torch
    P = _P()
    b = 128 if dtype == "bf16" else 16
    s = LayerShape("acc", T=400, n=256, m=384, b=b, k=4, dtype=dtype, config_id=302)
    inp = layer_inputs(s)
    full = run_layer(inp)
    layer = full["layer"]
    act = layer.W0.dtype
    x = tensor(inp.x, act)
    dy = tensor(inp.dy, act)
    y = torch.empty((s.T, s.m), dtype=act, device="cuda")
    dx = torch.empty((s.T, s.n), dtype=act, device="cuda")
    # split the tokens into two micro-batches sharing the same layer buffers
    halves = [(0, 150), (150, 400)]
    dG_sum = None
    for i, (t0, t1) in enumerate(halves):
        sub = P.PoetxLinear(layer.W0, layer.theta[: layer.nP], layer.theta[layer.nP:],
                            full["perm_P"], full["perm_R"], s.b, s.k, t1 - t0)
        sub.merge()
        sub.cnp_forward()
        sub.forward(x[t0:t1].contiguous(), y[t0:t1])
        if dG_sum is not None:
            sub.dG.copy_(dG_sum)
        sub.backward(x[t0:t1].contiguous(), dy[t0:t1].contiguous(), dx[t0:t1], accumulate=int(i > 0))
        dG_sum = sub.dG.clone()
    torch.cuda.synchronize()
    tol = 1e-6 if dtype == "f32" else 1e-5
    assert np.abs(host(dG_sum) - host(layer.dG)).max() <= tol * max(1.0, np.abs(host(layer.dG)).max())


def test_empty_token_set():
    import torch
    P = _P()
    s = LayerShape("empty", T=0, n=256, m=256, b=128, k=4, dtype="bf16", config_id=303)
    W0 = tensor(np.zeros((256, 256), np.float32), torch.bfloat16)
    th = torch.zeros((2, 128 * 127 // 2), dtype=torch.float32, device="cuda")
    pP, _ = P.make_perm(1, 256)
    pR, _ = P.make_perm(2, 256)
    layer = P.PoetxLinear(W0, th, th, pP, pR, 128, 4, 0)
    layer.merge()
    layer.cnp_forward()
    x = torch.empty((0, 256), dtype=torch.bfloat16, device="cuda")
    y = torch.empty((0, 256), dtype=torch.bfloat16, device="cuda")
    layer.forward(x, y)
    layer.dG.fill_(7.0)
    layer.backward(x, y, x)
    torch.cuda.synchronize()
    assert torch.count_nonzero(layer.dG).item() == 0


# ------------------------------------------------------------------ full size, every element
def _full_checks(out, s, inp, tol=BF16_NORM):
    """Every output element of one linear against the full float64 oracle: y, dX, and every
    block of dG_P, dG_R, dtheta_P, dtheta_R (normalised per tensor and per block), G to
    CNP_ABS, and W0' bit-exact."""
    pP = out["perm_P"].astype(np.int64)
    pR = out["perm_R"].astype(np.int64)
    o = ref.full_step(inp.x, inp.W0, inp.theta_P, inp.theta_R, inp.dy, pP, pR, s.b, s.k)
    assert np.array_equal(out["W0p"], o["W0p"])
    assert np.abs(out["G"] - np.concatenate([o["G_P"], o["G_R"]])).max() <= CNP_ABS
    errs = {key: norm_max_err(out[key], o[key])
            for key in ["y", "dx", "dG_P", "dG_R", "dtheta_P", "dtheta_R"]}
    bad = {kk: v for kk, v in errs.items() if not v <= tol}
    assert not bad, f"{s.name}: normalised max errors above {tol}: {errs}"
    worst = {}
    for key in ["dG_P", "dG_R", "dtheta_P", "dtheta_R"]:
        per_block = [norm_max_err(out[key][j], o[key][j]) for j in range(len(o[key]))]
        worst[key] = max(per_block)
        assert worst[key] <= tol, f"{s.name}: {key} block {int(np.argmax(per_block))}: " \
                                  f"{worst[key]:.3e} > {tol}"
    return errs, worst


@pytest.mark.slow
def test_layer_bf16_llama8b_up_full():
    """n = 4096 -> m = 14336, b = 256, T = 16384: every element of y and dX and every one of
    the 16 + 56 blocks of dG and dtheta against the full float64 oracle."""
    s = workload_llama8b_up()
    inp = layer_inputs(s)
    out = run_layer(inp)
    out.pop("layer")
    _full_checks(out, s, inp)


@pytest.mark.slow
def test_layer_bf16_llama13b_block_full():
    """The 7 linears of the 13B decoder block as one group (one CNP call over all 382
    blocks, as the bench runs it): every element of every linear's y and dX and every
    block of its dG and dtheta against the full float64 oracle."""
    shapes = workload_llama13b_block()
    inps = [layer_inputs(s) for s in shapes]
    outs, g = run_group(inps)
    del g
    for s, inp, out in zip(shapes, inps, outs):
        _full_checks(out, s, inp)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_group_matches_separate_layers_bit_for_bit(dtype):
    """One CNP call over the blocks of several linears and a shared layer scratch give
    exactly what separate layers (each with its own CNP call and scratch) give."""
    b = 128 if dtype == "bf16" else 32
    shapes = [LayerShape(f"grp{i}", T=300, n=n, m=m, b=b, k=4, dtype=dtype, config_id=400,
                         linear_id=i)
              for i, (n, m) in enumerate([(256, 256), (256, 512), (512, 256)])]
    inps = [layer_inputs(s) for s in shapes]
    outs, g = run_group(inps)
    for inp, o in zip(inps, outs):
        r = run_layer(inp)
        for key in ["W0p", "G", "y", "dx", "dG_P", "dG_R", "dtheta_P", "dtheta_R"]:
            assert np.array_equal(o[key], r[key]), key
