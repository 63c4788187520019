"""Pins of the float64 oracle against things other than itself (no GPU).

Each test names the mistake it is meant to catch.  Sources: the POET abstract (W = R W0 P,
spectrum preservation) and the POET-X technical summary, section 2 (input-centric form,
index-map permutations with reduction from four to two, block-diagonal factors, CNP with
upper-triangle storage).
"""
import os

import numpy as np
import pytest

from oracle import poetx_ref as ref


def _golden_rows(path):
    rows = []
    with open(path) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


# ----------------------------------------------------------------------------- perms
def test_splitmix64_known_answers(golden_dir):
    for row in _golden_rows(os.path.join(golden_dir, "splitmix64_kat.txt")):
        seed, outs = int(row[0]), [int(v) for v in row[1:]]
        g = ref.splitmix64(seed)
        assert [next(g) for _ in outs] == outs


def test_fisher_yates_hand_trace(golden_dir):
    rows = {r[0]: [int(v) for v in r[1:]] for r in _golden_rows(
        os.path.join(golden_dir, "fisher_yates_seed0_n4.txt"))}
    p, inv = ref.make_perm(0, 4)
    assert p.tolist() == rows["perm"]
    assert inv.tolist() == rows["inv"]


@pytest.mark.parametrize("n", [1, 2, 7, 256, 2048, 14336])
def test_perm_is_bijection_with_inverse(n):
    p, inv = ref.make_perm(12345 + n, n)
    assert np.array_equal(np.sort(p), np.arange(n))
    assert np.array_equal(p[inv], np.arange(n))
    assert np.array_equal(inv[p], np.arange(n))


def test_perm_uniform_on_three_elements():
    # Fisher-Yates with an unbiased draw gives each of the 3! orders with p = 1/6.
    counts = {}
    N = 6000
    for s in range(N):
        key = tuple(ref.make_perm(s, 3)[0].tolist())
        counts[key] = counts.get(key, 0) + 1
    assert len(counts) == 6
    for c in counts.values():
        assert abs(c - N / 6) < 5 * np.sqrt(N / 6)  # 5 sigma


def test_perm_matrix_convention():
    p = np.array([2, 0, 1])
    x = np.array([10.0, 20.0, 30.0])
    assert np.array_equal(ref.perm_matrix(p) @ x, x[p])
    assert np.array_equal(ref.perm_matrix(p).T @ x[p], x)


# ------------------------------------------------------------------------------ CNP
def test_theta_packing(golden_dir):
    rows = _golden_rows(os.path.join(golden_dir, "theta_packing_b4.txt"))
    theta = np.array([float(v) for v in rows[0][1:]])
    Q = np.array([[float(v) for v in r[1:]] for r in rows[1:]])
    assert np.array_equal(ref.theta_to_Q(theta, 4), Q)
    assert np.array_equal(ref.Q_to_theta(Q), theta)


def test_cnp_b2_golden(golden_dir):
    for row in _golden_rows(os.path.join(golden_dir, "cnp_b2_closed_form.txt")):
        t, k = float(row[0]), int(row[1])
        G_expect = np.array([float(v) for v in row[2:6]]).reshape(2, 2)
        gtg = float(row[6])
        G = ref.cnp_forward(np.array([[t]]), 2, k)[0]
        assert np.array_equal(G, G_expect)  # exact in binary
        assert np.array_equal(G.T @ G, gtg * np.eye(2))


@pytest.mark.parametrize("k", [1, 2, 3, 4, 5, 6, 9])
def test_cnp_b2_closed_form(k):
    # P2: Q^2 = -t^2 I collapses the Neumann sum to alpha I + beta Q.
    for t in [0.0, 0.013, -0.2, 0.37]:
        alpha = sum((-t * t) ** j for j in range(k // 2 + 1))
        beta = sum((-t * t) ** j for j in range((k - 1) // 2 + 1))
        G = ref.cnp_forward(np.array([[t]]), 2, k)[0]
        expect = np.array([[alpha - beta * t * t, (alpha + beta) * t],
                           [-(alpha + beta) * t, alpha - beta * t * t]])
        assert np.allclose(G, expect, rtol=0, atol=1e-15)
        C = ref.cayley_exact(ref.theta_to_Q(np.array([t]), 2))
        rot = np.array([[1 - t * t, 2 * t], [-2 * t, 1 - t * t]]) / (1 + t * t)
        assert np.allclose(C, rot, rtol=0, atol=1e-15)


def test_identity_at_zero_theta():
    # P1: theta = 0 gives G = I exactly.
    for b in [2, 4, 32, 256]:
        G = ref.cnp_forward(np.zeros((3, b * (b - 1) // 2)), b, 4)
        assert np.array_equal(G, np.broadcast_to(np.eye(b), G.shape))


@pytest.mark.parametrize("b,k", [(8, 1), (8, 2), (16, 3), (16, 4), (32, 4), (64, 6), (64, 5)])
def test_truncation_error_against_exact_cayley(b, k):
    # P4: G = C (I - Q^(k+1)) => ||G - C||_2 = ||Q||_2^(k+1) exactly (C orthogonal, Q normal).
    rng = np.random.default_rng(b * 100 + k)
    Q = ref.theta_to_Q(rng.standard_normal(b * (b - 1) // 2) * 0.05, b)
    G = ref.cnp_block(Q, k)
    C = ref.cayley_exact(Q)
    assert np.allclose(C.T @ C, np.eye(b), atol=1e-13)
    nq = np.linalg.norm(Q, 2)
    assert nq < 1
    assert np.isclose(np.linalg.norm(G - C, 2), nq ** (k + 1), rtol=1e-6, atol=1e-16)


@pytest.mark.parametrize("b", [4, 16, 64])
def test_orthogonality_defect_closed_form(b):
    # P5: G^T G = (I - Q^(k+1)) (I - (-Q)^(k+1)); for even k that is I - Q^(2k+2) and
    # ||G^T G - I||_2 = ||Q||_2^(2k+2); the defect shrinks as k grows.
    rng = np.random.default_rng(b)
    Q = ref.theta_to_Q(rng.standard_normal(b * (b - 1) // 2), b)
    Q *= 0.5 / np.linalg.norm(Q, 2)  # the Neumann series needs ||Q|| < 1
    nq = np.linalg.norm(Q, 2)
    prev = np.inf
    for k in range(1, 9):
        G = ref.cnp_block(Q, k)
        I = np.eye(b)
        Qk1 = np.linalg.matrix_power(Q, k + 1)
        mQk1 = np.linalg.matrix_power(-Q, k + 1)
        assert np.allclose(G.T @ G, (I - Qk1) @ (I - mQk1), rtol=0, atol=1e-14)
        defect = np.linalg.norm(G.T @ G - I, 2)
        if k % 2 == 0:
            # float64 rounding of G^T G - I is ~1e-15, so the closed form is checked to that
            assert np.isclose(defect, nq ** (2 * k + 2), rtol=1e-6, atol=1e-14)
            if defect > 1e-12:
                assert defect < prev
            prev = defect


def test_cnp_forward_batches_blocks():
    rng = np.random.default_rng(7)
    th = rng.standard_normal((3, 6)) * 0.1
    G = ref.cnp_forward(th, 4, 3)
    for j in range(3):
        assert np.array_equal(G[j], ref.cnp_block(ref.theta_to_Q(th[j], 4), 3))


@pytest.mark.parametrize("b,k", [(2, 1), (2, 4), (4, 1), (4, 2), (5, 3), (8, 4), (8, 6)])
def test_cnp_backward_finite_differences(b, k):
    # P10 on tiny blocks: <dtheta, e_i> against central differences of <dG, G(theta)>.
    rng = np.random.default_rng(100 * b + k)
    ntri = b * (b - 1) // 2
    th = rng.standard_normal((2, ntri)) * 0.1
    dG = rng.standard_normal((2, b, b))
    dth = ref.cnp_backward(th, dG, b, k)
    h = 1e-6
    for blk in range(2):
        for i in range(ntri):
            e = np.zeros(ntri)
            e[i] = h
            fp = np.sum(dG[blk] * ref.cnp_block(ref.theta_to_Q(th[blk] + e, b), k))
            fm = np.sum(dG[blk] * ref.cnp_block(ref.theta_to_Q(th[blk] - e, b), k))
            assert np.isclose(dth[blk, i], (fp - fm) / (2 * h), rtol=1e-7, atol=1e-8)


@pytest.mark.parametrize("b,k", [(64, 4), (256, 4), (128, 2)])
def test_cnp_backward_directional_derivative(b, k):
    # P10 at full block size: <dtheta, delta> = <dG, dG/dtheta[delta]> by central differences.
    rng = np.random.default_rng(b + k)
    ntri = b * (b - 1) // 2
    th = rng.standard_normal((1, ntri)) * 0.01
    dG = rng.standard_normal((1, b, b))
    dth = ref.cnp_backward(th, dG, b, k)[0]
    for _ in range(2):
        d = rng.standard_normal(ntri)
        d /= np.linalg.norm(d)
        h = 1e-4
        Gp = ref.cnp_block(ref.theta_to_Q(th[0] + h * d, b), k)
        Gm = ref.cnp_block(ref.theta_to_Q(th[0] - h * d, b), k)
        fd = np.sum(dG[0] * (Gp - Gm)) / (2 * h)
        assert np.isclose(np.dot(dth, d), fd, rtol=1e-7)


# ---------------------------------------------------------------------------- layer
def _small_layer(n, m, b, k, T, seed, scale=0.1):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, n))
    W0 = rng.standard_normal((m, n)) / np.sqrt(n)
    tP = rng.standard_normal((n // b, b * (b - 1) // 2)) * scale
    tR = rng.standard_normal((m // b, b * (b - 1) // 2)) * scale
    dy = rng.standard_normal((T, m))
    pP, _ = ref.make_perm(seed * 2 + 1, n)
    pR, _ = ref.make_perm(seed * 2 + 2, m)
    return x, W0, tP, tR, dy, pP, pR


def test_identity_layer_is_plain_linear():
    # P1: theta = 0 => G = I and the permutations cancel: y = W0 x for each token.
    n, m, b, T = 32, 48, 8, 6
    x, W0, tP, tR, dy, pP, pR = _small_layer(n, m, b, 4, T, 3)
    GP = ref.cnp_forward(np.zeros_like(tP), b, 4)
    GR = ref.cnp_forward(np.zeros_like(tR), b, 4)
    y = ref.layer_forward(x, ref.merge_perm(W0, pR, pP), GP, GR, pP, pR)[0]
    assert np.allclose(y, x @ W0.T, rtol=0, atol=1e-13)


def test_merge_perm_definition():
    # P7: W0'[i, j] = W0[p_R[i], p_P[j]] element by element, and W0' = Pi_R W0 Pi_P^T.
    rng = np.random.default_rng(0)
    m, n = 6, 5
    W0 = rng.standard_normal((m, n))
    pR, _ = ref.make_perm(1, m)
    pP, _ = ref.make_perm(2, n)
    W0p = ref.merge_perm(W0, pR, pP)
    for i in range(m):
        for j in range(n):
            assert W0p[i, j] == W0[pR[i], pP[j]]
    assert np.array_equal(W0p, ref.perm_matrix(pR) @ W0 @ ref.perm_matrix(pP).T)


@pytest.mark.parametrize("n,m,b,k,T", [(16, 24, 4, 4, 7), (64, 32, 16, 3, 5), (8, 12, 2, 1, 3)])
def test_merged_equals_unmerged(n, m, b, k, T):
    # P7: two merged permutations + index maps == the four-permutation dense form.
    x, W0, tP, tR, dy, pP, pR = _small_layer(n, m, b, k, T, n + m)
    GP, GR = ref.cnp_forward(tP, b, k), ref.cnp_forward(tR, b, k)
    y_dense = ref.layer_dense(x, W0, GP, GR, pP, pR)
    y = ref.layer_forward(x, ref.merge_perm(W0, pR, pP), GP, GR, pP, pR)[0]
    assert np.allclose(y, y_dense, rtol=1e-13, atol=1e-13 * np.abs(y_dense).max())


def test_spectrum_preserved_with_exact_cayley():
    # P6: R W0 P with exactly orthogonal R, P keeps the singular values of W0.
    n, m, b = 32, 24, 8
    x, W0, tP, tR, dy, pP, pR = _small_layer(n, m, b, 4, 2, 11, scale=0.3)
    CP = np.stack([ref.cayley_exact(ref.theta_to_Q(t, b)) for t in tP])
    CR = np.stack([ref.cayley_exact(ref.theta_to_Q(t, b)) for t in tR])
    Weff = ref.poet_weight(W0, CP, CR, pP, pR)
    s0 = np.linalg.svd(W0, compute_uv=False)
    s1 = np.linalg.svd(Weff, compute_uv=False)
    assert np.allclose(s0, s1, rtol=1e-12, atol=1e-12)


# ----------------------------------------------------------------- outer-loop merge
def test_outer_merge_at_zero_theta_is_a_pure_remerge():
    # theta = 0 => G = I: W0_new = W0 exactly and W0'_new is W0 gathered by the new maps.
    n, m, b = 32, 48, 8
    x, W0, tP, tR, dy, pP, pR = _small_layer(n, m, b, 4, 2, 21)
    GP = ref.cnp_forward(np.zeros_like(tP), b, 4)
    GR = ref.cnp_forward(np.zeros_like(tR), b, 4)
    pP2, _ = ref.make_perm(101, n)
    pR2, _ = ref.make_perm(102, m)
    W0_new, W0p_new = ref.outer_merge(W0, GP, GR, pP, pR, pP2, pR2)
    assert np.array_equal(W0_new, W0)
    assert np.array_equal(W0p_new, W0[np.ix_(pR2, pP2)])


def test_outer_merge_keeps_the_spectrum_with_exact_cayley():
    # [POET] abstract: the transform preserves the singular values of W0, so the merge
    # with exactly orthogonal factors must too.
    n, m, b = 32, 24, 8
    x, W0, tP, tR, dy, pP, pR = _small_layer(n, m, b, 4, 2, 23, scale=0.3)
    CP = np.stack([ref.cayley_exact(ref.theta_to_Q(t, b)) for t in tP])
    CR = np.stack([ref.cayley_exact(ref.theta_to_Q(t, b)) for t in tR])
    pP2, _ = ref.make_perm(7, n)
    pR2, _ = ref.make_perm(8, m)
    W0_new, W0p_new = ref.outer_merge(W0, CP, CR, pP, pR, pP2, pR2)
    s0 = np.linalg.svd(W0, compute_uv=False)
    assert np.allclose(np.linalg.svd(W0_new, compute_uv=False), s0, rtol=1e-12, atol=1e-12)
    assert np.allclose(np.linalg.svd(W0p_new, compute_uv=False), s0, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("n,m,b,k", [(16, 24, 4, 4), (64, 32, 16, 3)])
def test_outer_merge_preserves_the_layer(n, m, b, k):
    # The layer with rotations G and permutations p equals the layer after the merge with
    # theta = 0 and new permutations p' (input-centric forward with index maps on both
    # sides, so the merge is checked against a different code path than its own).
    x, W0, tP, tR, dy, pP, pR = _small_layer(n, m, b, k, 5, n * m)
    GP, GR = ref.cnp_forward(tP, b, k), ref.cnp_forward(tR, b, k)
    pP2, _ = ref.make_perm(n + 5, n)
    pR2, _ = ref.make_perm(m + 6, m)
    y0 = ref.layer_forward(x, ref.merge_perm(W0, pR, pP), GP, GR, pP, pR)[0]
    _, W0p_new = ref.outer_merge(W0, GP, GR, pP, pR, pP2, pR2)
    I_P = ref.cnp_forward(np.zeros_like(tP), b, k)
    I_R = ref.cnp_forward(np.zeros_like(tR), b, k)
    y1 = ref.layer_forward(x, W0p_new, I_P, I_R, pP2, pR2)[0]
    assert np.allclose(y1, y0, rtol=1e-12, atol=1e-12 * np.abs(y0).max())
    # a planted mistake (the rotations applied transposed) breaks the equivalence
    _, bad = ref.outer_merge(W0, GP.transpose(0, 2, 1), GR, pP, pR, pP2, pR2)
    y2 = ref.layer_forward(x, bad, I_P, I_R, pP2, pR2)[0]
    assert not np.allclose(y2, y0, rtol=1e-6, atol=1e-6 * np.abs(y0).max())


# ------------------------------------------------------------------ int8 base weight
def test_int8_rows_round_trip_within_half_a_step():
    # every element is within s/2 of its dequantised value (plus fp32 rounding of w / s),
    # each nonzero row reaches the full code range, and codes stay in [-127, 127]
    rng = np.random.default_rng(4)
    W = (rng.standard_normal((37, 53)) * rng.uniform(0.01, 3, (37, 1))).astype(np.float32)
    W[5] = 0.0
    q, s = ref.quantize_rows_int8(W)
    assert q.dtype == np.int8 and s.dtype == np.float32
    assert np.all(np.abs(q.astype(int)) <= 127)
    err = np.abs(ref.dequantize_rows(q, s) - W.astype(np.float64))
    assert np.all(err <= s[:, None].astype(np.float64) * (0.5 + 1e-5) + 1e-30)
    nz = s > 0
    assert np.all(np.abs(q[nz].astype(int)).max(axis=1) == 127)
    assert s[5] == 0 and np.all(q[5] == 0)


def test_int8_rows_exact_on_the_grid():
    # weights that are integer multiples of a power-of-two step with max |k| = 127 come
    # back exactly (s = step exactly, w / s exact)
    rng = np.random.default_rng(6)
    k = rng.integers(-127, 128, size=(9, 40))
    k[:, 0] = 127
    step = 2.0 ** -rng.integers(1, 12, size=(9, 1))
    W = (k * step).astype(np.float32)
    q, s = ref.quantize_rows_int8(W)
    assert np.array_equal(q.astype(int), k)
    assert np.array_equal(s.astype(np.float64), step[:, 0])
    # and a planted mistake (truncation instead of rounding) breaks the half-step bound
    Wr = rng.standard_normal((8, 64)).astype(np.float32)
    q2, s2 = ref.quantize_rows_int8(Wr)
    trunc = np.trunc(Wr / s2[:, None])
    assert not np.array_equal(trunc, q2.astype(np.float32))


@pytest.mark.parametrize("k", [2, 4])
def test_spectrum_bounds_with_cnp(k):
    # P6 with the truncated G: each factor has singular values in [1-eps, 1+eps],
    # eps = ||Q||^(k+1), so sigma_i(R W0 P) / sigma_i(W0) lies in [(1-eps)^2, (1+eps)^2].
    n, m, b = 32, 24, 8
    x, W0, tP, tR, dy, pP, pR = _small_layer(n, m, b, k, 2, 13, scale=0.1)
    GP, GR = ref.cnp_forward(tP, b, k), ref.cnp_forward(tR, b, k)
    eps = max(np.linalg.norm(ref.theta_to_Q(t, b), 2) for t in np.concatenate([tP, tR])) ** (k + 1)
    r = np.linalg.svd(ref.poet_weight(W0, GP, GR, pP, pR), compute_uv=False) / \
        np.linalg.svd(W0, compute_uv=False)
    assert np.all(r >= (1 - eps) ** 2 - 1e-12) and np.all(r <= (1 + eps) ** 2 + 1e-12)
    assert 1e-6 < eps < 1  # the bound is meaningful here


@pytest.mark.parametrize("n,m,b,k", [(8, 12, 4, 1), (8, 12, 4, 2), (8, 12, 4, 3), (8, 12, 4, 4),
                                     (8, 12, 2, 4)])
def test_layer_finite_differences(n, m, b, k):
    # P8: gradients of L = <dY, Y> w.r.t. x, theta_P, theta_R by central differences.
    T = 5
    x, W0, tP, tR, dy, pP, pR = _small_layer(n, m, b, k, T, 31 * n + m + b + k, scale=0.2)
    W0p = ref.merge_perm(W0, pR, pP)

    def loss(x_, tP_, tR_):
        y = ref.layer_forward(x_, W0p, ref.cnp_forward(tP_, b, k), ref.cnp_forward(tR_, b, k),
                              pP, pR)[0]
        return np.sum(dy * y)

    GP, GR = ref.cnp_forward(tP, b, k), ref.cnp_forward(tR, b, k)
    dx, dGP, dGR = ref.layer_backward(x, dy, W0p, GP, GR, pP, pR)
    dtP = ref.cnp_backward(tP, dGP, b, k)
    dtR = ref.cnp_backward(tR, dGR, b, k)
    h = 1e-6

    def fd(arr, idx, which):
        a1, a2 = arr.copy(), arr.copy()
        a1[idx] += h
        a2[idx] -= h
        args1 = {"x": (a1, tP, tR), "P": (x, a1, tR), "R": (x, tP, a1)}[which]
        args2 = {"x": (a2, tP, tR), "P": (x, a2, tR), "R": (x, tP, a2)}[which]
        return (loss(*args1) - loss(*args2)) / (2 * h)

    for idx in np.ndindex(x.shape):
        assert np.isclose(dx[idx], fd(x, idx, "x"), rtol=1e-7, atol=1e-8)
    for idx in np.ndindex(tP.shape):
        assert np.isclose(dtP[idx], fd(tP, idx, "P"), rtol=1e-7, atol=1e-8)
    for idx in np.ndindex(tR.shape):
        assert np.isclose(dtR[idx], fd(tR, idx, "R"), rtol=1e-7, atol=1e-8)


def test_inner_product_identities():
    # P9: Y is linear in X, in G_P and in G_R separately, so
    # <dY, Y> = <dX, X> = sum_j <dG_P,j, G_P,j> = sum_j <dG_R,j, G_R,j>.
    n, m, b, k, T = 64, 96, 16, 4, 37
    x, W0, tP, tR, dy, pP, pR = _small_layer(n, m, b, k, T, 5)
    W0p = ref.merge_perm(W0, pR, pP)
    GP, GR = ref.cnp_forward(tP, b, k), ref.cnp_forward(tR, b, k)
    y = ref.layer_forward(x, W0p, GP, GR, pP, pR)[0]
    dx, dGP, dGR = ref.layer_backward(x, dy, W0p, GP, GR, pP, pR)
    L = np.sum(dy * y)
    for v in [np.sum(dx * x), np.sum(dGP * GP), np.sum(dGR * GR)]:
        assert np.isclose(v, L, rtol=1e-12)


def test_row_subset_helpers_match_full():
    n, m, b, k, T = 32, 16, 8, 2, 9
    x, W0, tP, tR, dy, pP, pR = _small_layer(n, m, b, k, T, 17)
    W0p = ref.merge_perm(W0, pR, pP)
    GP, GR = ref.cnp_forward(tP, b, k), ref.cnp_forward(tR, b, k)
    y = ref.layer_forward(x, W0p, GP, GR, pP, pR)[0]
    dx = ref.layer_backward(x, dy, W0p, GP, GR, pP, pR)[0]
    rows = [0, 4, 8]
    assert np.array_equal(ref.layer_forward_rows(x[rows], W0p, GP, GR, pP, pR), y[rows])
    assert np.allclose(ref.layer_backward_dx_rows(dy[rows], W0p, GP, GR, pP, pR), dx[rows],
                       rtol=0, atol=1e-14)


# ------------------------------------------------------------- planted mistakes
def _p4_holds(cnp_block_fn, b=16, k=4):
    rng = np.random.default_rng(1)
    Q = ref.theta_to_Q(rng.standard_normal(b * (b - 1) // 2) * 0.05, b)
    G = cnp_block_fn(Q, k)
    return np.isclose(np.linalg.norm(G - ref.cayley_exact(Q), 2),
                      np.linalg.norm(Q, 2) ** (k + 1), rtol=1e-6)


def _fd_holds(backward_block_fn, b=4, k=3):
    rng = np.random.default_rng(2)
    th = rng.standard_normal(b * (b - 1) // 2) * 0.1
    dG = rng.standard_normal((b, b))
    iu, ju = np.triu_indices(b, 1)
    dQ = backward_block_fn(ref.theta_to_Q(th, b), dG, k)
    dth = dQ[iu, ju] - dQ[ju, iu]
    h = 1e-6
    for i in range(len(th)):
        e = np.zeros_like(th)
        e[i] = h
        fd = (np.sum(dG * ref.cnp_block(ref.theta_to_Q(th + e, b), k)) -
              np.sum(dG * ref.cnp_block(ref.theta_to_Q(th - e, b), k))) / (2 * h)
        if not np.isclose(dth[i], fd, rtol=1e-7, atol=1e-8):
            return False
    return True


def test_pins_catch_planted_mistakes():
    """Plant plausible slips in copies of oracle steps and check that a pin rejects each."""
    assert _p4_holds(ref.cnp_block) and _fd_holds(ref.cnp_backward_block)

    def dropped_last_power(Q, k):  # Neumann sum one term short
        return (np.eye(Q.shape[0]) + Q) @ ref.neumann_sum(Q, k - 1)
    assert not _p4_holds(dropped_last_power)

    def wrong_cayley_sign(Q, k):  # (I - Q)(sum Q^i): truncates neither Cayley form
        return (np.eye(Q.shape[0]) - Q) @ ref.neumann_sum(Q, k)
    assert not _p4_holds(wrong_cayley_sign)

    def transposed_upstream(Q, dG, k):  # (I+Q) dG instead of (I+Q)^T dG
        b = Q.shape[0]
        I = np.eye(b)
        dQ = dG @ ref.neumann_sum(Q, k).T
        up = (I + Q) @ dG
        pw = [I]
        for _ in range(k):
            pw.append(pw[-1] @ Q.T)
        for i in range(1, k + 1):
            for a in range(i):
                dQ = dQ + pw[a] @ up @ pw[i - 1 - a]
        return dQ
    assert not _fd_holds(transposed_upstream)

    def missing_direct_term(Q, dG, k):  # forgets dG N^T
        return ref.cnp_backward_block(Q, dG, k) - dG @ ref.neumann_sum(Q, k).T
    assert not _fd_holds(missing_direct_term)

    # Packing sign flip (Q_ij = -theta): the b = 2 closed form sees it.
    t = 0.5
    G_flip = ref.cnp_block(-ref.theta_to_Q(np.array([t]), 2), 4)
    assert not np.array_equal(G_flip, np.array([[0.625, 0.78125], [-0.78125, 0.625]]))


def test_block_grads_helper_matches_full_backward():
    n, m, b, k, T = 32, 48, 8, 4, 11
    x, W0, tP, tR, dy, pP, pR = _small_layer(n, m, b, k, T, 23)
    W0p = ref.merge_perm(W0, pR, pP)
    GP, GR = ref.cnp_forward(tP, b, k), ref.cnp_forward(tR, b, k)
    _, dGP, dGR = ref.layer_backward(x, dy, W0p, GP, GR, pP, pR)
    for jR, jP in [(0, 0), (5, 3), (2, 1)]:
        gP, gR = ref.layer_block_grads(x, dy, W0p, GP, GR, pP, pR, jR, jP)
        assert np.allclose(gP, dGP[jP], rtol=0, atol=1e-13)
        assert np.allclose(gR, dGR[jR], rtol=0, atol=1e-13)
