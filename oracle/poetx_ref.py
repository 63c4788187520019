"""Float64 CPU oracle for the POET-X orthogonal-equivalence linear layer.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or execute this
module: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` use it.  It shares no code with the CUDA library and the library does not
share code with it; the only common module is ``poetx_inputs`` (seeded numbers, no
arithmetic of the method).

What it computes, and where each step is stated
-----------------------------------------------
Sources (web pages on the subject; formulas there are inline fragments):
  [POET]   "Reparameterized LLM Training via Orthogonal Equivalence Transformation",
           abstract: every weight is W = R W0 P with R, P learnable orthogonal matrices and
           W0 a fixed random matrix; the transform preserves the singular values of W0.
  [POET-X] "POET-X: Memory-efficient LLM Training by Scaling Orthogonal Transformation",
           technical summary section 2 (Methodology):
             2.1 input-centric (matrix-free) computation: the product is applied to the
                 input, no weight-sized intermediate is formed;
             2.2 permutations applied by index maps, never as matrices; two of the four
                 permutations of the forward are merged into W once;
             2.3 block-diagonal orthogonal factors, each b x b block an independent matrix;
             2.4 Cayley-Neumann parameterisation (CNP) of each block from a skew-symmetric
                 Q stored as its strict upper triangle, b(b-1)/2 numbers per block;
             2.5 gradient checkpointing variant (recompute in backward).
The pages never print the CNP polynomial, the layer equation, the permutation convention
or the packing order.  The readings used here (all listed with their reasons in the
design notes) are:
  * CNP: G = (I + Q) (I + Q + Q^2 + ... + Q^k), the k-term Neumann truncation of the
    Cayley transform (I + Q)(I - Q)^-1.  Computed here in that product form with explicit
    powers.
  * theta packing: strict upper triangle row-major (numpy.triu_indices(b, 1) order),
    Q[i, j] = theta, Q[j, i] = -theta for i < j.
  * permutation p acts as (Pi x)_i = x[p[i]]; Pi^T x is the gather by the inverse.
  * y = (Pi_R^T G_R Pi_R) W0 (Pi_P^T G_P Pi_P) x, merged weight W0' = Pi_R W0 Pi_P^T,
    i.e. W0'[i, j] = W0[p_R[i], p_P[j]].
  * W0 is frozen (the abstract's "fixed random weight matrix"): no dW0.
  * permutation generator: SplitMix64 (Steele, Lea, Flood 2014) feeding a Durstenfeld
    Fisher-Yates shuffle with Lemire's multiply-shift bounded draw (no rejection).

Pins (tests/test_oracle_pins.py) tie every function to something other than itself:
closed forms (b = 2 rotation), the exact Cayley transform from LAPACK, the orthogonality
defect identity, singular-value preservation, permutation invariants, the dense
4-permutation form against the merged input-centric form, and central finite differences.
"""
from __future__ import annotations

import numpy as np

MASK64 = (1 << 64) - 1

# ---------------------------------------------------------------------------------------
# Permutations  [POET-X 2.2: fixed random permutations applied through index maps]
# ---------------------------------------------------------------------------------------


def splitmix64(state: int):
    """Generator of SplitMix64 outputs (Steele, Lea & Flood, OOPSLA 2014; Vigna's
    public-domain reference).  state advances by the golden-ratio increment, the output
    is the variant-13 finaliser of the new state."""
    while True:
        state = (state + 0x9E3779B97F4A7C15) & MASK64
        z = state
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK64
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK64
        yield z ^ (z >> 31)


def make_perm(seed: int, n: int):
    """Seeded random permutation of range(n) and its inverse (int64 arrays).

    Durstenfeld's Fisher-Yates: for i = n-1 down to 1, draw j uniformly in [0, i] as the
    high 64 bits of (r * (i + 1)) for a 64-bit draw r (Lemire's multiply-shift, no
    rejection step), swap p[i], p[j].  inv[p[i]] = i.
    """
    p = list(range(n))
    rng = splitmix64(seed & MASK64)
    for i in range(n - 1, 0, -1):
        r = next(rng)
        j = (r * (i + 1)) >> 64
        p[i], p[j] = p[j], p[i]
    perm = np.array(p, dtype=np.int64)
    inv = np.empty(n, dtype=np.int64)
    inv[perm] = np.arange(n, dtype=np.int64)
    return perm, inv


def perm_matrix(p: np.ndarray) -> np.ndarray:
    """Dense Pi with (Pi x)_i = x[p[i]]  -- only for small-n cross-checks."""
    n = len(p)
    P = np.zeros((n, n))
    P[np.arange(n), p] = 1.0
    return P


# ---------------------------------------------------------------------------------------
# Cayley-Neumann parameterisation  [POET-X 2.4]
# ---------------------------------------------------------------------------------------


def theta_to_Q(theta_blk: np.ndarray, b: int) -> np.ndarray:
    """Skew-symmetric Q (b x b) from its packed strict upper triangle (row-major order)."""
    iu, ju = np.triu_indices(b, 1)
    Q = np.zeros((b, b))
    Q[iu, ju] = theta_blk
    Q[ju, iu] = -np.asarray(theta_blk, dtype=np.float64)
    return Q


def Q_to_theta(Q: np.ndarray) -> np.ndarray:
    b = Q.shape[0]
    iu, ju = np.triu_indices(b, 1)
    return Q[iu, ju].copy()


def neumann_sum(Q: np.ndarray, k: int) -> np.ndarray:
    """I + Q + Q^2 + ... + Q^k with explicit powers."""
    b = Q.shape[0]
    acc = np.eye(b)
    Qi = np.eye(b)
    for _ in range(k):
        Qi = Qi @ Q
        acc = acc + Qi
    return acc


def cnp_block(Q: np.ndarray, k: int) -> np.ndarray:
    """G = (I + Q) (I + Q + ... + Q^k)."""
    b = Q.shape[0]
    return (np.eye(b) + Q) @ neumann_sum(Q, k)


def cnp_forward(theta: np.ndarray, b: int, k: int) -> np.ndarray:
    """theta [nblk, b(b-1)/2] -> G [nblk, b, b] (float64)."""
    theta = np.asarray(theta, dtype=np.float64)
    return np.stack([cnp_block(theta_to_Q(t, b), k) for t in theta]) if len(theta) else \
        np.zeros((0, b, b))


def cayley_exact(Q: np.ndarray) -> np.ndarray:
    """C = (I + Q)(I - Q)^-1 via a LAPACK solve (C (I - Q) = I + Q)."""
    b = Q.shape[0]
    I = np.eye(b)
    # C = (I+Q) (I-Q)^{-1}  <=>  (I-Q)^T C^T = (I+Q)^T
    return np.linalg.solve((I - Q).T, (I + Q).T).T


def cnp_backward_block(Q: np.ndarray, dG: np.ndarray, k: int) -> np.ndarray:
    """dL/dQ for G = (I + Q) N(Q), N(Q) = sum_{i=0..k} Q^i, by the chain rule on that
    product form:

        dQ = dG N^T + sum_{i=1..k} sum_{a=0..i-1} (Q^T)^a [(I + Q)^T dG] (Q^T)^(i-1-a)

    (the second term is the adjoint of Q -> Q^i, d(Q^i)[H] = sum_a Q^a H Q^(i-1-a)).
    """
    b = Q.shape[0]
    I = np.eye(b)
    N = neumann_sum(Q, k)
    dQ = dG @ N.T
    upstream_N = (I + Q).T @ dG
    QT = Q.T
    powT = [I]
    for _ in range(k):
        powT.append(powT[-1] @ QT)
    for i in range(1, k + 1):
        for a in range(i):
            dQ = dQ + powT[a] @ upstream_N @ powT[i - 1 - a]
    return dQ


def cnp_backward(theta: np.ndarray, dG: np.ndarray, b: int, k: int) -> np.ndarray:
    """dtheta [nblk, b(b-1)/2]: dtheta_(i,j) = dQ_ij - dQ_ji for i < j (Q_ij = theta,
    Q_ji = -theta)."""
    theta = np.asarray(theta, dtype=np.float64)
    dG = np.asarray(dG, dtype=np.float64)
    iu, ju = np.triu_indices(b, 1)
    out = np.zeros((len(theta), len(iu)))
    for blk in range(len(theta)):
        dQ = cnp_backward_block(theta_to_Q(theta[blk], b), dG[blk], k)
        out[blk] = dQ[iu, ju] - dQ[ju, iu]
    return out


# ---------------------------------------------------------------------------------------
# The layer  [POET abstract: W = R W0 P;  POET-X 2.1-2.3]
# ---------------------------------------------------------------------------------------


def blockdiag(Gs: np.ndarray) -> np.ndarray:
    nblk, b, _ = Gs.shape
    D = np.zeros((nblk * b, nblk * b))
    for j in range(nblk):
        D[j * b:(j + 1) * b, j * b:(j + 1) * b] = Gs[j]
    return D


def merge_perm(W0: np.ndarray, perm_R: np.ndarray, perm_P: np.ndarray) -> np.ndarray:
    """W0' = Pi_R W0 Pi_P^T, i.e. W0'[i, j] = W0[p_R[i], p_P[j]]  [POET-X 2.2, reduction]."""
    return np.asarray(W0)[np.ix_(perm_R, perm_P)]


def poet_weight(W0, G_P, G_R, perm_P, perm_R) -> np.ndarray:
    """The effective weight R W0 P with R = Pi_R^T G_R Pi_R and P = Pi_P^T G_P Pi_P
    (dense matrices; small sizes only)."""
    PiP, PiR = perm_matrix(perm_P), perm_matrix(perm_R)
    R = PiR.T @ blockdiag(G_R) @ PiR
    P = PiP.T @ blockdiag(G_P) @ PiP
    return R @ np.asarray(W0, dtype=np.float64) @ P


def outer_merge(W0, G_P, G_R, perm_P, perm_R, perm_P_new, perm_R_new):
    """Outer-loop merge and re-initialisation.  The original POET step folds the rotations
    into the weight, W <- R_i W P_i ([POET-X] technical summary 2.1, where it is the
    weight-centric update the input-centric form replaces; [POET] abstract: W = R W0 P).
    At the end of an inner loop the learnt R, P are absorbed this way, W0_new = R W0 P
    (dense R, P built as in poet_weight), and the next inner loop starts from theta = 0
    with fresh permutations, whose merged weight is W0'_new = Pi_R' W0_new Pi_P'^T.

    Returns (W0_new, W0'_new)."""
    W0_new = poet_weight(W0, G_P, G_R, perm_P, perm_R)
    return W0_new, merge_perm(W0_new, perm_R_new, perm_P_new)


def quantize_rows_int8(W):
    """Per-row symmetric int8 base weight (POET-XQ: training on a low-bit base model whose
    weight is dequantised on the fly, [POET-X] technical summary 2.6).  The pages give no
    scheme; the reading here: one fp32 scale per output channel (row), s = max|w| / 127,
    q = round-to-nearest-even(w / s) clamped to [-127, 127]; an all-zero row has s = 0
    and q = 0.  The rounding decides integers, so it is taken in fp32 (IEEE division,
    as the GPU takes it).  Returns (q int8 [m, n], s float32 [m])."""
    W32 = np.asarray(W, dtype=np.float32)
    amax = np.max(np.abs(W32), axis=1) if W32.shape[1] else np.zeros(W32.shape[0], np.float32)
    s = (amax / np.float32(127.0)).astype(np.float32)
    safe = np.where(s > 0, s, np.float32(1.0)).astype(np.float32)
    q = np.rint(W32 / safe[:, None]).astype(np.float32)
    q = np.clip(q, -127, 127)
    q[s == 0] = 0
    return q.astype(np.int8), s


def dequantize_rows(q, s) -> np.ndarray:
    """W = s[i] q[i, j] (float64)."""
    return np.asarray(s, dtype=np.float64)[:, None] * np.asarray(q, dtype=np.float64)


def layer_dense(x, W0, G_P, G_R, perm_P, perm_R) -> np.ndarray:
    """Rows of Y = (R W0 P x_t)^T with the four permutations as matrices and the unmerged
    W0 (the weight-centric reading; small sizes only)."""
    Weff = poet_weight(W0, G_P, G_R, perm_P, perm_R)
    return np.asarray(x, dtype=np.float64) @ Weff.T


def _block_apply(A: np.ndarray, Gs: np.ndarray, transpose: bool) -> np.ndarray:
    """Per block j: A[:, jb:(j+1)b] @ (G_j^T if transpose else G_j)."""
    nblk, b, _ = Gs.shape
    out = np.empty_like(A)
    for j in range(nblk):
        Gj = Gs[j].T if transpose else Gs[j]
        out[:, j * b:(j + 1) * b] = A[:, j * b:(j + 1) * b] @ Gj
    return out


def layer_forward(x, W0p, G_P, G_R, perm_P, perm_R):
    """Input-centric forward with the merged weight and two index-map permutations.

    Token rows: U = X[:, p_P]; V_j = U_j G_P,j^T; W = V W0'^T; Z_j = W_j G_R,j^T;
    Y[:, p_R[i]] = Z[:, i].   Returns (Y, U, V, W).
    """
    x = np.asarray(x, dtype=np.float64)
    W0p = np.asarray(W0p, dtype=np.float64)
    G_P = np.asarray(G_P, dtype=np.float64)
    G_R = np.asarray(G_R, dtype=np.float64)
    U = x[:, perm_P]
    V = _block_apply(U, G_P, transpose=True)
    W = V @ W0p.T
    Z = _block_apply(W, G_R, transpose=True)
    Y = np.empty_like(Z)
    Y[:, perm_R] = Z
    return Y, U, V, W


def layer_backward(x, dy, W0p, G_P, G_R, perm_P, perm_R, U=None, W=None):
    """Gradients of <dY, Y> with W0' frozen.  Returns (dX, dG_P, dG_R).

    dZ = dY[:, p_R]; dW_j = dZ_j G_R,j; dG_R,j = dZ_j^T W_j; dV = dW W0';
    dU_j = dV_j G_P,j; dG_P,j = dV_j^T U_j; dX[:, p_P[i]] = dU[:, i].
    """
    x = np.asarray(x, dtype=np.float64)
    dy = np.asarray(dy, dtype=np.float64)
    W0p = np.asarray(W0p, dtype=np.float64)
    G_P = np.asarray(G_P, dtype=np.float64)
    G_R = np.asarray(G_R, dtype=np.float64)
    if U is None or W is None:
        _, U, _, W = layer_forward(x, W0p, G_P, G_R, perm_P, perm_R)
    nP, b, _ = G_P.shape
    nR = G_R.shape[0]
    dZ = dy[:, perm_R]
    dW = _block_apply(dZ, G_R, transpose=False)
    dG_R = np.stack([dZ[:, j * b:(j + 1) * b].T @ W[:, j * b:(j + 1) * b] for j in range(nR)])
    dV = dW @ W0p
    dU = _block_apply(dV, G_P, transpose=False)
    dG_P = np.stack([dV[:, j * b:(j + 1) * b].T @ U[:, j * b:(j + 1) * b] for j in range(nP)])
    dX = np.empty_like(dU)
    dX[:, perm_P] = dU
    return dX, dG_P, dG_R


def layer_forward_rows(x_rows, W0p, G_P, G_R, perm_P, perm_R):
    """Forward restricted to a subset of token rows (the layer is per-token)."""
    return layer_forward(x_rows, W0p, G_P, G_R, perm_P, perm_R)[0]


def layer_backward_dx_rows(dy_rows, W0p, G_P, G_R, perm_P, perm_R):
    """dX for a subset of token rows (dX is per-token and independent of X)."""
    dy = np.asarray(dy_rows, dtype=np.float64)
    dZ = dy[:, perm_R]
    dW = _block_apply(dZ, np.asarray(G_R, dtype=np.float64), transpose=False)
    dV = dW @ np.asarray(W0p, dtype=np.float64)
    dU = _block_apply(dV, np.asarray(G_P, dtype=np.float64), transpose=False)
    dX = np.empty_like(dU)
    dX[:, perm_P] = dU
    return dX


def full_step(x, W0, theta_P, theta_R, dy, perm_P, perm_R, b, k):
    """One pass of the whole path: merge, CNP forward (both sides), layer forward and
    backward, CNP backward.  Returns a dict of every output."""
    W0p = merge_perm(W0, perm_R, perm_P)
    G_P = cnp_forward(theta_P, b, k)
    G_R = cnp_forward(theta_R, b, k)
    Y, U, V, W = layer_forward(x, W0p, G_P, G_R, perm_P, perm_R)
    dX, dG_P, dG_R = layer_backward(x, dy, W0p, G_P, G_R, perm_P, perm_R, U=U, W=W)
    dth_P = cnp_backward(theta_P, dG_P, b, k)
    dth_R = cnp_backward(theta_R, dG_R, b, k)
    return dict(W0p=W0p, G_P=G_P, G_R=G_R, y=Y, dx=dX, dG_P=dG_P, dG_R=dG_R,
                dtheta_P=dth_P, dtheta_R=dth_R)


def layer_block_grads(x, dy, W0p, G_P, G_R, perm_P, perm_R, j_R, j_P):
    """dG_R,j_R and dG_P,j_P over all tokens, by their definitions, without forming the
    other blocks' gradients (for spot checks at full size):
        dG_R,j = dZ_j^T W_j   with W_j = V W0'[j-block rows]^T, V_i = U_i G_P,i^T
        dG_P,j = dV_j^T U_j   with dV_j = dW W0'[:, j-block],  dW_i = dZ_i G_R,i
    """
    x = np.asarray(x, dtype=np.float64)
    dy = np.asarray(dy, dtype=np.float64)
    W0p = np.asarray(W0p, dtype=np.float64)
    G_P = np.asarray(G_P, dtype=np.float64)
    G_R = np.asarray(G_R, dtype=np.float64)
    b = G_P.shape[1]
    U = x[:, perm_P]
    V = _block_apply(U, G_P, transpose=True)
    rs = slice(j_R * b, (j_R + 1) * b)
    W_j = V @ W0p[rs, :].T
    dZ = dy[:, perm_R]
    dG_R = dZ[:, rs].T @ W_j
    dW = _block_apply(dZ, G_R, transpose=False)
    ps = slice(j_P * b, (j_P + 1) * b)
    dV_j = dW @ W0p[:, ps]
    dG_P = dV_j.T @ U[:, ps]
    return dG_P, dG_R
