"""Float64 CPU oracle of the POET-X layer: CNP, forward, backward, merge.

TEST INFRASTRUCTURE ONLY.  Nothing in the CUDA library imports, links or calls this file, and
this file imports nothing from the library.  Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py`` (its CPU baseline and its ``--impl reference`` arm) may use it.

Everything is plain numpy float64, written for a reader to check against the pages by eye:
no blocking, fusion or reordering beyond what the definitions state.

Sources (web pages on POET-X; cited by page and section):
  [RR]  sai.science, "POET-X: Memory-efficient LLM Training by Scaling Orthogonal
        Transformation", SAI replication review (referee report): sections "Summary",
        "Weaknesses", "Reproducibility & code".
  [AD]  agidaily.cc, news article on POET-X (in Chinese): the section on fixing the base
        weight and training the two orthogonal transforms (W_RP = R . W0 . P), and the
        section on how POET-X changes the order of computation.
  [AB]  geekgo.top, the POET-X abstract (spectrum-preserving orthogonal equivalence).

Conventions (the pages leave them open; each is one plain reading, listed with the others in
the design notes):
  * tokens are rows: X [N, d_in], Y [N, d_out], Y = X (R W0 P)^T, i.e. y = R W0 P x per token;
  * P acts on the input side (d_in), R on the output side (d_out);
  * a permutation pi acts by gathering: (Pi a)_i = a_{pi(i)}, i.e. Pi = I[pi];
  * R = Pi_L^T BD_R Pi_L and P = Pi_R^T BD_P Pi_R, BD = blockdiag(Q_1, ..., Q_nb);
  * the skew block S has S[i, j] = theta[p] and S[j, i] = -theta[p] for i < j, with the
    strict upper triangle packed row by row: p = i*b - i(i+1)/2 + (j - i - 1);
  * CNP: Q = (I + S) (I + S + S^2 + ... + S^k), the Neumann truncation of the Cayley map
    (I + S)(I - S)^{-1}; its first-order form is I + 2S.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "packed_pairs", "packed_index", "unpack_skew", "pack_skew_grad", "cayley_exact",
    "cayley_neumann", "cnp", "block_diag", "perm_matrix", "absorb", "unabsorb",
    "dense_transforms", "dense_weight", "forward_dense", "backward_dense", "cnp_grad",
    "forward_chain", "backward_chain", "backward_chain_G", "merge", "adamw_step", "train_schedule",
    "quantize_rows", "dequantize_rows", "xq_merge",
]


# ----------------------------------------------------------------------------------------------
# Compact skew storage.  [RR] "Summary": the trainable skew blocks are stored as their upper
# triangle only; [RR] "Reproducibility & code", item "Partial coverage that does exist": the
# packed length per block is b*(b-1)/2.  [AD] article, same point (only the upper triangle of the
# skew-symmetric matrix is kept, and gradients/optimiser state shrink with it).
# ----------------------------------------------------------------------------------------------
def packed_index(i: int, j: int, b: int) -> int:
    """Position of S[i, j] (i < j) in the packed vector: row-major over the strict upper triangle."""
    assert 0 <= i < j < b
    return i * b - i * (i + 1) // 2 + (j - i - 1)


def packed_pairs(b: int):
    """(rows, cols) of the strict upper triangle in packed order (row-major over i < j)."""
    return np.triu_indices(b, k=1)


def unpack_skew(theta: np.ndarray, b: int) -> np.ndarray:
    """theta [nb, b(b-1)/2] -> skew blocks S [nb, b, b] with S = U - U^T, U strictly upper."""
    theta = np.asarray(theta, dtype=np.float64)
    nb = theta.shape[0]
    assert theta.shape[1] == b * (b - 1) // 2
    rows, cols = packed_pairs(b)
    S = np.zeros((nb, b, b), dtype=np.float64)
    S[:, rows, cols] = theta
    S[:, cols, rows] = -theta
    return S


def pack_skew_grad(G_S: np.ndarray) -> np.ndarray:
    """Gradient w.r.t. the packed parameters from the gradient w.r.t. an unconstrained S.

    theta[p] enters S at (i, j) with +1 and at (j, i) with -1, so dL/dtheta[p] = G_S[i,j] - G_S[j,i].
    """
    b = G_S.shape[-1]
    rows, cols = packed_pairs(b)
    return G_S[:, rows, cols] - G_S[:, cols, rows]


# ----------------------------------------------------------------------------------------------
# Cayley-Neumann parameterisation.  [RR] "Summary": R and P are parameterised by block-diagonal
# Cayley-Neumann orthogonalisation, and POET-X fuses the Cayley-Neumann series into one kernel
# (reusing Q and Q^2); [RR] "Reproducibility & code", item "Partial coverage that does exist":
# the shipped kernel matches the paper's Eq. 8/9 with k = 3.  [RR] "Weaknesses", item on the
# Cayley approximation: to first order the transform is I + 2Q (Q the skew parameter), which
# fixes the sign convention (I + S)(I - S)^{-1}.
# ----------------------------------------------------------------------------------------------
def cayley_exact(S: np.ndarray) -> np.ndarray:
    """C = (I + S)(I - S)^{-1}, computed by a linear solve ((I+S) and (I-S)^{-1} commute)."""
    b = S.shape[-1]
    I = np.eye(b)
    return np.linalg.solve(I - S, I + S)


def cayley_neumann(S: np.ndarray, k: int) -> np.ndarray:
    """Q = (I + S) * sum_{j=0..k} S^j: the Cayley map with (I - S)^{-1} truncated after S^k."""
    assert k >= 0
    b = S.shape[-1]
    I = np.broadcast_to(np.eye(b), S.shape)
    power = np.array(I, dtype=np.float64)
    series = np.array(I, dtype=np.float64)
    for _ in range(k):
        power = power @ S
        series = series + power
    return (I + S) @ series


def cnp(theta: np.ndarray, b: int, k: int) -> np.ndarray:
    """Packed skew parameters [nb, b(b-1)/2] -> orthogonal-ish blocks Q [nb, b, b]."""
    return cayley_neumann(unpack_skew(theta, b), k)


# ----------------------------------------------------------------------------------------------
# Dense definition.  [AD] article, section on fixing the base weight: W_RP = R . W0 . P with W0
# frozen and R, P trainable orthogonal transforms.  [RR] "Summary": R and P are block-diagonal
# in a randomly permuted basis; POET-X absorbs two of the four permutations into W in advance.
# ----------------------------------------------------------------------------------------------
def block_diag(Q: np.ndarray) -> np.ndarray:
    """[nb, b, b] -> the dense block-diagonal matrix blockdiag(Q_1, ..., Q_nb)."""
    nb, b, _ = Q.shape
    D = np.zeros((nb * b, nb * b), dtype=np.float64)
    for i in range(nb):
        D[i * b:(i + 1) * b, i * b:(i + 1) * b] = Q[i]
    return D


def perm_matrix(pi: np.ndarray) -> np.ndarray:
    """Gather-convention permutation matrix: (Pi a)_i = a_{pi(i)}, so Pi[i, pi(i)] = 1."""
    n = len(pi)
    Pm = np.zeros((n, n), dtype=np.float64)
    Pm[np.arange(n), np.asarray(pi)] = 1.0
    return Pm


def absorb(W0: np.ndarray, pi_L: np.ndarray, pi_R: np.ndarray) -> np.ndarray:
    """W0' = Pi_L W0 Pi_R^T, i.e. W0'[i, j] = W0[pi_L(i), pi_R(j)] (two permutations absorbed)."""
    return np.asarray(W0, np.float64)[np.asarray(pi_L)][:, np.asarray(pi_R)]


def unabsorb(W0p: np.ndarray, pi_L: np.ndarray, pi_R: np.ndarray) -> np.ndarray:
    """Inverse of absorb: W0 = Pi_L^T W0' Pi_R, i.e. W0[pi_L(i), pi_R(j)] = W0'[i, j]."""
    W0 = np.empty_like(np.asarray(W0p, np.float64))
    W0[np.ix_(np.asarray(pi_L), np.asarray(pi_R))] = W0p
    return W0


def dense_transforms(Q_R, Q_P, pi_L, pi_R):
    """R = Pi_L^T BD_R Pi_L (d_out x d_out) and P = Pi_R^T BD_P Pi_R (d_in x d_in)."""
    PL, PR = perm_matrix(pi_L), perm_matrix(pi_R)
    R = PL.T @ block_diag(Q_R) @ PL
    P = PR.T @ block_diag(Q_P) @ PR
    return R, P


def dense_weight(W0, Q_R, Q_P, pi_L, pi_R):
    """The materialised weight W = R W0 P (original basis)."""
    R, P = dense_transforms(Q_R, Q_P, pi_L, pi_R)
    return R @ np.asarray(W0, np.float64) @ P


def forward_dense(X, W0, theta_R, theta_P, pi_L, pi_R, b, k):
    """Y = X W^T with W = R W0 P built densely from the packed parameters."""
    W = dense_weight(W0, cnp(theta_R, b, k), cnp(theta_P, b, k), pi_L, pi_R)
    return np.asarray(X, np.float64) @ W.T


def cnp_grad(theta: np.ndarray, G: np.ndarray, b: int, k: int) -> np.ndarray:
    """Adjoint of the CNP: dL/dtheta (packed) from G = dL/dQ [nb, b, b].

    Differentiating Q = (I + S) N, N = sum_{j=0..k} S^j, and S^j = S...S:
        dQ = dS N + (I + S) sum_{j=1..k} sum_{a=0..j-1} S^a dS S^{j-1-a},
    so with T = S^T and H = (I + S)^T G = (I + T) G the gradient w.r.t. an unconstrained S is
        G_S = G N^T + sum_{j=1..k} sum_{a=0..j-1} T^a H T^{j-1-a},
    and the packed gradient is G_S[i, j] - G_S[j, i] (pack_skew_grad).
    """
    S = unpack_skew(theta, b)
    G = np.asarray(G, np.float64)
    nb = S.shape[0]
    I = np.eye(b)
    out = np.zeros((nb, b * (b - 1) // 2))
    for z in range(nb):
        Sz = S[z]
        T = Sz.T
        powers_S = [I]
        powers_T = [I]
        for _ in range(k):
            powers_S.append(powers_S[-1] @ Sz)
            powers_T.append(powers_T[-1] @ T)
        N = sum(powers_S)
        H = (I + T) @ G[z]
        GS = G[z] @ N.T
        for j in range(1, k + 1):
            for a in range(j):
                GS = GS + powers_T[a] @ H @ powers_T[j - 1 - a]
        out[z] = pack_skew_grad(GS[None])[0]
    return out


def _diag_blocks(M: np.ndarray, b: int) -> np.ndarray:
    nb = M.shape[0] // b
    return np.stack([M[i * b:(i + 1) * b, i * b:(i + 1) * b] for i in range(nb)])


def backward_dense(X, dY, W0, theta_R, theta_P, pi_L, pi_R, b, k):
    """Hand-derived adjoints of Y = X (R W0 P)^T; W0 is frozen (no dW0).

    dW = dY^T X;  dX = dY W;  dL/dR = dW (W0 P)^T;  dL/dP = (R W0)^T dW.
    R = Pi_L^T BD_R Pi_L, so dL/dBD_R = Pi_L (dL/dR) Pi_L^T and G_R,i is its i-th diagonal block
    (likewise G_P,i with Pi_R); the CNP adjoint then gives the packed gradients.
    Returns (dX, g_theta_R, g_theta_P).
    """
    X = np.asarray(X, np.float64)
    dY = np.asarray(dY, np.float64)
    W0 = np.asarray(W0, np.float64)
    Q_R, Q_P = cnp(theta_R, b, k), cnp(theta_P, b, k)
    R, P = dense_transforms(Q_R, Q_P, pi_L, pi_R)
    W = R @ W0 @ P
    dW = dY.T @ X
    dX = dY @ W
    dR = dW @ (W0 @ P).T
    dP = (R @ W0).T @ dW
    PL, PR = perm_matrix(pi_L), perm_matrix(pi_R)
    G_R = _diag_blocks(PL @ dR @ PL.T, b)
    G_P = _diag_blocks(PR @ dP @ PR.T, b)
    return dX, cnp_grad(theta_R, G_R, b, k), cnp_grad(theta_P, G_P, b, k)


# ----------------------------------------------------------------------------------------------
# Input-centric chain (second route).  [RR] "Summary": POET-X evaluates R W P x as a matrix-free
# chain of transforms on the activations, applies the block-diagonal factors as a batch of
# per-block matmuls that never builds the sparse matrix, and keeps two permutations outside W.
# [RR] "Weaknesses", item on notation gaps: the simplified forward is stated as a product of
# G-factors, W and x, with shapes left open; the reading here is the one above.
# ----------------------------------------------------------------------------------------------
def forward_chain(X, W0p, Q_R, Q_P, pi_L, pi_R):
    """y = Pi_L^T BD_R W0' BD_P Pi_R x, evaluated on the activations.

    Returns (Y, U, V, Z, Yp): U = X[:, pi_R]; V[:, blk] = U[:, blk] Q_P,blk^T; Z = V W0'^T;
    Yp[:, blk] = Z[:, blk] Q_R,blk^T; Y[:, pi_L] = Yp.
    """
    X = np.asarray(X, np.float64)
    W0p = np.asarray(W0p, np.float64)
    b = Q_P.shape[-1]
    U = X[:, np.asarray(pi_R)]
    V = np.empty_like(U)
    for i in range(Q_P.shape[0]):
        V[:, i * b:(i + 1) * b] = U[:, i * b:(i + 1) * b] @ Q_P[i].T
    Z = V @ W0p.T
    Yp = np.empty_like(Z)
    for i in range(Q_R.shape[0]):
        Yp[:, i * b:(i + 1) * b] = Z[:, i * b:(i + 1) * b] @ Q_R[i].T
    Y = np.empty_like(Yp)
    Y[:, np.asarray(pi_L)] = Yp
    return Y, U, V, Z, Yp


def backward_chain(X, dY, W0p, theta_R, theta_P, pi_L, pi_R, b, k):
    """Adjoint of forward_chain, step by step.  Returns (dX, g_theta_R, g_theta_P).

    dYp = dY[:, pi_L]; G_R,i = dYp_i^T Z_i; dZ_i = dYp_i Q_R,i; dV = dZ W0';
    G_P,i = dV_i^T U_i; dU_i = dV_i Q_P,i; dX[:, pi_R] = dU; then the CNP adjoint.
    """
    Q_R, Q_P = cnp(theta_R, b, k), cnp(theta_P, b, k)
    dX, G_R, G_P = backward_chain_G(X, dY, W0p, Q_R, Q_P, pi_L, pi_R, b)
    return dX, cnp_grad(theta_R, G_R, b, k), cnp_grad(theta_P, G_P, b, k)


def backward_chain_G(X, dY, W0p, Q_R, Q_P, pi_L, pi_R, b):
    """The activation part of backward_chain: (dX, G_R, G_P) with G = dL/dQ per block, before
    the CNP adjoint."""
    _, U, _, Z, _ = forward_chain(X, W0p, Q_R, Q_P, pi_L, pi_R)
    dY = np.asarray(dY, np.float64)
    W0p = np.asarray(W0p, np.float64)
    dYp = dY[:, np.asarray(pi_L)]
    G_R = np.empty_like(Q_R)
    dZ = np.empty_like(Z)
    for i in range(Q_R.shape[0]):
        blk = slice(i * b, (i + 1) * b)
        G_R[i] = dYp[:, blk].T @ Z[:, blk]
        dZ[:, blk] = dYp[:, blk] @ Q_R[i]
    dV = dZ @ W0p
    G_P = np.empty_like(Q_P)
    dU = np.empty_like(U)
    for i in range(Q_P.shape[0]):
        blk = slice(i * b, (i + 1) * b)
        G_P[i] = dV[:, blk].T @ U[:, blk]
        dU[:, blk] = dV[:, blk] @ Q_P[i]
    dX = np.empty_like(dU)
    dX[:, np.asarray(pi_R)] = dU
    return dX, G_R, G_P


# ----------------------------------------------------------------------------------------------
# Merge-then-reinitialise.  [AD] article, section on fixing the base weight: during training the
# transforms are periodically merged into the weight and re-initialised; [RR] "Reproducibility &
# code" names merge_then_reinitialize and notes that the 4-permutation path is baked into it.
# Reading: the Neumann Q used by the forward pass is what is merged (so the layer function is
# unchanged), theta is reset to zero and fresh permutations are absorbed.
# ----------------------------------------------------------------------------------------------
def merge(W0p, theta_R, theta_P, pi_L, pi_R, pi_L_new, pi_R_new, b, k):
    """Returns (W0'_new, theta_R_new, theta_P_new) with W0'_new = absorb(R W0 P, new perms)."""
    W0 = unabsorb(W0p, pi_L, pi_R)
    W_full = dense_weight(W0, cnp(theta_R, b, k), cnp(theta_P, b, k), pi_L, pi_R)
    return (absorb(W_full, pi_L_new, pi_R_new),
            np.zeros_like(np.asarray(theta_R, np.float64)),
            np.zeros_like(np.asarray(theta_P, np.float64)))


# ------------------------------------------------------------------ optimiser on packed theta
# The trainable state is the packed theta, so the optimiser state lives at the packed size too
# ([AD], the section on compact storage: gradients and optimiser state shrink with it).  The
# pages name AdamW as the baseline optimiser and give the POET learning-rate scale gamma = 0.5
# and the reset gap of 400 steps ([RR] "Weaknesses"), but not AdamW's own constants; those are
# arguments here.  AdamW is the decoupled-weight-decay Adam (Loshchilov and Hutter): with
# step t >= 1 and eta = gamma * lr,
#   m <- beta1 m + (1 - beta1) g,   v <- beta2 v + (1 - beta2) g^2,
#   theta <- theta - eta * (lam * theta + (m / (1 - beta1^t)) / (sqrt(v / (1 - beta2^t)) + eps)),
# the decay acting on the theta before this step.
def adamw_step(theta, grad, m, v, t, lr, gamma=0.5, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.0):
    """One AdamW step on packed parameters; returns (theta, m, v) in float64."""
    theta = np.asarray(theta, np.float64)
    g = np.asarray(grad, np.float64)
    m = beta1 * np.asarray(m, np.float64) + (1.0 - beta1) * g
    v = beta2 * np.asarray(v, np.float64) + (1.0 - beta2) * g * g
    m_hat = m / (1.0 - beta1 ** t)
    v_hat = v / (1.0 - beta2 ** t)
    eta = gamma * lr
    theta = theta - eta * (weight_decay * theta + m_hat / (np.sqrt(v_hat) + eps))
    return theta, m, v


def train_schedule(n_steps, reset_gap=400):
    """What happens after each training step s = 1..n_steps of the merge schedule: a list of
    (s, t, merge) with t the AdamW step count used at s and merge True when step s is followed
    by merge-then-reinitialise.  Reading of the pages' reset gap: after every reset_gap steps
    the transforms are merged and theta is zeroed; the moments of theta restart with it (they
    belonged to the parameters that were folded away), so t counts from 1 again."""
    out, t = [], 0
    for s in range(1, n_steps + 1):
        t += 1
        merge_now = s % reset_gap == 0
        out.append((s, t, merge_now))
        if merge_now:
            t = 0
    return out


# ----------------------------------------------------------------- POET-XQ: 8-bit resident W0'
# [RR] "Summary": a quantised variant, POET-XQ, is possible because POET-Xmem never keeps a
# high-precision weight resident; [RR] "Strengths": it is implemented through POET-Xmem (the
# recompute means the dequantised W is never stored) and compared with 8-bit Q-GaLore and
# Q-APOLLO; [AD], the section on how POET-X differs from existing methods: POET-X has a
# quantised version, POET-XQ.  The pages give no format.  Reading: W0' is held as int8 codes
# with one scale per row (symmetric, absmax): s_o = max_i |W0'[o, i]| / 127 and
# q[o, i] = round(W0'[o, i] / s_o) to nearest, ties to even, clipped to [-127, 127]; a row of
# zeros gets s_o = 0 and q = 0.  The layer is the POET-Xmem layer with W0' = s * q.  Since the
# codes are integers decided by floating point, the scale and the division are taken in float32
# (the precision in which the library decides them too).
def quantize_rows(W0p):
    """W0' [d_out, d_in] -> (q int8 [d_out, d_in], s float32 [d_out]), per-row symmetric absmax."""
    W = np.asarray(W0p, np.float32)
    amax = np.max(np.abs(W), axis=1)
    s = (amax / np.float32(127.0)).astype(np.float32)
    q = np.zeros(W.shape, np.int8)
    live = s > 0
    codes = np.rint(W[live] / s[live, None])  # float32 division, round half to even
    q[live] = np.clip(codes, -127, 127).astype(np.int8)
    return q, s


def dequantize_rows(q, s):
    """The POET-XQ weight: W0'[o, i] = s_o * q[o, i] (float64)."""
    return np.asarray(s, np.float64)[:, None] * np.asarray(q, np.float64)


def xq_merge(q, s, theta_R, theta_P, pi_L, pi_R, pi_L_new, pi_R_new, b, k):
    """Merge of the POET-XQ layer: the POET-X merge of W0' = s * q, then the new W0' quantised
    again.  Returns (W0'_new before quantisation, q_new, s_new, theta_R_new, theta_P_new)."""
    Wn, tR, tP = merge(dequantize_rows(q, s), theta_R, theta_P, pi_L, pi_R, pi_L_new, pi_R_new, b, k)
    qn, sn = quantize_rows(Wn)
    return Wn, qn, sn, tR, tP
