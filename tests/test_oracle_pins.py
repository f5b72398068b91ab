"""Pins for the float64 oracle: closed forms, invariants, brute force and hand-derived fixtures.

Nothing here re-types an oracle formula: each check comes from an independent fact (a closed
form, an invariant of orthogonal maps, finite differences, exhaustive enumeration, or a value
derived by hand in tests/golden/).  ``test_planted_mistakes_are_caught`` plants plausible slips
into a copy of the oracle and checks that the pins notice them.
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _rand_layer(rng, d_in, d_out, b, n, scale=0.3):
    nb_in, nb_out, p = d_in // b, d_out // b, b * (b - 1) // 2
    return dict(
        X=rng.standard_normal((n, d_in)), dY=rng.standard_normal((n, d_out)),
        W0=rng.standard_normal((d_out, d_in)) / np.sqrt(d_in),
        theta_R=scale * rng.standard_normal((nb_out, p)), theta_P=scale * rng.standard_normal((nb_in, p)),
        pi_L=rng.permutation(d_out), pi_R=rng.permutation(d_in))


def _rel(a, b):
    return np.linalg.norm(np.asarray(a) - np.asarray(b)) / max(np.linalg.norm(np.asarray(b)), 1e-300)


# ---------------------------------------------------------------------------------------------
# Packing and permutations (bit-exact, brute force)
# ---------------------------------------------------------------------------------------------
@pytest.mark.parametrize("b", [2, 3, 4, 5, 8])
def test_packed_index_brute_force(b):
    counter = 0
    rows, cols = O.packed_pairs(b)
    for i in range(b):
        for j in range(i + 1, b):
            assert O.packed_index(i, j, b) == counter
            assert rows[counter] == i and cols[counter] == j
            counter += 1
    assert counter == b * (b - 1) // 2 == len(rows)


def test_unpack_fixture_b4():
    g = _load("packing_b4.json")
    S = O.unpack_skew(np.array([g["theta"]], dtype=np.float64), g["b"])[0]
    assert np.array_equal(S, np.array(g["S"], dtype=np.float64))


def test_unpack_skew_and_pack():
    rng = np.random.default_rng(0)
    theta = rng.standard_normal((3, 28))
    S = O.unpack_skew(theta, 8)
    assert np.array_equal(S, -np.transpose(S, (0, 2, 1)))
    assert np.all(np.diagonal(S, axis1=1, axis2=2) == 0)
    # theta enters S twice (+ above, - below), so the packed gradient of <S, S>/2 w.r.t. theta
    # (= pack of S itself) is 2 theta.
    assert np.array_equal(O.pack_skew_grad(S), 2 * theta)


def test_perm_matrix_gather_convention():
    pi = np.array([2, 0, 3, 1])
    a = np.array([10.0, 11.0, 12.0, 13.0])
    assert np.array_equal(O.perm_matrix(pi) @ a, a[pi])
    W = np.arange(12.0).reshape(3, 4)
    pl, pr = np.array([1, 2, 0]), np.array([3, 1, 0, 2])
    Wp = O.absorb(W, pl, pr)
    for i in range(3):
        for j in range(4):
            assert Wp[i, j] == W[pl[i], pr[j]]
    assert np.array_equal(O.unabsorb(Wp, pl, pr), W)


# ---------------------------------------------------------------------------------------------
# Cayley and Cayley-Neumann
# ---------------------------------------------------------------------------------------------
def test_cnp_golden_b2():
    g = _load("cnp_b2_theta_half.json")
    theta = np.array([g["theta"]])
    S = O.unpack_skew(theta, 2)
    assert np.allclose(O.cayley_exact(S)[0], g["cayley_exact"], atol=1e-15, rtol=0)
    for k, Qk in g["neumann"].items():
        assert np.allclose(O.cnp(theta, 2, int(k))[0], Qk, atol=1e-15, rtol=0), k


def test_cnp_grad_golden_b2():
    g = _load("cnp_b2_theta_half.json")
    theta = np.array([g["theta"]])
    G = np.array([g["G"]])
    for k, expect in g["packed_grad"].items():
        assert np.allclose(O.cnp_grad(theta, G, 2, int(k))[0], expect, atol=1e-14, rtol=0), k


@pytest.mark.parametrize("b", [4, 16, 33])
def test_cayley_exact_orthogonal(b):
    rng = np.random.default_rng(b)
    S = O.unpack_skew(0.4 * rng.standard_normal((3, b * (b - 1) // 2)), b)
    C = O.cayley_exact(S)
    for c in C:
        assert np.abs(c.T @ c - np.eye(b)).max() <= 1e-12
        assert abs(np.linalg.det(c) - 1.0) <= 1e-10


@pytest.mark.parametrize("k", [0, 1, 2, 3, 4, 7])
def test_neumann_closed_form(k):
    # All factors are functions of S, so they commute: (I+S) sum_{j<=k} S^j = C (I - S^{k+1}).
    b = 12
    rng = np.random.default_rng(100 + k)
    S = O.unpack_skew(0.05 * rng.standard_normal((2, b * (b - 1) // 2)), b)
    C = O.cayley_exact(S)
    Q = O.cayley_neumann(S, k)
    I = np.eye(b)
    for z in range(2):
        Sk1 = np.linalg.matrix_power(S[z], k + 1)
        assert np.abs(Q[z] - C[z] @ (I - Sk1)).max() <= 1e-13
        # S is normal, so ||Q_k - C||_2 = ||S^{k+1}||_2 = ||S||_2^{k+1}.
        s = np.linalg.norm(S[z], 2)
        assert abs(np.linalg.norm(Q[z] - C[z], 2) - s ** (k + 1)) <= 1e-12 * max(1.0, s ** (k + 1)) + 1e-15
        # Q^T Q - I = -2 S^{k+1} + S^{2k+2} (k odd), -S^{2k+2} (k even).
        S2k2 = np.linalg.matrix_power(S[z], 2 * k + 2)
        expect = (-2 * Sk1 + S2k2) if k % 2 == 1 else -S2k2
        assert np.abs(Q[z].T @ Q[z] - I - expect).max() <= 1e-13


def test_neumann_deviation_shrinks_with_k():
    b = 16
    rng = np.random.default_rng(7)
    S = O.unpack_skew(0.08 * rng.standard_normal((1, b * (b - 1) // 2)), b)
    assert np.linalg.norm(S[0], 2) < 1
    C = O.cayley_exact(S)[0]
    Qs = [O.cayley_neumann(S, k)[0] for k in range(10)]
    # Distance to the exact Cayley map, ||S||_2^{k+1}, shrinks strictly with k.
    dist = [np.linalg.norm(Q - C, 2) for Q in Qs]
    assert all(dist[i + 1] < dist[i] for i in range(9))
    # The orthogonality defect Q^T Q - I is -2S^{k+1}+S^{2k+2} (odd k) or -S^{2k+2} (even k), so
    # it shrinks along each parity class of k but is NOT monotone across parities (k=2 < k=3).
    defect = [np.linalg.norm(Q.T @ Q - np.eye(b)) for Q in Qs]
    assert all(defect[i + 2] < defect[i] for i in range(8))
    assert defect[2] < defect[3]


def test_cnp_special_cases():
    b = 8
    rng = np.random.default_rng(3)
    theta = 0.1 * rng.standard_normal((2, 28))
    # S = 0 gives exactly I for any k.
    for k in range(5):
        assert np.array_equal(O.cnp(np.zeros((2, 28)), b, k), np.broadcast_to(np.eye(b), (2, b, b)))
    # k = 0 gives I + S.
    assert np.allclose(O.cnp(theta, b, 0), np.eye(b) + O.unpack_skew(theta, b), atol=1e-15)
    # First order: Q(eps S) = I + 2 eps S + O(eps^2), and the eps^2 coefficient is 2 S^2 for k >= 2.
    S = O.unpack_skew(theta, b)
    for eps in (1e-3, 1e-4):
        Q = O.cayley_neumann(eps * S, 3)
        r = (Q - np.eye(b) - 2 * eps * S) / eps ** 2
        assert np.abs(r - 2 * S @ S).max() <= 10 * eps * np.abs(S).max() ** 3 * 8


# ---------------------------------------------------------------------------------------------
# The layer: spectrum, two routes, special cases
# ---------------------------------------------------------------------------------------------
def test_spectrum_preserved_with_exact_cayley():
    rng = np.random.default_rng(11)
    L = _rand_layer(rng, 24, 16, 4, 3)
    C_R = O.cayley_exact(O.unpack_skew(L["theta_R"], 4))
    C_P = O.cayley_exact(O.unpack_skew(L["theta_P"], 4))
    W = O.dense_weight(L["W0"], C_R, C_P, L["pi_L"], L["pi_R"])
    s0 = np.linalg.svd(L["W0"], compute_uv=False)
    s1 = np.linalg.svd(W, compute_uv=False)
    assert np.abs(s0 - s1).max() <= 1e-10


@pytest.mark.parametrize("k", [0, 1, 3])
def test_forward_two_routes(k):
    rng = np.random.default_rng(20 + k)
    b = 4
    L = _rand_layer(rng, 24, 16, b, 5)
    Y_dense = O.forward_dense(L["X"], L["W0"], L["theta_R"], L["theta_P"], L["pi_L"], L["pi_R"], b, k)
    W0p = O.absorb(L["W0"], L["pi_L"], L["pi_R"])
    Y_chain = O.forward_chain(L["X"], W0p, O.cnp(L["theta_R"], b, k), O.cnp(L["theta_P"], b, k),
                              L["pi_L"], L["pi_R"])[0]
    assert _rel(Y_chain, Y_dense) <= 1e-12


def test_batched_block_diag_equals_dense_block_diag():
    rng = np.random.default_rng(5)
    b, nb, n = 4, 6, 7
    Q = O.cnp(0.3 * rng.standard_normal((nb, 6)), b, 3)
    U = rng.standard_normal((n, nb * b))
    V = np.empty_like(U)
    for i in range(nb):
        V[:, i * b:(i + 1) * b] = U[:, i * b:(i + 1) * b] @ Q[i].T
    assert np.abs(V - U @ O.block_diag(Q).T).max() <= 1e-14


def test_forward_theta_zero_is_plain_matmul():
    rng = np.random.default_rng(6)
    L = _rand_layer(rng, 16, 8, 4, 3)
    z_R, z_P = np.zeros_like(L["theta_R"]), np.zeros_like(L["theta_P"])
    Y = O.forward_dense(L["X"], L["W0"], z_R, z_P, L["pi_L"], L["pi_R"], 4, 3)
    assert np.abs(Y - L["X"] @ L["W0"].T).max() <= 1e-13
    dX, gR, gP = O.backward_dense(L["X"], L["dY"], L["W0"], z_R, z_P, L["pi_L"], L["pi_R"], 4, 3)
    assert np.abs(dX - L["dY"] @ L["W0"]).max() <= 1e-13


def test_forward_single_block_identity_perm():
    # b = d and identity permutations: Y = X (Q_R W0 Q_P)^T.
    rng = np.random.default_rng(8)
    d, n = 6, 4
    th_R, th_P = 0.2 * rng.standard_normal((1, 15)), 0.2 * rng.standard_normal((1, 15))
    W0, X = rng.standard_normal((d, d)), rng.standard_normal((n, d))
    idp = np.arange(d)
    Q_R, Q_P = O.cnp(th_R, d, 3)[0], O.cnp(th_P, d, 3)[0]
    Y = O.forward_dense(X, W0, th_R, th_P, idp, idp, d, 3)
    assert np.abs(Y - X @ (Q_R @ W0 @ Q_P).T).max() <= 1e-13


# ---------------------------------------------------------------------------------------------
# Gradients
# ---------------------------------------------------------------------------------------------
def _loss(X, dY, W0, tR, tP, pL, pR, b, k):
    return float(np.sum(dY * O.forward_dense(X, W0, tR, tP, pL, pR, b, k)))


@pytest.mark.parametrize("k", [0, 1, 2, 3, 5])
def test_gradients_central_differences(k):
    rng = np.random.default_rng(40 + k)
    b = 4
    L = _rand_layer(rng, 16, 8, b, 3)
    args = (L["W0"], L["theta_R"], L["theta_P"], L["pi_L"], L["pi_R"], b, k)
    dX, gR, gP = O.backward_dense(L["X"], L["dY"], *args)
    h = 1e-6
    for name, g in (("theta_R", gR), ("theta_P", gP)):
        fd = np.zeros_like(g)
        for idx in np.ndindex(g.shape):
            tp, tm = dict(L), dict(L)
            tp[name] = L[name].copy(); tp[name][idx] += h
            tm[name] = L[name].copy(); tm[name][idx] -= h
            lp = _loss(tp["X"], tp["dY"], tp["W0"], tp["theta_R"], tp["theta_P"], tp["pi_L"], tp["pi_R"], b, k)
            lm = _loss(tm["X"], tm["dY"], tm["W0"], tm["theta_R"], tm["theta_P"], tm["pi_L"], tm["pi_R"], b, k)
            fd[idx] = (lp - lm) / (2 * h)
        assert _rel(g, fd) <= 1e-7, name
    fdX = np.zeros_like(dX)
    for idx in np.ndindex(dX.shape):
        Xp, Xm = L["X"].copy(), L["X"].copy()
        Xp[idx] += h
        Xm[idx] -= h
        fdX[idx] = (_loss(Xp, L["dY"], *args) - _loss(Xm, L["dY"], *args)) / (2 * h)
    assert _rel(dX, fdX) <= 1e-7


def test_backward_two_routes():
    rng = np.random.default_rng(50)
    b = 4
    L = _rand_layer(rng, 24, 16, b, 6)
    W0p = O.absorb(L["W0"], L["pi_L"], L["pi_R"])
    d1 = O.backward_dense(L["X"], L["dY"], L["W0"], L["theta_R"], L["theta_P"], L["pi_L"], L["pi_R"], b, 3)
    d2 = O.backward_chain(L["X"], L["dY"], W0p, L["theta_R"], L["theta_P"], L["pi_L"], L["pi_R"], b, 3)
    for a, c in zip(d1, d2):
        assert _rel(c, a) <= 1e-11


@pytest.mark.parametrize("k", [0, 1, 3])
def test_cnp_grad_at_zero_closed_form(k):
    rng = np.random.default_rng(60 + k)
    b = 6
    G = rng.standard_normal((2, b, b))
    g = O.cnp_grad(np.zeros((2, 15)), G, b, k)
    r, c = np.triu_indices(b, 1)
    expect = (1 if k == 0 else 2) * (G[:, r, c] - G[:, c, r])
    assert np.abs(g - expect).max() <= 1e-14


def test_cnp_grad_directional_finite_difference():
    rng = np.random.default_rng(70)
    b, k = 16, 3
    theta = 0.1 * rng.standard_normal((2, 120))
    G = rng.standard_normal((2, b, b))
    E = rng.standard_normal((2, 120))
    g = O.cnp_grad(theta, G, b, k)
    h = 1e-6
    dQ = (O.cnp(theta + h * E, b, k) - O.cnp(theta - h * E, b, k)) / (2 * h)
    assert abs(np.sum(G * dQ) - np.sum(g * E)) <= 1e-8 * abs(np.sum(g * E))


# ---------------------------------------------------------------------------------------------
# Merge
# ---------------------------------------------------------------------------------------------
def test_merge_preserves_layer_function():
    rng = np.random.default_rng(80)
    b = 4
    L = _rand_layer(rng, 16, 12, b, 5)
    W0p = O.absorb(L["W0"], L["pi_L"], L["pi_R"])
    pL2, pR2 = rng.permutation(12), rng.permutation(16)
    Wn, tR, tP = O.merge(W0p, L["theta_R"], L["theta_P"], L["pi_L"], L["pi_R"], pL2, pR2, b, 3)
    assert np.all(tR == 0) and np.all(tP == 0)
    Y_before = O.forward_dense(L["X"], L["W0"], L["theta_R"], L["theta_P"], L["pi_L"], L["pi_R"], b, 3)
    Y_after = O.forward_chain(L["X"], Wn, O.cnp(tR, b, 3), O.cnp(tP, b, 3), pL2, pR2)[0]
    assert _rel(Y_after, Y_before) <= 1e-12


def test_merge_identity():
    rng = np.random.default_rng(81)
    L = _rand_layer(rng, 8, 8, 4, 2)
    W0p = O.absorb(L["W0"], L["pi_L"], L["pi_R"])
    z = np.zeros_like(L["theta_R"])
    Wn, _, _ = O.merge(W0p, z, z, L["pi_L"], L["pi_R"], L["pi_L"], L["pi_R"], 4, 3)
    assert np.abs(Wn - W0p).max() <= 1e-15


# ---------------------------------------------------------------------------------------------
# Planted mistakes: a copy of the oracle with a plausible slip must fail at least one pin.
# ---------------------------------------------------------------------------------------------
def _pins_pass(mod):
    rng = np.random.default_rng(90)
    b, k = 4, 3
    L = _rand_layer(rng, 16, 8, b, 3)
    ok = True
    g = _load("cnp_b2_theta_half.json")
    th = np.array([g["theta"]])
    ok &= np.allclose(mod.cnp(th, 2, 3)[0], g["neumann"]["3"], atol=1e-14)
    ok &= np.allclose(mod.cnp_grad(th, np.array([g["G"]]), 2, 3)[0], g["packed_grad"]["3"], atol=1e-12)
    p = _load("packing_b4.json")
    ok &= np.array_equal(mod.unpack_skew(np.array([p["theta"]], float), 4)[0], np.array(p["S"], float))
    W0p = mod.absorb(L["W0"], L["pi_L"], L["pi_R"])
    Yd = mod.forward_dense(L["X"], L["W0"], L["theta_R"], L["theta_P"], L["pi_L"], L["pi_R"], b, k)
    Yc = mod.forward_chain(L["X"], W0p, mod.cnp(L["theta_R"], b, k), mod.cnp(L["theta_P"], b, k),
                           L["pi_L"], L["pi_R"])[0]
    ok &= _rel(Yc, Yd) <= 1e-12
    dX, gR, gP = mod.backward_chain(L["X"], L["dY"], W0p, L["theta_R"], L["theta_P"], L["pi_L"], L["pi_R"], b, k)
    h = 1e-6
    idx = (0, 2)
    tp, tm = L["theta_R"].copy(), L["theta_R"].copy()
    tp[idx] += h
    tm[idx] -= h
    fd = (np.sum(L["dY"] * mod.forward_dense(L["X"], L["W0"], tp, L["theta_P"], L["pi_L"], L["pi_R"], b, k))
          - np.sum(L["dY"] * mod.forward_dense(L["X"], L["W0"], tm, L["theta_P"], L["pi_L"], L["pi_R"], b, k))) / (2 * h)
    ok &= abs(gR[idx] - fd) <= 1e-6 * max(1.0, abs(fd))
    return bool(ok)


def test_planted_mistakes_are_caught():
    import importlib
    import types
    src_path = os.path.join(os.path.dirname(O.__file__), "poetx_ref.py")
    with open(src_path) as f:
        src = f.read()

    def variant(old, new):
        assert old in src, old
        m = types.ModuleType("oracle_variant")
        exec(compile(src.replace(old, new, 1), "oracle_variant", "exec"), m.__dict__)
        return m

    base = types.ModuleType("oracle_base")
    exec(compile(src, "oracle_base", "exec"), base.__dict__)
    assert _pins_pass(base)
    mistakes = [
        ("S[:, cols, rows] = -theta", "S[:, cols, rows] = theta"),                 # lost skew sign
        ("return (I + S) @ series", "return (I - S) @ series"),                   # wrong Cayley sign
        ("for _ in range(k):\n        power = power @ S", "for _ in range(k - 1):\n        power = power @ S"),  # dropped term
        ("H = (I + T) @ G[z]", "H = G[z]"),                                       # dropped (I+T) factor
        ("GS = G[z] @ N.T", "GS = G[z] @ N"),                                      # transposed operand
        ("V[:, i * b:(i + 1) * b] = U[:, i * b:(i + 1) * b] @ Q_P[i].T",
         "V[:, i * b:(i + 1) * b] = U[:, i * b:(i + 1) * b] @ Q_P[i]"),             # transposed block
        ("Y[:, np.asarray(pi_L)] = Yp", "Y[:] = Yp[:, np.asarray(pi_L)]"),        # gather instead of scatter
        ("return G_S[:, rows, cols] - G_S[:, cols, rows]", "return G_S[:, rows, cols]"),  # half of the pack
    ]
    for old, new in mistakes:
        assert not _pins_pass(variant(old, new)), new


def test_absorb_equals_permutation_matrix_product():
    rng = np.random.default_rng(12)
    W = rng.standard_normal((6, 10))
    pl, pr = rng.permutation(6), rng.permutation(10)
    assert np.array_equal(O.absorb(W, pl, pr), O.perm_matrix(pl) @ W @ O.perm_matrix(pr).T)
    assert np.array_equal(O.unabsorb(O.absorb(W, pl, pr), pl, pr), W)


# ------------------------------------------------------------- optimiser on packed theta
def test_adamw_first_step_is_the_closed_form():
    # From zero moments the bias-corrected moments are g and g^2, so the step is
    # -gamma*lr*(lam*theta + g/(|g| + eps)).
    rng = np.random.default_rng(3)
    th, g = rng.normal(size=1000), rng.normal(size=1000)
    lr, gamma, lam, eps = 1e-3, 0.5, 0.1, 1e-8
    th1, m1, v1 = O.adamw_step(th, g, np.zeros(1000), np.zeros(1000), 1, lr, gamma, 0.9, 0.999, eps, lam)
    np.testing.assert_allclose(th1, th - gamma * lr * (lam * th + g / (np.abs(g) + eps)), rtol=0, atol=1e-15)
    np.testing.assert_allclose(m1, 0.1 * g, rtol=1e-15)
    np.testing.assert_allclose(v1, 0.001 * g * g, rtol=1e-12)


def test_adamw_constant_gradient_moves_linearly_and_decay_alone_is_geometric():
    # A constant gradient keeps the corrected moments at g and g^2 exactly at every step.
    g = np.array([0.5, -2.0, 3e-3])
    th, m, v = np.zeros(3), np.zeros(3), np.zeros(3)
    for t in range(1, 8):
        th, m, v = O.adamw_step(th, g, m, v, t, 0.01, 0.5)
    np.testing.assert_allclose(th, -7 * 0.5 * 0.01 * g / (np.abs(g) + 1e-8), rtol=1e-10)
    # Zero gradient, weight decay only: theta shrinks by (1 - gamma*lr*lam) per step.
    th = np.array([1.0, -3.0])
    m = v = np.zeros(2)
    for t in range(1, 6):
        th, m, v = O.adamw_step(th, np.zeros(2), m, v, t, 0.1, 0.5, weight_decay=0.2)
    np.testing.assert_allclose(th, np.array([1.0, -3.0]) * (1 - 0.5 * 0.1 * 0.2) ** 5, rtol=1e-14)


def test_adamw_matches_the_library_optimiser():
    # torch.optim.AdamW (CPU, float64) with lr = gamma * lr is the same algorithm.
    rng = np.random.default_rng(11)
    th0 = rng.normal(size=257)
    p = torch.nn.Parameter(torch.tensor(th0, dtype=torch.float64))
    opt = torch.optim.AdamW([p], lr=0.5 * 2e-3, betas=(0.85, 0.99), eps=1e-6, weight_decay=0.05)
    th, m, v = th0.copy(), np.zeros(257), np.zeros(257)
    for t in range(1, 13):
        g = rng.normal(size=257) * (1 + t)
        p.grad = torch.tensor(g, dtype=torch.float64)
        opt.step()
        th, m, v = O.adamw_step(th, g, m, v, t, 2e-3, 0.5, 0.85, 0.99, 1e-6, 0.05)
    np.testing.assert_allclose(th, p.detach().numpy(), rtol=0, atol=1e-14)


def test_adamw_planted_mistakes_are_caught():
    # Each slip below changes the constant-gradient trajectory or the library comparison.
    g = np.array([0.5, -2.0])
    def run(step):
        th, m, v = np.zeros(2), np.zeros(2), np.zeros(2)
        for t in range(1, 6):
            th, m, v = step(th, g, m, v, t)
        return th
    ref = -5 * 0.5 * 0.01 * g / (np.abs(g) + 1e-8)
    def no_bias_correction(th, g, m, v, t):
        m = 0.9 * m + 0.1 * g; v = 0.999 * v + 0.001 * g * g
        return th - 0.005 * m / (np.sqrt(v) + 1e-8), m, v
    def eps_inside_sqrt(th, g, m, v, t):
        m = 0.9 * m + 0.1 * g; v = 0.999 * v + 0.001 * g * g
        return th - 0.005 * (m / (1 - 0.9 ** t)) / np.sqrt(v / (1 - 0.999 ** t) + 1e-2), m, v
    def no_gamma(th, g, m, v, t):
        return O.adamw_step(th, g, m, v, t, 0.01, 1.0)
    for slip in (no_bias_correction, eps_inside_sqrt, no_gamma):
        assert not np.allclose(run(slip), ref, rtol=1e-6), slip.__name__
    assert np.allclose(run(lambda th, g, m, v, t: O.adamw_step(th, g, m, v, t, 0.01, 0.5)), ref, rtol=1e-10)


def test_merge_schedule_resets_every_gap():
    sch = O.train_schedule(1000, reset_gap=400)
    assert [s for s, _, mg in sch if mg] == [400, 800]
    assert [t for s, t, _ in sch if s in (1, 400, 401, 800, 801, 1000)] == [1, 400, 1, 400, 1, 200]


# ------------------------------------------------------- POET-XQ weight format (8-bit reading)
def _xq_pins_pass(mod):
    """The quantiser pins below, run against a module (the oracle or a planted variant); a variant
    that raises counts as caught."""
    try:
        return _xq_pins(mod)
    except (IndexError, ValueError, TypeError):
        return False


def _xq_pins(mod):
    ok = True
    # Hand example.  Row 0: absmax 127/128, so s = 1/128 exactly (127/128 / 127 is exact in
    # float32) and each code is w * 128 rounded half to even: 0.5 -> 64, 64.5/128 -> 64,
    # 65.5/128 -> 66, -127/128 -> -127, 1/256 -> 0, 3/256 -> 2.  Row 1: zeros -> s = 0, q = 0.
    # Row 2: +-2 are the absmax -> +-127 whatever the rounding of 2/127; 0.25 -> 16 (15.875).
    W = np.array([[0.5, 64.5 / 128, 65.5 / 128, -127 / 128, 1 / 256, 3 / 256],
                  [0, 0, 0, 0, 0, 0],
                  [2.0, -2.0, 0.25, 0, -0.25, 1e-6]], np.float32)
    q, s = mod.quantize_rows(W)
    ok &= q.dtype == np.int8 and s.dtype == np.float32
    ok &= np.array_equal(q, np.array([[64, 64, 66, -127, 0, 2], [0] * 6, [127, -127, 16, 0, -16, 0]]))
    ok &= s[0] == np.float32(1 / 128) and s[1] == 0 and s[2] == np.float32(np.float32(2.0) / np.float32(127))
    # On-grid rows come back exactly: W = s0 * K with integer K (|K| <= 127, a +-127 in every
    # row) and a power-of-two s0 per row.
    rng = np.random.default_rng(21)
    K = rng.integers(-127, 128, size=(5, 40))
    K[np.arange(5), rng.integers(0, 40, 5)] = 127 * rng.choice([-1, 1], 5)
    s0 = 2.0 ** rng.integers(-12, 3, size=5)
    q, s = mod.quantize_rows((s0[:, None] * K).astype(np.float32))
    ok &= np.array_equal(q, K) and np.array_equal(s, s0.astype(np.float32))
    # Random rows of very different size: error at most half a step (plus float32 rounding of
    # w / s), every row reaches +-127 at its absmax, odd symmetry, power-of-two scale invariance.
    W = (rng.standard_normal((7, 300)) * (10.0 ** rng.integers(-4, 2, size=7))[:, None]).astype(np.float32)
    q, s = mod.quantize_rows(W)
    err = np.abs(W.astype(np.float64) - s.astype(np.float64)[:, None] * q)
    ok &= bool(np.all(err <= s.astype(np.float64)[:, None] * (0.5 + 1e-5)))
    ok &= bool(np.all(np.abs(q).max(axis=1) == 127))
    ok &= bool(np.all(q[np.arange(7), np.abs(W).argmax(axis=1)] == 127 * np.sign(W[np.arange(7), np.abs(W).argmax(axis=1)])))
    qn, sn = mod.quantize_rows(-W)
    ok &= np.array_equal(qn, -q) and np.array_equal(sn, s)
    q8, s8 = mod.quantize_rows(W * np.float32(8.0))
    ok &= np.array_equal(q8, q) and np.array_equal(s8, s * np.float32(8.0))
    return bool(ok)


def test_quantize_rows_pins():
    assert _xq_pins_pass(O)


def test_dequantize_rows_is_scale_times_code():
    q = np.array([[1, -127, 0], [5, 6, 7]], np.int8)
    s = np.array([0.5, 0.25], np.float32)
    assert np.array_equal(O.dequantize_rows(q, s), np.array([[0.5, -63.5, 0.0], [1.25, 1.5, 1.75]]))


def test_xq_merge_is_merge_then_requantise_and_fixed_at_zero_theta():
    rng = np.random.default_rng(82)
    b = 4
    L = _rand_layer(rng, 16, 12, b, 3)
    q, s = O.quantize_rows(O.absorb(L["W0"], L["pi_L"], L["pi_R"]))
    # Zero theta and the same permutations: the merged weight is the dequantised one and
    # quantising it again gives back the same codes and scales.
    z, zP = np.zeros_like(L["theta_R"]), np.zeros_like(L["theta_P"])
    Wn, qn, sn, _, _ = O.xq_merge(q, s, z, zP, L["pi_L"], L["pi_R"], L["pi_L"], L["pi_R"], b, 3)
    assert np.abs(Wn - O.dequantize_rows(q, s)).max() <= 1e-15
    assert np.array_equal(qn, q) and np.array_equal(sn, s)
    # General theta: the layer function of the merged (unquantised) weight is that of the
    # dequantised layer before the merge; the new codes are within half a step of it.
    pL2, pR2 = rng.permutation(12), rng.permutation(16)
    Wn, qn, sn, tR, tP = O.xq_merge(q, s, L["theta_R"], L["theta_P"], L["pi_L"], L["pi_R"], pL2, pR2, b, 3)
    assert np.all(tR == 0) and np.all(tP == 0)
    Wdq = O.dequantize_rows(q, s)
    Y_before = O.forward_chain(L["X"], Wdq, O.cnp(L["theta_R"], b, 3), O.cnp(L["theta_P"], b, 3), L["pi_L"], L["pi_R"])[0]
    Y_after = O.forward_chain(L["X"], Wn, O.cnp(tR, b, 3), O.cnp(tP, b, 3), pL2, pR2)[0]
    assert _rel(Y_after, Y_before) <= 1e-12
    assert np.all(np.abs(np.float32(Wn) - O.dequantize_rows(qn, sn)) <= sn[:, None] * (0.5 + 1e-5) + 1e-7 * np.abs(Wn))


def test_quantize_planted_mistakes_are_caught():
    import types
    src_path = os.path.join(os.path.dirname(O.__file__), "poetx_ref.py")
    with open(src_path) as f:
        src = f.read()

    def variant(old, new):
        assert old in src, old
        m = types.ModuleType("oracle_variant")
        exec(compile(src.replace(old, new, 1), "oracle_variant", "exec"), m.__dict__)
        return m

    mistakes = [
        ("codes = np.rint(W[live] / s[live, None])", "codes = np.floor(W[live] / s[live, None])"),   # truncation
        ("codes = np.rint(W[live] / s[live, None])", "codes = np.round(W[live] / s[live, None] + 0.5 * (W[live] > 0))"),  # ties away
        ("amax = np.max(np.abs(W), axis=1)", "amax = np.max(np.abs(W))"),                          # one scale per tensor
        ("s = (amax / np.float32(127.0))", "s = (amax / np.float32(128.0))"),                      # 128 levels
        ("np.clip(codes, -127, 127)", "np.clip(codes, -128, 126)"),                                # asymmetric clip
    ]
    for old, new in mistakes:
        assert not _xq_pins_pass(variant(old, new)), new
