"""Parity of the CUDA layer (through the C ABI) with the float64 oracle on the same seeded inputs."""
import numpy as np
import pytest
import torch

import oracle as O
import orthogonal_equivalence_cnp_b200 as P
import poetx_inputs as I
from helpers import TOL, device_clean, gpu_layer, oracle_layer, rel, to_np
from orthogonal_equivalence_cnp_b200.layer import PoetxLayer, make_desc

pytestmark = pytest.mark.gpu

KEYS = ("Q_R", "Q_P", "Y", "dX", "g_R", "g_P")


def _check_all(g, o, tol, keys=KEYS):
    errs = {k: rel(g[k], o[k]) for k in keys}
    bad = {k: e for k, e in errs.items() if not e <= tol}
    assert not bad, f"errors {errs} exceed {tol}"
    return errs


# ------------------------------------------------------------------------------ CNP alone
@pytest.mark.parametrize("k", [0, 1, 2, 3, 5])
def test_cnp_f32(k):
    s = I.small_shape(256, 128, 32, k, 8, "f32", theta_std=0.05)
    inp = I.make_layer(s, 7 + k, with_activations=False)
    desc = make_desc(256, 128, 32, k, "f32", "fast")
    L = PoetxLayer(desc, 8)
    L.load_state(inp.W0, inp.theta_R, inp.theta_P, inp.pi_L, inp.pi_R)
    L.cnp()
    torch.cuda.synchronize()
    device_clean()
    assert rel(to_np(L.Q_R), O.cnp(inp.theta_R, 32, k)) <= TOL["f32"]
    assert rel(to_np(L.Q_P), O.cnp(inp.theta_P, 32, k)) <= TOL["f32"]


@pytest.mark.parametrize("b", [64, 128, 256, 512])
def test_cnp_bf16(b):
    s = I.small_shape(2 * b, b, b, 3, 8, "bf16", theta_std=0.005)
    inp = I.make_layer(s, 100 + b, with_activations=False)
    L = PoetxLayer(make_desc(2 * b, b, b, 3, "bf16", "fast"), 8)
    L.load_state(inp.W0, inp.theta_R, inp.theta_P, inp.pi_L, inp.pi_R)
    L.cnp()
    torch.cuda.synchronize()
    device_clean()
    assert rel(to_np(L.Q_R), O.cnp(inp.theta_R, b, 3)) <= TOL["bf16"]
    assert rel(to_np(L.Q_P), O.cnp(inp.theta_P, b, 3)) <= TOL["bf16"]


# ------------------------------------------------------------- Neumann order resolved (bf16)
# theta is drawn with std 0.45 / sqrt(b), so that ||S||_2 is about 0.9.  Then the parts of the
# outputs beyond their exact leading terms, Q - I - 2S and g - 2 pack(G - G^T), differ between
# order k and order k - 1 by many times the bf16 tolerance.  Each test asserts that on the oracle
# alone before comparing the GPU result at order k, so a kernel that dropped, repeated or
# mis-weighted one term of the series (forward) or of its adjoint would fail.
def _resolving_std(b):
    return 0.45 / np.sqrt(b)


def _remainders(inp, Q_R, Q_P, G_R, G_P, g_R, g_P):
    """Q - I - 2S and g - 2 pack(G - G^T): the outputs less their exact first-order terms (k >= 1)."""
    s = inp.shape
    S_R, S_P = O.unpack_skew(inp.theta_R, s.b), O.unpack_skew(inp.theta_P, s.b)
    eye = np.eye(s.b)
    lead_R = 2 * O.cnp_grad(inp.theta_R, G_R, s.b, 0)
    lead_P = 2 * O.cnp_grad(inp.theta_P, G_P, s.b, 0)
    return dict(Q_R=Q_R - eye - 2 * S_R, Q_P=Q_P - eye - 2 * S_P, g_R=g_R - lead_R, g_P=g_P - lead_P)


@pytest.mark.parametrize("b", [64, 128, 256, 512])
@pytest.mark.parametrize("k", [1, 2, 3, 5])
def test_bf16_layer_resolves_neumann_order(b, k):
    d_in, d_out, n = 2 * b, b, 136
    s = I.small_shape(d_in, d_out, b, k, n, "bf16", theta_std=_resolving_std(b), w_std=0.02)
    inp = I.make_layer(s, 300 + 7 * b + k)
    g, _ = gpu_layer(inp, mode="mem" if k % 2 else "fast")
    device_clean()
    o = oracle_layer(inp)
    _check_all(g, o, TOL["bf16"])
    W0p = O.absorb(inp.W0, inp.pi_L, inp.pi_R)
    _, G_R, G_P = O.backward_chain_G(inp.X, inp.dY, W0p, o["Q_R"], o["Q_P"], inp.pi_L, inp.pi_R, b)
    want = _remainders(inp, o["Q_R"], o["Q_P"], G_R, G_P, o["g_R"], o["g_P"])
    lower = _remainders(inp, O.cnp(inp.theta_R, b, k - 1), O.cnp(inp.theta_P, b, k - 1), G_R, G_P,
                        O.cnp_grad(inp.theta_R, G_R, b, k - 1), O.cnp_grad(inp.theta_P, G_P, b, k - 1))
    for key in want:
        assert rel(lower[key], want[key]) >= 4 * TOL["bf16"], (key, "orders k and k-1 are not resolved")
    got = _remainders(inp, g["Q_R"], g["Q_P"], G_R, G_P, g["g_R"], g["g_P"])
    errs = {key: rel(got[key], want[key]) for key in want}
    assert all(e <= TOL["bf16"] for e in errs.values()), errs


def test_unpack_bit_exact():
    # k = 0 gives Q = I + S: every entry is a theta value, its negative, 0 or 1 -- bit-exact.
    s = I.small_shape(64, 64, 32, 0, 4, "f32", theta_std=0.3)
    inp = I.make_layer(s, 3, with_activations=False)
    L = PoetxLayer(make_desc(64, 64, 32, 0, "f32", "fast"), 4)
    L.load_state(inp.W0, inp.theta_R, inp.theta_P, inp.pi_L, inp.pi_R)
    L.cnp()
    torch.cuda.synchronize()
    expect = np.eye(32) + O.unpack_skew(inp.theta_R, 32)
    assert np.array_equal(to_np(L.Q_R), expect)


# ------------------------------------------------------------------------ index plumbing
# Every permutation kernel path: 1216 rows x 4096 columns (several four-row groups per block,
# ragged last group), 6144 columns (four-row groups), 10240 columns (two-row groups), 17408
# columns (the register-staged kernel for rows too wide for the bulk-copy ring).
@pytest.mark.parametrize("dtype,d_in,d_out", [("f32", 512, 384), ("bf16", 512, 384), ("bf16", 4096, 1216),
                                              ("bf16", 6144, 512), ("bf16", 10240, 256), ("bf16", 17408, 128)])
def test_absorb_bit_exact(dtype, d_in, d_out):
    s = I.small_shape(d_in, d_out, 64, 3, 4, dtype)
    inp = I.make_layer(s, 11, with_activations=False)
    L = PoetxLayer(make_desc(d_in, d_out, 64, 3, dtype, "fast"), 4)
    L.load_state(inp.W0, inp.theta_R, inp.theta_P, inp.pi_L, inp.pi_R)
    torch.cuda.synchronize()
    assert np.array_equal(to_np(L.W0p), O.absorb(inp.W0, inp.pi_L, inp.pi_R))


@pytest.mark.parametrize("dtype,b", [("f32", 32), ("bf16", 64), ("bf16", 256)])
@pytest.mark.parametrize("mode", ["fast", "mem"])
def test_identity_layer_is_bit_exact(dtype, b, mode):
    # W0 = I and theta = 0 make R W0 P = I: Y must equal X and dX must equal dY bit for bit,
    # which checks every gather, scatter and absorbed index of the chain.
    d, n = 512, 193
    s = I.small_shape(d, d, b, 3, n, dtype)
    inp = I.make_layer(s, 21)
    inp.W0 = np.eye(d, dtype=np.float32)
    inp.theta_R[:] = 0
    inp.theta_P[:] = 0
    g, _ = gpu_layer(inp, mode=mode)
    device_clean()
    assert np.array_equal(g["Y"], inp.X.astype(np.float64))
    assert np.array_equal(g["dX"], inp.dY.astype(np.float64))


# ------------------------------------------------------------------------- full layer
def test_layer_f32_256_b32():
    inp = I.make_workload("layer256_b32_f32")
    g, _ = gpu_layer(inp)
    device_clean()
    _check_all(g, oracle_layer(inp), TOL["f32"])


@pytest.mark.parametrize("k", [0, 1, 2, 3])
def test_layer_f32_orders(k):
    s = I.small_shape(128, 192, 32, k, 70, "f32", theta_std=0.05)
    inp = I.make_layer(s, 40 + k)
    g, _ = gpu_layer(inp, mode="mem" if k % 2 else "fast")
    device_clean()
    _check_all(g, oracle_layer(inp), TOL["f32"])


@pytest.mark.parametrize("d_in,d_out,b,n", [(512, 384, 128, 300), (256, 512, 64, 130), (1024, 768, 256, 200),
                                            (512, 1280, 256, 333), (512, 512, 256, 600),
                                            (1024, 1024, 512, 129)])
@pytest.mark.parametrize("mode", ["fast", "mem"])
def test_layer_bf16_small(d_in, d_out, b, n, mode):
    s = I.small_shape(d_in, d_out, b, 3, n, "bf16", theta_std=0.005, w_std=0.02)
    inp = I.make_layer(s, d_in + d_out + b + n)
    g, _ = gpu_layer(inp, mode=mode)
    device_clean()
    _check_all(g, oracle_layer(inp), TOL["bf16"])


# Shapes whose W0' GEMMs take the 256 x 256-tile kernel (>= 111 tiles) with a ragged last row
# tile: forward (d_out wide) and backward (d_in wide), with (b = 256) and without the fused
# block factor.
@pytest.mark.parametrize("d_in,d_out,b", [(512, 7168, 256), (7168, 512, 256), (512, 7168, 128), (7168, 512, 128)])
@pytest.mark.parametrize("mode", ["fast", "mem"])
def test_layer_bf16_wide_tiles(d_in, d_out, b, mode):
    s = I.small_shape(d_in, d_out, b, 3, 1000, "bf16", theta_std=0.005, w_std=0.02)
    inp = I.make_layer(s, 5 + d_in + b)
    g, _ = gpu_layer(inp, mode=mode)
    device_clean()
    _check_all(g, oracle_layer(inp), TOL["bf16"])


@pytest.mark.parametrize("k", [0, 1, 2])
def test_layer_bf16_orders(k):
    s = I.small_shape(512, 512, 128, k, 160, "bf16", theta_std=0.005, w_std=0.02)
    inp = I.make_layer(s, 60 + k)
    g, _ = gpu_layer(inp)
    device_clean()
    _check_all(g, oracle_layer(inp), TOL["bf16"])


@pytest.mark.parametrize("dtype,b,mode", [("bf16", 256, "fast"), ("bf16", 64, "mem"), ("f32", 32, "fast")])
def test_cnp_forward_call_equals_the_two_calls(dtype, b, mode):
    # poetx_cnp_forward runs the CNP beside the input gather; the results are the same kernels'
    # results, so they must equal poetx_cnp followed by poetx_forward bit for bit.
    s = I.small_shape(4 * b, 2 * b, b, 3, 200, dtype, theta_std=0.005 if dtype == "bf16" else 0.05, w_std=0.02)
    inp = I.make_layer(s, 17 + b)
    L = PoetxLayer(make_desc(4 * b, 2 * b, b, 3, dtype, mode), 200)
    L.load_state(inp.W0, inp.theta_R, inp.theta_P, inp.pi_L, inp.pi_R)
    X = L.to_dev(inp.X)
    L.cnp()
    L.forward(X)
    torch.cuda.synchronize()
    ref = {k: t.clone() for k, t in (("Q_R", L.Q_R), ("Q_P", L.Q_P), ("Y", L.Y))}
    saved_ref = L.saved.clone() if L.saved is not None else None
    for t in (L.Q_R, L.Q_P, L.Y):
        t.fill_(float("nan"))
    L.cnp_forward(X)
    torch.cuda.synchronize()
    device_clean()
    for k, t in (("Q_R", L.Q_R), ("Q_P", L.Q_P), ("Y", L.Y)):
        assert torch.equal(t, ref[k]), k
    if saved_ref is not None:
        assert torch.equal(L.saved, saved_ref)


@pytest.mark.parametrize("mode", ["fast", "mem"])
def test_repeated_steps_are_bit_identical(mode):
    # 600 tokens, two 256-blocks per side: theta_P's block gradients run as two K splits that add
    # into one tile set zeroed in every backward call, so a second step on the same inputs must
    # reproduce the first bit for bit (two addends onto zero: the order cannot change the sum).
    s = I.small_shape(512, 512, 256, 3, 600, "bf16", theta_std=0.005, w_std=0.02)
    inp = I.make_layer(s, 4242)
    g1, L = gpu_layer(inp, mode=mode)
    X, dY = L.to_dev(inp.X), L.to_dev(inp.dY)
    L.step(X, dY)
    torch.cuda.synchronize()
    g2 = dict(Q_R=to_np(L.Q_R), Q_P=to_np(L.Q_P), Y=to_np(L.Y), dX=to_np(L.dX), g_R=to_np(L.g_R), g_P=to_np(L.g_P))
    device_clean()
    for k in KEYS:
        assert np.array_equal(g1[k], g2[k]), k
    _check_all(g2, oracle_layer(inp), TOL["bf16"])


def test_fast_and_mem_agree():
    s = I.small_shape(512, 512, 128, 3, 200, "bf16", theta_std=0.005, w_std=0.02)
    inp = I.make_layer(s, 77)
    gf, _ = gpu_layer(inp, mode="fast")
    gm, _ = gpu_layer(inp, mode="mem")
    for k in KEYS:
        assert np.array_equal(gf[k], gm[k]), k


def test_layer_llama8b_attn_full_size():
    # The benchmark workload (4096 x 4096, b = 256, 2048 tokens, bf16, fast mode), compared
    # element by element with the oracle over every output.
    inp = I.make_workload("llama8b_attn_4096_b256_bf16")
    g, _ = gpu_layer(inp)
    device_clean()
    _check_all(g, oracle_layer(inp), TOL["bf16"])


@pytest.mark.parametrize("name", ["llama8b_up_4096x14336_b256_bf16_mem", "llama8b_up_4096x14336_b512_bf16_mem"])
def test_layer_llama8b_up_full_size_sampled(name):
    # Full-size mem-mode layer (8192 tokens).  Y and dX rows are checked on sampled tokens; the
    # gradients, which sum over all tokens, are checked through linearity: the upstream gradient
    # is zero except on the sampled tokens, so the oracle needs only those rows.
    inp = I.make_workload(name)
    rows = np.sort(np.random.default_rng(5).choice(inp.X.shape[0], 96, replace=False))
    g, _ = gpu_layer(inp, dY_rows=rows)
    device_clean()
    o = oracle_layer(inp, rows=rows)
    errs = {"Y": rel(g["Y"][rows], o["Y"]), "dX": rel(g["dX"][rows], o["dX"]),
            "g_R": rel(g["g_R"], o["g_R"]), "g_P": rel(g["g_P"], o["g_P"]),
            "Q_R": rel(g["Q_R"], o["Q_R"]), "Q_P": rel(g["Q_P"], o["Q_P"])}
    assert all(e <= TOL["bf16"] for e in errs.values()), errs
    others = np.setdiff1d(np.arange(inp.X.shape[0]), rows)[:64]
    assert np.all(g["dX"][others] == 0)


# ------------------------------------------------------------------------------- merge
@pytest.mark.parametrize("dtype,d_in,d_out,b", [("f32", 256, 128, 32), ("bf16", 1024, 512, 256), ("bf16", 512, 1024, 64)])
def test_merge(dtype, d_in, d_out, b):
    s = I.small_shape(d_in, d_out, b, 3, 64, dtype, theta_std=0.005 if dtype == "bf16" else 0.05, w_std=0.02)
    inp = I.make_layer(s, 90 + b)
    pL2, pR2 = I.fresh_permutations(s, 90 + b)
    L = PoetxLayer(make_desc(d_in, d_out, b, 3, dtype, "fast"), 64)
    L.load_state(inp.W0, inp.theta_R, inp.theta_P, inp.pi_L, inp.pi_R)
    L.cnp()
    L.merge(torch.from_numpy(pL2).cuda(), torch.from_numpy(pR2).cuda())
    torch.cuda.synchronize()
    device_clean()
    W0p = O.absorb(inp.W0, inp.pi_L, inp.pi_R)
    Wn, _, _ = O.merge(W0p, inp.theta_R, inp.theta_P, inp.pi_L, inp.pi_R, pL2, pR2, b, 3)
    assert rel(to_np(L.W0p), Wn) <= TOL[dtype]
    assert torch.count_nonzero(L.theta_R).item() == 0 and torch.count_nonzero(L.theta_P).item() == 0
    # After the merge the layer (theta = 0, new permutations) computes the same function.
    L.cnp()
    X = L.to_dev(inp.X)
    L.forward(X)
    torch.cuda.synchronize()
    Y_before = O.forward_chain(inp.X, W0p, O.cnp(inp.theta_R, b, 3), O.cnp(inp.theta_P, b, 3), inp.pi_L, inp.pi_R)[0]
    assert rel(to_np(L.Y), Y_before) <= TOL[dtype]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_merge_with_zero_theta_is_bit_exact(dtype):
    # theta = 0 makes Q = I exactly, so the merge is a pure composed permutation of W0'.
    d_in, d_out, b = 512, 256, 64
    s = I.small_shape(d_in, d_out, b, 3, 8, dtype)
    inp = I.make_layer(s, 5, with_activations=False)
    inp.theta_R[:] = 0
    inp.theta_P[:] = 0
    pL2, pR2 = I.fresh_permutations(s, 5)
    L = PoetxLayer(make_desc(d_in, d_out, b, 3, dtype, "fast"), 8)
    L.load_state(inp.W0, inp.theta_R, inp.theta_P, inp.pi_L, inp.pi_R)
    L.cnp()
    L.merge(torch.from_numpy(pL2).cuda(), torch.from_numpy(pR2).cuda())
    torch.cuda.synchronize()
    assert np.array_equal(to_np(L.W0p), O.absorb(inp.W0, pL2, pR2))


def test_zero_tokens():
    s = I.small_shape(256, 256, 64, 3, 1, "bf16")
    inp = I.make_layer(s, 1, with_activations=False)
    desc = make_desc(256, 256, 64, 3, "bf16", "fast")
    L = PoetxLayer(desc, 0)
    L.load_state(inp.W0, inp.theta_R, inp.theta_P, inp.pi_L, inp.pi_R)
    L.g_R.fill_(7.0)
    L.cnp()
    L.forward(torch.empty(0, 256, dtype=torch.bfloat16, device="cuda"))
    L.backward(torch.empty(0, 256, dtype=torch.bfloat16, device="cuda"), torch.empty(0, 256, dtype=torch.bfloat16, device="cuda"))
    torch.cuda.synchronize()
    assert torch.count_nonzero(L.g_R).item() == 0
