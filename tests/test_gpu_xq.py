"""POET-XQ against the oracle: W0' held as int8 codes with one float32 scale per row (the
library's reading of the pages' 8-bit variant), run through POET-Xmem with the W0' GEMMs
dequantising their tiles in shared memory.

The codes and scales are integer/float decisions taken in float32 on both sides from the same
bf16 W0', so they are compared bit for bit.  The layer outputs are compared with the oracle's
POET-Xmem layer on W0' = s * q (the oracle's own codes) at the bf16 tolerance: the GEMMs see
bf16(s * q), one more rounding of the same size as storing W0' in bf16.
"""
import numpy as np
import pytest
import torch

import oracle as O
import orthogonal_equivalence_cnp_b200 as P
import poetx_inputs as I
from helpers import TOL, device_clean, rel, to_np
from orthogonal_equivalence_cnp_b200.layer import PoetxLayer, make_desc

pytestmark = pytest.mark.gpu


def _gpu_xq(inp, dY_rows=None):
    s = inp.shape
    L = PoetxLayer(make_desc(s.d_in, s.d_out, s.b, s.k, "bf16", "mem"), inp.X.shape[0])
    L.load_state(inp.W0, inp.theta_R, inp.theta_P, inp.pi_L, inp.pi_R)
    L.quantize()
    X = L.to_dev(inp.X)
    dY_np = inp.dY
    if dY_rows is not None:
        dY_np = np.zeros_like(inp.dY)
        dY_np[dY_rows] = inp.dY[dY_rows]
    L.step(X, L.to_dev(dY_np))
    torch.cuda.synchronize()
    out = dict(Y=to_np(L.Y), dX=to_np(L.dX), g_R=to_np(L.g_R), g_P=to_np(L.g_P),
               q=L.W0q.cpu().numpy(), s=L.W0s.cpu().numpy())
    return out, L


def _oracle_xq(inp, rows=None):
    s = inp.shape
    X, dY = (inp.X, inp.dY) if rows is None else (inp.X[rows], inp.dY[rows])
    q, sc = O.quantize_rows(O.absorb(inp.W0, inp.pi_L, inp.pi_R))
    Wd = O.dequantize_rows(q, sc)
    Y = O.forward_chain(X, Wd, O.cnp(inp.theta_R, s.b, s.k), O.cnp(inp.theta_P, s.b, s.k), inp.pi_L, inp.pi_R)[0]
    dX, gR, gP = O.backward_chain(X, dY, Wd, inp.theta_R, inp.theta_P, inp.pi_L, inp.pi_R, s.b, s.k)
    return dict(Y=Y, dX=dX, g_R=gR, g_P=gP, q=q, s=sc)


def _codes_equal(g, o):
    assert np.array_equal(g["q"], o["q"]), int(np.count_nonzero(g["q"] != o["q"]))
    assert np.array_equal(g["s"].view(np.uint32), o["s"].view(np.uint32))


# ------------------------------------------------------------------------ the weight format
@pytest.mark.parametrize("d_in,d_out", [(256, 256), (512, 768), (4096, 4096), (4096, 14336)])
def test_quantize_bit_exact(d_in, d_out):
    rng = np.random.default_rng(d_in + d_out)
    W = I.round_to_bf16((rng.standard_normal((d_out, d_in)) * 0.02).astype(np.float32))
    W[1] = 0.0                                             # zero row: s = 0, q = 0
    W[2] = 0.0
    W[2, :6] = [0.5, 64.5 / 128, 65.5 / 128, -127 / 128, 1 / 256, 3 / 256]  # exact ties (s = 1/128)
    W[3] = I.round_to_bf16(W[3] * np.float32(1e4))         # rows of very different size
    W[4] = I.round_to_bf16(W[4] * np.float32(1e-6))
    desc = make_desc(d_in, d_out, 256, 3, "bf16", "mem")
    Wd = torch.from_numpy(W).to("cuda", torch.bfloat16)
    q = torch.empty(d_out, d_in, dtype=torch.int8, device="cuda")
    s = torch.empty(d_out, dtype=torch.float32, device="cuda")
    P.poetx_xq_quantize(desc, Wd, q, s)
    torch.cuda.synchronize()
    device_clean()
    qo, so = O.quantize_rows(W)
    _codes_equal(dict(q=q.cpu().numpy(), s=s.cpu().numpy()), dict(q=qo, s=so))
    assert np.array_equal(qo[2, :6], [64, 64, 66, -127, 0, 2]) and so[1] == 0
    # bf16(s * q) within one bf16 rounding of the oracle's s * q
    back = torch.empty_like(Wd)
    P.poetx_xq_dequantize(desc, q, s, back)
    torch.cuda.synchronize()
    ref = O.dequantize_rows(qo, so)
    assert np.all(np.abs(to_np(back) - ref) <= np.abs(ref) * 2.0 ** -8)


# ------------------------------------------------------------------------------ the layer
@pytest.mark.parametrize("d_in,d_out,b,n", [(512, 768, 256, 300), (768, 512, 128, 200), (1024, 1024, 512, 129),
                                            (512, 512, 256, 600), (256, 1280, 64, 77)])
def test_xq_layer_matches_oracle(d_in, d_out, b, n):
    # b = 256: the W0' GEMMs carry the fused block factor; other b: plain dequantising GEMM then
    # separate block products.  Token counts leave a ragged last row tile.
    s = I.small_shape(d_in, d_out, b, 3, n, "bf16", "mem", theta_std=0.005, w_std=0.02)
    inp = I.make_layer(s, 7 * d_in + d_out + b + n)
    g, _ = _gpu_xq(inp)
    device_clean()
    o = _oracle_xq(inp)
    _codes_equal(g, o)
    errs = {k: rel(g[k], o[k]) for k in ("Y", "dX", "g_R", "g_P")}
    assert all(e <= TOL["bf16"] for e in errs.values()), errs


@pytest.mark.parametrize("name", ["llama8b_attn_4096_b256_bf16", "llama8b_up_4096x14336_b256_bf16_mem",
                                  "llama8b_up_4096x14336_b512_bf16_mem"])
def test_xq_full_size_sampled(name):
    # Full-size layers (the attention projection run in mem mode for POET-XQ); Y and dX on
    # sampled tokens, the gradients through linearity (upstream gradient zero elsewhere).
    inp = I.make_workload(name)
    rows = np.sort(np.random.default_rng(6).choice(inp.X.shape[0], 64, replace=False))
    g, _ = _gpu_xq(inp, dY_rows=rows)
    device_clean()
    o = _oracle_xq(inp, rows=rows)
    _codes_equal(g, o)
    errs = {"Y": rel(g["Y"][rows], o["Y"]), "dX": rel(g["dX"][rows], o["dX"]),
            "g_R": rel(g["g_R"], o["g_R"]), "g_P": rel(g["g_P"], o["g_P"])}
    assert all(e <= TOL["bf16"] for e in errs.values()), errs


def test_xq_equals_bf16_mem_layer_on_the_dequantised_weight():
    # At the bench size both routes run the same 256 x 256-tile kernel on the same bf16 values
    # (the in-kernel dequantisation and the standalone one round s * q identically), so the
    # results agree bit for bit.
    inp = I.make_workload("llama8b_attn_4096_b256_bf16")
    g, Lq = _gpu_xq(inp)
    s = inp.shape
    L = PoetxLayer(make_desc(s.d_in, s.d_out, s.b, s.k, "bf16", "mem"), inp.X.shape[0])
    L.load_state(inp.W0, inp.theta_R, inp.theta_P, inp.pi_L, inp.pi_R)
    P.poetx_xq_dequantize(L.desc, Lq.W0q, Lq.W0s, L.W0p)
    L.step(L.to_dev(inp.X), L.to_dev(inp.dY))
    torch.cuda.synchronize()
    device_clean()
    for k, t in (("Y", L.Y), ("dX", L.dX), ("g_R", L.g_R), ("g_P", L.g_P)):
        assert np.array_equal(to_np(t), g[k]), k


# ------------------------------------------------------------------------------ the merge
@pytest.mark.parametrize("d_in,d_out,b", [(1024, 512, 256), (512, 768, 128)])
def test_xq_merge(d_in, d_out, b):
    s = I.small_shape(d_in, d_out, b, 3, 64, "bf16", "mem", theta_std=0.005, w_std=0.02)
    inp = I.make_layer(s, 91 + b)
    pL2, pR2 = I.fresh_permutations(s, 91 + b)
    L = PoetxLayer(make_desc(d_in, d_out, b, 3, "bf16", "mem"), 64)
    L.load_state(inp.W0, inp.theta_R, inp.theta_P, inp.pi_L, inp.pi_R)
    L.quantize()
    L.cnp()
    L.merge(torch.from_numpy(pL2).cuda(), torch.from_numpy(pR2).cuda())
    torch.cuda.synchronize()
    device_clean()
    assert torch.count_nonzero(L.theta_R).item() == 0 and torch.count_nonzero(L.theta_P).item() == 0
    q, sc = O.quantize_rows(O.absorb(inp.W0, inp.pi_L, inp.pi_R))
    Wn, qn, sn, _, _ = O.xq_merge(q, sc, inp.theta_R, inp.theta_P, inp.pi_L, inp.pi_R, pL2, pR2, b, 3)
    gq, gs = L.W0q.cpu().numpy(), L.W0s.cpu().numpy()
    # The library's merge products round to bf16 before the new weight is quantised, so codes
    # near a rounding boundary may land one step away from the oracle's; the scales (row
    # absmax / 127) and the dequantised weight are compared instead.
    assert rel(gs, sn) <= 2.0 ** -7
    assert rel(O.dequantize_rows(gq, gs), Wn) <= TOL["bf16"]
    # The merged layer (theta = 0, new permutations) computes the pre-merge POET-XQ layer.
    L.cnp()
    L.forward(L.to_dev(inp.X))
    torch.cuda.synchronize()
    Wd = O.dequantize_rows(q, sc)
    Y_before = O.forward_chain(inp.X, Wd, O.cnp(inp.theta_R, b, 3), O.cnp(inp.theta_P, b, 3), inp.pi_L, inp.pi_R)[0]
    assert rel(to_np(L.Y), Y_before) <= TOL["bf16"]


def test_xq_zero_tokens_and_rejections():
    desc = make_desc(512, 512, 256, 3, "bf16", "mem")
    L = PoetxLayer(desc, 8)
    L.W0p.zero_()
    L.quantize()
    assert torch.count_nonzero(L.W0q).item() == 0 and torch.count_nonzero(L.W0s).item() == 0
    P.poetx_xq_forward(desc, 0, L.dX, L.W0q, L.W0s, L.perm_L, L.perm_R, L.Q_R, L.Q_P, L.Y, L.ws)
    fast = make_desc(512, 512, 256, 3, "bf16", "fast")
    with pytest.raises(P.PoetxError):
        P.poetx_xq_forward(fast, 8, L.dX, L.W0q, L.W0s, L.perm_L, L.perm_R, L.Q_R, L.Q_P, L.Y, L.ws)
    device_clean()
