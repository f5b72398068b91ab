"""The four-permutation comparator (R and P applied around the un-absorbed W0, four activation
permutations per pass) against the oracle's dense definition, which builds R = Pi_L^T BD_R Pi_L and
P = Pi_R^T BD_P Pi_R with their four explicit permutations, and against the two-permutation path."""
import pytest
import torch

import oracle as O
import poetx_inputs as I
from helpers import TOL, device_clean, gpu_layer, rel, to_np
from orthogonal_equivalence_cnp_b200.layer import PoetxLayer, make_desc

pytestmark = pytest.mark.gpu


def _fp(inp):
    s = inp.shape
    L = PoetxLayer(make_desc(s.d_in, s.d_out, s.b, s.k, s.dtype, "fast"), inp.X.shape[0])
    L.load_state(inp.W0, inp.theta_R, inp.theta_P, inp.pi_L, inp.pi_R)
    X, dY = L.to_dev(inp.X), L.to_dev(inp.dY)
    L.fourperm_step(X, dY)
    torch.cuda.synchronize()
    return dict(Y=to_np(L.Y), dX=to_np(L.dX), g_R=to_np(L.g_R), g_P=to_np(L.g_P))


@pytest.mark.parametrize("dtype,d_in,d_out,b,n", [("f32", 256, 256, 32, 64), ("bf16", 512, 768, 256, 130),
                                                  ("bf16", 768, 512, 128, 200), ("bf16", 1024, 512, 512, 129)])
def test_fourperm_matches_dense_oracle(dtype, d_in, d_out, b, n):
    if dtype == "f32":
        inp = I.make_workload("layer256_b32_f32")
    else:
        inp = I.make_layer(I.small_shape(d_in, d_out, b, 3, n, dtype, theta_std=0.005, w_std=0.02), 41 + b)
    s = inp.shape
    g = _fp(inp)
    device_clean()
    Y = O.forward_dense(inp.X, inp.W0, inp.theta_R, inp.theta_P, inp.pi_L, inp.pi_R, s.b, s.k)
    dX, gR, gP = O.backward_dense(inp.X, inp.dY, inp.W0, inp.theta_R, inp.theta_P, inp.pi_L, inp.pi_R, s.b, s.k)
    errs = {"Y": rel(g["Y"], Y), "dX": rel(g["dX"], dX), "g_R": rel(g["g_R"], gR), "g_P": rel(g["g_P"], gP)}
    assert all(e <= TOL[dtype] for e in errs.values()), errs


def test_fourperm_agrees_with_two_permutation_path():
    inp = I.make_layer(I.small_shape(1024, 512, 256, 3, 256, "bf16", theta_std=0.005, w_std=0.02), 78)
    gi, _ = gpu_layer(inp, mode="fast")
    gf = _fp(inp)
    device_clean()
    for k in ("Y", "dX", "g_R", "g_P"):
        assert rel(gf[k], gi[k]) <= TOL["bf16"], k
