"""The weight-centric comparator (the original POET order: form W = R W0 P, then dense products)
against the oracle's dense definition, and against the input-centric path on the same inputs."""
import numpy as np
import pytest
import torch

import oracle as O
import poetx_inputs as I
from helpers import TOL, device_clean, gpu_layer, rel, to_np
from orthogonal_equivalence_cnp_b200.layer import PoetxLayer, make_desc

pytestmark = pytest.mark.gpu


def _wc(inp, mode):
    s = inp.shape
    L = PoetxLayer(make_desc(s.d_in, s.d_out, s.b, s.k, s.dtype, mode), inp.X.shape[0])
    L.load_state(inp.W0, inp.theta_R, inp.theta_P, inp.pi_L, inp.pi_R)
    X, dY = L.to_dev(inp.X), L.to_dev(inp.dY)
    L.wc_step(X, dY)
    torch.cuda.synchronize()
    W = to_np(L.wc_saved[: s.d_out * s.d_in * (2 if s.dtype == "bf16" else 4)].view(L.dtype).reshape(s.d_out, s.d_in))
    return dict(Y=to_np(L.Y), dX=to_np(L.dX), g_R=to_np(L.g_R), g_P=to_np(L.g_P), W=W)


@pytest.mark.parametrize("dtype,d_in,d_out,b,n", [("f32", 256, 256, 32, 64), ("bf16", 512, 768, 256, 130),
                                                  ("bf16", 768, 512, 128, 200)])
def test_weight_centric_matches_dense_oracle(dtype, d_in, d_out, b, n):
    if dtype == "f32":
        inp = I.make_workload("layer256_b32_f32")
    else:
        inp = I.make_layer(I.small_shape(d_in, d_out, b, 3, n, dtype, theta_std=0.005, w_std=0.02), 31 + b)
    s = inp.shape
    g = _wc(inp, "fast")
    device_clean()
    Y = O.forward_dense(inp.X, inp.W0, inp.theta_R, inp.theta_P, inp.pi_L, inp.pi_R, s.b, s.k)
    dX, gR, gP = O.backward_dense(inp.X, inp.dY, inp.W0, inp.theta_R, inp.theta_P, inp.pi_L, inp.pi_R, s.b, s.k)
    W = O.dense_weight(inp.W0, O.cnp(inp.theta_R, s.b, s.k), O.cnp(inp.theta_P, s.b, s.k), inp.pi_L, inp.pi_R)
    tol = TOL[dtype]
    errs = {"W": rel(g["W"], W), "Y": rel(g["Y"], Y), "dX": rel(g["dX"], dX), "g_R": rel(g["g_R"], gR),
            "g_P": rel(g["g_P"], gP)}
    assert all(e <= tol for e in errs.values()), errs


def test_weight_centric_agrees_with_input_centric():
    inp = I.make_layer(I.small_shape(1024, 512, 256, 3, 256, "bf16", theta_std=0.005, w_std=0.02), 77)
    gi, _ = gpu_layer(inp, mode="fast")
    gw = _wc(inp, "fast")
    device_clean()
    for k in ("Y", "dX", "g_R", "g_P"):
        assert rel(gw[k], gi[k]) <= TOL["bf16"], k
