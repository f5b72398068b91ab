"""Shared helpers of the GPU parity tests (the CUDA side through the C ABI, the oracle side in f64)."""
from __future__ import annotations

import numpy as np

import oracle as O
import poetx_inputs as I

# Tolerances on relative Frobenius error: the fp32 path computes in fp32 throughout (only the
# summation order differs from the f64 oracle); the bf16 path rounds Q, V, Z, Y', dY', dZ, dV,
# dU and the stored outputs to bf16 (8 significant bits, relative rounding error <= 2^-9 per
# rounding), a handful of roundings in sequence, with fp32 accumulation in every product.
TOL = {"f32": 1e-5, "bf16": 2e-2}


def rel(gpu, ref) -> float:
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    return float(np.linalg.norm(gpu - ref) / max(np.linalg.norm(ref), 1e-300))


def to_np(t) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def device_clean():
    import orthogonal_equivalence_cnp_b200 as P
    s, d = P.poetx_device_status()
    assert s == 0, f"device-side wait gave up: status {s}, detail {d:#x}"


def gpu_layer(inp: I.LayerInputs, mode: str | None = None, dY_rows=None):
    """Runs CNP + forward + backward of one layer on cuda:0; returns a dict of numpy results."""
    import torch
    from orthogonal_equivalence_cnp_b200.layer import PoetxLayer, make_desc
    s = inp.shape
    desc = make_desc(s.d_in, s.d_out, s.b, s.k, s.dtype, mode or s.mode)
    n = inp.X.shape[0]
    layer = PoetxLayer(desc, n)
    layer.load_state(inp.W0, inp.theta_R, inp.theta_P, inp.pi_L, inp.pi_R)
    X = layer.to_dev(inp.X)
    dY_np = inp.dY
    if dY_rows is not None:
        dY_np = np.zeros_like(inp.dY)
        dY_np[dY_rows] = inp.dY[dY_rows]
    dY = layer.to_dev(dY_np)
    layer.step(X, dY)
    torch.cuda.synchronize()
    out = dict(Q_R=to_np(layer.Q_R), Q_P=to_np(layer.Q_P), Y=to_np(layer.Y), dX=to_np(layer.dX),
               g_R=to_np(layer.g_R), g_P=to_np(layer.g_P), W0p=to_np(layer.W0p))
    return out, layer


def oracle_layer(inp: I.LayerInputs, rows=None):
    """The f64 oracle on the same inputs (input-centric route; optionally on a subset of tokens)."""
    s = inp.shape
    X, dY = inp.X, inp.dY
    if rows is not None:
        X, dY = X[rows], dY[rows]
    Q_R, Q_P = O.cnp(inp.theta_R, s.b, s.k), O.cnp(inp.theta_P, s.b, s.k)
    W0p = O.absorb(inp.W0, inp.pi_L, inp.pi_R)
    Y = O.forward_chain(X, W0p, Q_R, Q_P, inp.pi_L, inp.pi_R)[0]
    dX, gR, gP = O.backward_chain(X, dY, W0p, inp.theta_R, inp.theta_P, inp.pi_L, inp.pi_R, s.b, s.k)
    return dict(Q_R=Q_R, Q_P=Q_P, Y=Y, dX=dX, g_R=gR, g_P=gP, W0p=W0p)
