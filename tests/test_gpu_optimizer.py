"""AdamW on the packed skew parameters and the merge schedule, against the oracle.

The optimiser kernel is fp32 elementwise arithmetic, so the fp32 tolerance (1e-5 relative
Frobenius) applies to theta, m, v and to the update theta' - theta itself.  The schedule test
runs whole training steps of the fp32 layer (CNP, forward, backward, AdamW, merge every two
steps with fresh permutations) and compares the trajectory with the oracle doing the same.
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

CFG = dict(lr=1e-3, gamma=0.5, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01)


def _cfg(c=CFG):
    return P.poetx_adamw_cfg(c["lr"], c["gamma"], c["beta1"], c["beta2"], c["eps"], c["weight_decay"])


@pytest.mark.parametrize("n,t", [(1_044_483, 7), (5, 1), (4096, 1000)])
def test_adamw_step_matches_oracle(n, t):
    # n = both sides of the 4096 x 4096, b = 256 layer plus a ragged tail of 3; a tiny case
    # that only the tail loop handles; a late step (bias corrections near 1).
    rng = np.random.default_rng(n + t)
    th = (rng.normal(size=n) * 0.005).astype(np.float32)
    g = rng.normal(size=n).astype(np.float32)
    m = (rng.normal(size=n) * 0.1).astype(np.float32)
    v = (rng.random(size=n) * 0.01).astype(np.float32)
    dth, dg, dm, dv = (torch.from_numpy(a.copy()).cuda() for a in (th, g, m, v))
    P.poetx_adamw_step(_cfg(), n, t, dth, dg, dm, dv)
    torch.cuda.synchronize()
    th1, m1, v1 = O.adamw_step(th, g, m, v, t, CFG["lr"], CFG["gamma"], CFG["beta1"], CFG["beta2"], CFG["eps"],
                               CFG["weight_decay"])
    gth, gm, gv = to_np(dth), to_np(dm), to_np(dv)
    assert rel(gth, th1) <= TOL["f32"] and rel(gm, m1) <= TOL["f32"] and rel(gv, v1) <= TOL["f32"]
    assert rel(gth - th.astype(np.float64), th1 - th.astype(np.float64)) <= TOL["f32"]
    P.poetx_adamw_reset(n, dm, dv)
    torch.cuda.synchronize()
    assert torch.count_nonzero(dm).item() == 0 and torch.count_nonzero(dv).item() == 0
    device_clean()


def test_training_steps_with_merge_schedule_match_oracle():
    # Five steps of the fp32 correctness layer with reset gap 2 (merges after steps 2 and 4).
    # The trajectory tolerance is 1e-4: each step's gradients carry fp32 rounding (~1e-6
    # relative) and AdamW divides them by their own running scale, so the relative error of an
    # update is that of its gradient; five steps and two merges compound it well below 1e-4.
    inp = I.make_workload("layer256_b32_f32")
    s = inp.shape
    desc = make_desc(s.d_in, s.d_out, s.b, s.k, s.dtype, s.mode)
    L = PoetxLayer(desc, s.n_tokens)
    L.load_state(inp.W0, inp.theta_R, inp.theta_P, inp.pi_L, inp.pi_R)
    X, dY = L.to_dev(inp.X), L.to_dev(inp.dY)
    merges = []

    def new_perms():
        perms = I.fresh_permutations(s, 1001 + len(merges))
        merges.append(perms)
        return perms

    for _ in range(5):
        L.train_step(X, dY, _cfg(), reset_gap=2, new_perms=new_perms)
    L.cnp()
    L.forward(X)
    torch.cuda.synchronize()

    W0p = O.absorb(inp.W0, inp.pi_L, inp.pi_R)
    thR, thP = inp.theta_R.astype(np.float64), inp.theta_P.astype(np.float64)
    pL, pR = inp.pi_L, inp.pi_R
    m = v = np.zeros(thR.size + thP.size)
    nR = thR.size
    k = 0
    for step, t, merge_now in O.train_schedule(5, reset_gap=2):
        _, gR, gP = O.backward_chain(inp.X, inp.dY, W0p, thR, thP, pL, pR, s.b, s.k)
        th, m, v = O.adamw_step(np.concatenate([thR.ravel(), thP.ravel()]), np.concatenate([gR.ravel(), gP.ravel()]),
                                m, v, t, CFG["lr"], CFG["gamma"], CFG["beta1"], CFG["beta2"], CFG["eps"],
                                CFG["weight_decay"])
        thR, thP = th[:nR].reshape(thR.shape), th[nR:].reshape(thP.shape)
        if merge_now:
            pL2, pR2 = merges[k]
            k += 1
            W0p, thR, thP = O.merge(W0p, thR, thP, pL, pR, pL2, pR2, s.b, s.k)
            pL, pR = pL2, pR2
            m = v = np.zeros_like(m)
    assert k == len(merges) == 2
    Y = O.forward_chain(inp.X, W0p, O.cnp(thR, s.b, s.k), O.cnp(thP, s.b, s.k), pL, pR)[0]
    tol = 1e-4
    errs = {"theta_R": rel(to_np(L.theta_R), thR), "theta_P": rel(to_np(L.theta_P), thP),
            "m": rel(to_np(L.m).ravel(), m), "v": rel(to_np(L.v).ravel(), v),
            "W0p": rel(to_np(L.W0p), W0p), "Y": rel(to_np(L.Y), Y)}
    assert all(e <= tol for e in errs.values()), errs
    assert np.array_equal(L.perm_L.cpu().numpy(), pL) and np.array_equal(L.perm_R.cpu().numpy(), pR)
    assert L.t == 1 and L.steps == 5
    device_clean()
