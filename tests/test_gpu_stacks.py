"""The two stacked workloads at full size: the 32-block Llama-8B-shaped stack (224 linears, b = 256,
fast mode, 2048 tokens) and the 40-block Llama-13B-shaped stack (280 linears, b = 512, mem mode,
4096 tokens, each step followed by a merge with fresh permutations).

Every layer's CNP is computed on the GPU (all blocks of a transformer block in one launch) and
checked against the oracle on the first and last block of each side; the first and last
transformer blocks' linears run the full layer step and are checked on sampled tokens (the
upstream gradient is zero outside them, so the oracle needs only those rows, and the gradients,
which sum over tokens, are compared whole).  For the 13B stack each of those layers is merged
and the layer function after the merge (theta = 0, new permutations) is compared with the
oracle's forward before it.
"""
import numpy as np
import pytest
import torch

import oracle as O
import orthogonal_equivalence_cnp_b200 as P
import poetx_inputs as I
from helpers import TOL, device_clean, gpu_layer, oracle_layer, rel, to_np
from orthogonal_equivalence_cnp_b200.layer import PoetxLayer, make_desc

pytestmark = pytest.mark.gpu

STACK8 = "llama8b_stack_32x7_b256_bf16"
STACK13 = "llama13b_stack_40x7_b512_bf16_mem"


def _cnp_every_layer(name):
    layers = I.stack_layers(name)
    sh0 = layers[0][1]
    desc = make_desc(sh0.d_in, sh0.d_out, sh0.b, sh0.k, "bf16", "fast")  # b, k and dtype are used
    per_block = len(layers) // I.STACKS[name][1]
    worst = 0.0
    for start in range(0, len(layers), per_block):
        chunk = layers[start:start + per_block]
        thetas = [I.make_theta(sh, seed) for _, sh, seed in chunk]
        flat = np.concatenate([np.concatenate([tR, tP]) for tR, tP in thetas])
        n = flat.shape[0]
        theta = torch.from_numpy(flat).cuda()
        Q = torch.empty(n, sh0.b, sh0.b, dtype=torch.bfloat16, device="cuda")
        ws = torch.empty(max(P.poetx_cnp_blocks_workspace_size(desc, n), 256), dtype=torch.uint8, device="cuda")
        P.poetx_cnp_blocks(desc, n, theta, Q, ws)
        torch.cuda.synchronize()
        Qh = Q.float().cpu().numpy().astype(np.float64)
        off = 0
        for (l, sh, _), (tR, tP) in zip(chunk, thetas):
            for side_off, nb, th in ((0, sh.nb_out, tR), (sh.nb_out, sh.nb_in, tP)):
                # first and last block of each side (b = 512: one of them, alternating by layer)
                pick = [0, nb - 1] if sh.b <= 256 else [0 if l % 2 == 0 else nb - 1]
                ref = O.cnp(th[pick], sh.b, sh.k)
                e = rel(Qh[off + side_off + np.array(pick)], ref)
                worst = max(worst, e)
                assert e <= TOL["bf16"], (l, side_off, e)
            off += sh.nb_out + sh.nb_in
        assert off == n
        del theta, Q, ws
    device_clean()
    return worst


def test_llama8b_stack_cnp_every_layer():
    _cnp_every_layer(STACK8)


def test_llama13b_stack_cnp_every_layer():
    _cnp_every_layer(STACK13)


def test_stack_layer_cnp_matches_flat_batch_bitwise():
    # One layer's CNP through the layer call (both sides in one program) equals the flat batch.
    l, sh, seed = I.stack_layers(STACK8)[4]  # the gate projection, 4096 -> 14336
    tR, tP = I.make_theta(sh, seed)
    desc = make_desc(sh.d_in, sh.d_out, sh.b, sh.k, "bf16", "fast")
    L = PoetxLayer(desc, 1)
    L.theta_R.copy_(torch.from_numpy(tR))
    L.theta_P.copy_(torch.from_numpy(tP))
    L.cnp()
    flat = torch.from_numpy(np.concatenate([tR, tP])).cuda()
    n = flat.shape[0]
    Q = torch.empty(n, sh.b, sh.b, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(max(P.poetx_cnp_blocks_workspace_size(desc, n), 256), dtype=torch.uint8, device="cuda")
    P.poetx_cnp_blocks(desc, n, flat, Q, ws)
    torch.cuda.synchronize()
    assert torch.equal(Q[:sh.nb_out], L.Q_R) and torch.equal(Q[sh.nb_out:], L.Q_P)
    device_clean()


def _sampled_layers(name):
    layers = I.stack_layers(name)
    per_block = len(layers) // I.STACKS[name][1]
    return layers[:per_block] + layers[-per_block:]


def _check_sampled(g, o, rows):
    errs = {"Y": rel(g["Y"][rows], o["Y"]), "dX": rel(g["dX"][rows], o["dX"]),
            "g_R": rel(g["g_R"], o["g_R"]), "g_P": rel(g["g_P"], o["g_P"]),
            "Q_R": rel(g["Q_R"], o["Q_R"]), "Q_P": rel(g["Q_P"], o["Q_P"])}
    assert all(e <= TOL["bf16"] for e in errs.values()), errs
    return errs


@pytest.mark.parametrize("idx", range(14))
def test_llama8b_stack_first_and_last_block_layers(idx):
    l, sh, seed = _sampled_layers(STACK8)[idx]
    inp = I.make_layer(sh, seed)
    rows = np.sort(np.random.default_rng(seed).choice(sh.n_tokens, 16, replace=False))
    g, _ = gpu_layer(inp, dY_rows=rows)
    device_clean()
    _check_sampled(g, oracle_layer(inp, rows=rows), rows)


@pytest.mark.parametrize("idx", range(14))
def test_llama13b_stack_first_and_last_block_layers_then_merge(idx):
    l, sh, seed = _sampled_layers(STACK13)[idx]
    inp = I.make_layer(sh, seed)
    rows = np.sort(np.random.default_rng(seed).choice(sh.n_tokens, 16, replace=False))
    g, L = gpu_layer(inp, dY_rows=rows)
    o = oracle_layer(inp, rows=rows)
    _check_sampled(g, o, rows)
    # Merge with fresh permutations (Q is the one the forward used), then the forward with
    # theta = 0 must reproduce the oracle's pre-merge forward on the sampled tokens.
    pL2, pR2 = I.fresh_permutations(sh, seed)
    L.merge(torch.from_numpy(pL2).cuda(), torch.from_numpy(pR2).cuda())
    torch.cuda.synchronize()
    assert torch.count_nonzero(L.theta_R).item() == 0 and torch.count_nonzero(L.theta_P).item() == 0
    L.cnp()
    X = L.to_dev(inp.X)
    L.forward(X)
    torch.cuda.synchronize()
    e = rel(to_np(L.Y)[rows], o["Y"])
    assert e <= TOL["bf16"], e
    del L, X
    device_clean()
