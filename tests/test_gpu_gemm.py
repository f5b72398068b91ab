"""The batched GEMM core (tcgen05 bf16 path and fp32 SIMT path) against a plain PyTorch fp32 matmul
of the same operands, for every operand layout, tile width, batching, split-K and epilogue."""
import math

import numpy as np
import pytest
import torch

import orthogonal_equivalence_cnp_b200 as P
from helpers import device_clean

pytestmark = pytest.mark.gpu


def _view(mem, z, zrow, zcol, mn, ext_mn, ext_k):
    if not mn:
        return mem[z * zrow: z * zrow + ext_mn, z * zcol: z * zcol + ext_k]
    return mem[z * zrow: z * zrow + ext_k, z * zcol: z * zcol + ext_mn].t()


def _run(dtype, M, N, K, batch=1, splits=1, a_mn=0, b_mn=0, a_shape=None, b_shape=None, a_z=(0, 0), b_z=(0, 0),
         d_z=None, alpha=1.0, beta=0.0, with_c=False, diag=0, d_dtype=P.POETX_F32, seed=0):
    g = torch.Generator(device="cuda").manual_seed(seed)
    tdt = torch.bfloat16 if dtype == P.POETX_BF16 else torch.float32
    if a_shape is None:
        a_shape = (K, M) if a_mn else (M, K)
    if b_shape is None:
        b_shape = (K, N) if b_mn else (N, K)
    A = torch.randn(a_shape, device="cuda", generator=g).to(tdt)
    B = torch.randn(b_shape, device="cuda", generator=g).to(tdt)
    if d_z is None:
        d_z = (M, 0)
    d_rows = (batch - 1) * d_z[0] + M
    d_cols = (batch - 1) * d_z[1] + N
    odt = torch.bfloat16 if d_dtype == P.POETX_BF16 else torch.float32
    D = torch.full((splits, d_rows, d_cols), float("nan"), device="cuda", dtype=odt)
    C = torch.randn(d_rows, d_cols, device="cuda", generator=g) if with_c else None
    P.poetx_test_gemm(dtype, M, N, K, batch, splits, A, a_shape[0], a_shape[1], a_shape[1], a_z[0], a_z[1], a_mn,
                      B, b_shape[0], b_shape[1], b_shape[1], b_z[0], b_z[1], b_mn, D, d_dtype, d_cols, d_z[0],
                      d_z[1], d_rows * d_cols, alpha, beta, C, d_cols if with_c else 0, d_z[0], d_z[1], diag)
    torch.cuda.synchronize()
    device_clean()
    Af, Bf = A.float(), B.float()
    worst = 0.0
    total = D.float().sum(0) if not with_c and not diag else None
    for z in range(batch):
        a = _view(Af, z, *a_z, a_mn, M, K)
        b = _view(Bf, z, *b_z, b_mn, N, K)
        ref = alpha * (a @ b.t())
        rs, cs = slice(z * d_z[0], z * d_z[0] + M), slice(z * d_z[1], z * d_z[1] + N)
        if splits == 1:
            got = D[0, rs, cs].float()
            if with_c:
                ref = ref + beta * C[rs, cs]
            if diag:
                ref = ref + torch.eye(M, N, device="cuda")
        else:
            got = total[rs, cs]
        err = ((got - ref).norm() / ref.norm()).item()
        worst = max(worst, err)
    return worst


TOL_F32_OUT = 1e-5


@pytest.mark.parametrize("dtype", [P.POETX_BF16, P.POETX_F32])
@pytest.mark.parametrize("a_mn,b_mn", [(0, 0), (0, 1), (1, 0), (1, 1)])
@pytest.mark.parametrize("N", [64, 128, 256, 512])
def test_plain_layouts(dtype, a_mn, b_mn, N):
    assert _run(dtype, 200, N, 320, a_mn=a_mn, b_mn=b_mn) <= TOL_F32_OUT


@pytest.mark.parametrize("dtype", [P.POETX_BF16, P.POETX_F32])
def test_block_diagonal_forward_shape(dtype):
    # V[:, blk z] = U[:, blk z] Q_z^T: A = U [n, d] batched along columns, B = Q [nb*b, b] along rows.
    n, b, nb = 300, 128, 4
    assert _run(dtype, n, b, b, batch=nb, a_shape=(n, nb * b), a_z=(0, b), b_shape=(nb * b, b), b_z=(b, 0),
                d_z=(0, b)) <= TOL_F32_OUT


@pytest.mark.parametrize("dtype", [P.POETX_BF16, P.POETX_F32])
def test_block_diagonal_adjoint_shape(dtype):
    n, b, nb = 257, 256, 2
    assert _run(dtype, n, b, b, batch=nb, a_shape=(n, nb * b), a_z=(0, b), b_mn=1, b_shape=(nb * b, b), b_z=(b, 0),
                d_z=(0, b)) <= TOL_F32_OUT


@pytest.mark.parametrize("dtype", [P.POETX_BF16, P.POETX_F32])
@pytest.mark.parametrize("splits", [1, 3])
def test_block_gradient_shape(dtype, splits):
    # G_z = L[:, blk z]^T R[:, blk z] with K = tokens (ragged), split-K partials summed.
    n, b, nb = 333, 128, 3
    assert _run(dtype, b, b, n, batch=nb, splits=splits, a_mn=1, b_mn=1, a_shape=(n, nb * b), a_z=(0, b),
                b_shape=(n, nb * b), b_z=(0, b), d_z=(b, 0)) <= TOL_F32_OUT


@pytest.mark.parametrize("dtype", [P.POETX_BF16, P.POETX_F32])
def test_epilogue_alpha_beta_diag(dtype):
    assert _run(dtype, 256, 256, 256, batch=2, a_shape=(512, 256), a_z=(256, 0), b_mn=1, b_shape=(512, 256),
                b_z=(256, 0), d_z=(256, 0), alpha=-0.5, beta=2.0, with_c=True, diag=1) <= TOL_F32_OUT


def test_bf16_output_rounding():
    err = _run(P.POETX_BF16, 256, 256, 512, d_dtype=P.POETX_BF16)
    assert err <= 2.0 ** -8
