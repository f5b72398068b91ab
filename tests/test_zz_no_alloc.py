"""The allocation-free CNP entry point (poetx_cnp_blocks_noalloc) against the workspace one and
against the oracle.

poetx_cnp_blocks_noalloc serves callers that cannot give the library device scratch (a plugin
inside a framework that owns every device allocation, a loop that must never call cudaMalloc):
where the CNP forward needs scratch (fp32, b = 512) it uses a fixed 32 MiB array built into the
library.  This file is named so that pytest collects it last; it must pass on its own in a fresh
process and after the rest.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle as O
import orthogonal_equivalence_cnp_b200 as P
import poetx_inputs as I
from helpers import TOL, device_clean, rel, to_np
from orthogonal_equivalence_cnp_b200.layer import make_desc

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype,b,nblocks", [("bf16", 256, 85), ("bf16", 128, 20), ("bf16", 512, 9), ("f32", 32, 24)])
def test_noalloc_matches_workspace_entry_point_twice(dtype, b, nblocks):
    desc = make_desc(b, b, b, 3, dtype, "fast")
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    ws = torch.empty(max(P.poetx_cnp_blocks_workspace_size(desc, nblocks), 256), dtype=torch.uint8, device="cuda")
    rng = np.random.default_rng(b + nblocks)
    for call in range(2):  # two calls in a row: the second must not see the first one's scratch
        theta = torch.from_numpy(
            rng.normal(0, 0.005 if dtype == "bf16" else 0.05, (nblocks, b * (b - 1) // 2)).astype(np.float32)).cuda()
        Q_ref = torch.full((nblocks, b, b), float("nan"), dtype=tdt, device="cuda")
        Q_na = torch.full((nblocks, b, b), float("nan"), dtype=tdt, device="cuda")
        P.poetx_cnp_blocks(desc, nblocks, theta, Q_ref, ws)
        P.poetx_cnp_blocks_noalloc(desc, nblocks, theta, Q_na)
        torch.cuda.synchronize()
        device_clean()
        assert torch.isfinite(Q_na.float()).all()
        assert rel(to_np(Q_na), to_np(Q_ref)) <= TOL[dtype], call
        assert rel(to_np(Q_na), O.cnp(theta.cpu().numpy(), b, 3)) <= TOL[dtype], call


def test_noalloc_rejects_more_than_its_scratch():
    desc = make_desc(512, 512, 512, 3, "bf16", "fast")
    assert P.poetx_cnp_blocks_workspace_size(desc, 9) <= 32 << 20 < P.poetx_cnp_blocks_workspace_size(desc, 10)
    theta = torch.zeros(10, 512 * 511 // 2, dtype=torch.float32, device="cuda")
    Q = torch.empty(10, 512, 512, dtype=torch.bfloat16, device="cuda")
    st = P.lib().poetx_cnp_blocks_noalloc(ctypes.byref(desc), 10, theta.data_ptr(), Q.data_ptr(),
                                           torch.cuda.current_stream().cuda_stream)
    assert st == 4  # POETX_ERR_WORKSPACE: beyond the built-in 32 MiB, nothing launched
