"""Failure detection without a GPU fault: every device-side wait of the library is bounded, and a
wait that runs out is reported through poetx_device_status().  The probe kernel waits on an
mbarrier that nothing arrives on, with a 1 ms bound; the test checks that the kernel returns,
that the status names the probe's kernel and wait site, and that the context stays usable."""
import numpy as np
import pytest
import torch

import oracle as O
import orthogonal_equivalence_cnp_b200 as P
import poetx_inputs as I
from helpers import TOL, rel, to_np
from orthogonal_equivalence_cnp_b200.layer import PoetxLayer, make_desc

pytestmark = pytest.mark.gpu


def test_bounded_wait_runs_out_and_is_reported():
    assert P.poetx_device_status()[0] == 0
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    P.poetx_test_wait_timeout(1_000_000, flag)  # 1 ms
    st, detail = P.poetx_device_status()
    assert st == 6, P.STATUS.get(st)  # POETX_ERR_DEVICE_TIMEOUT
    assert detail == (7 << 8) | 1
    assert flag.item() == 2  # the wait gave up and the kernel went on to its end
    assert P.poetx_device_status() == (0, 0)  # reading the status clears it
    # The context is still usable: a CNP launch right after is correct.
    s = I.small_shape(256, 256, 64, 3, 8, "bf16", theta_std=0.005)
    inp = I.make_layer(s, 2, with_activations=False)
    L = PoetxLayer(make_desc(256, 256, 64, 3, "bf16", "fast"), 8)
    L.load_state(inp.W0, inp.theta_R, inp.theta_P, inp.pi_L, inp.pi_R)
    L.cnp()
    torch.cuda.synchronize()
    assert P.poetx_device_status()[0] == 0
    assert rel(to_np(L.Q_R), O.cnp(inp.theta_R, 64, 3)) <= TOL["bf16"]
