"""POETX_DEBUG: with the variable set, the entry points that take permutations check on the host
that they are bijections and reject a bad one before launching anything.  Run in a child
process, because the library reads the variable once per process."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

pytestmark = pytest.mark.gpu

CHILD = r"""
import torch
import orthogonal_equivalence_cnp_b200 as P
from orthogonal_equivalence_cnp_b200.layer import make_desc
d = make_desc(512, 256, 64, 3, "bf16", "fast")
W0 = torch.randn(256, 512, device="cuda").to(torch.bfloat16)
W0p = torch.empty_like(W0)
pL = torch.randperm(256, device="cuda").to(torch.int32)
pR = torch.randperm(512, device="cuda").to(torch.int32)
P.poetx_absorb(d, W0, pL, pR, W0p)                 # bijections: accepted
torch.cuda.synchronize()
assert torch.equal(W0p, W0[pL.long()][:, pR.long()])
bad = pR.clone()
bad[7] = bad[3]                                     # a repeated index
before = P.poetx_launch_count()
try:
    P.poetx_absorb(d, W0, pL, bad, W0p)
    raise SystemExit("bad permutation accepted")
except P.PoetxError as e:
    assert e.status == 1, e.status
assert P.poetx_launch_count() == before             # nothing was launched
print("debug checks ok")
"""


def test_debug_mode_rejects_a_repeated_index():
    env = dict(os.environ, POETX_DEBUG="1")
    r = subprocess.run([sys.executable, "-c", CHILD], capture_output=True, text=True, env=env, cwd=ROOT, timeout=300)
    assert r.returncode == 0 and "debug checks ok" in r.stdout, r.stdout + r.stderr[-2000:]
