"""Data-parallel gradient buckets (orthogonal_equivalence_cnp_b200.ddp) on CPU: two gloo ranks
(world size 2, 127.0.0.1) and the host-side bucket plan.

The packed-gradient layout is the real one: every linear of the 32-block Llama-8B-shaped stack
keeps theta_R then theta_P gradients back to back, b(b-1)/2 floats per block, in one flat buffer
in forward order; the backward pass reports the linears in reverse order.  A scale factor keeps
the buffer small on CPU (every layer keeps its relative size).
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import poetx_inputs as I  # noqa: E402
from orthogonal_equivalence_cnp_b200.ddp import plan_buckets  # noqa: E402

STACK8 = "llama8b_stack_32x7_b256_bf16"


def _layer_sizes(scale=1):
    return [(sh.nb_out + sh.nb_in) * sh.n_packed // scale for _, sh, _ in I.stack_layers(STACK8)]


def test_bucket_plan_covers_every_layer_once_in_backward_order():
    sizes = _layer_sizes()
    assert len(sizes) == 224 and sum(sizes) == 10240 * 256 * 255 // 2
    buckets = plan_buckets(sizes, 25 << 20)
    seen = [l for lo, hi in buckets for l in range(lo, hi)]
    assert sorted(seen) == list(range(224))
    assert buckets[0][1] == 224 and buckets[-1][0] == 0  # the last layers' bucket goes first
    for (lo, hi), (lo2, hi2) in zip(buckets, buckets[1:]):
        assert hi2 == lo  # consecutive runs, reported in reverse order
    for lo, hi in buckets[:-1]:
        assert 4 * sum(sizes[lo:hi]) >= 25 << 20
    assert plan_buckets([5], 1 << 30) == [(0, 1)]
    with pytest.raises(ValueError):
        plan_buckets([1, 2], 0)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import datetime

    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from orthogonal_equivalence_cnp_b200.ddp import GradBuckets
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    sizes = _layer_sizes(scale=64)
    flat = torch.zeros(sum(sizes), dtype=torch.float32)
    gb = GradBuckets(flat, sizes, bucket_bytes=4 * sum(sizes) // 9)
    results = []
    for step in range(2):  # the buckets re-arm after finish()
        offs = np.concatenate([[0], np.cumsum(sizes)])
        for layer in reversed(range(len(sizes))):  # the backward pass: last linear first
            # this rank's gradient of the layer (written before the layer is reported)
            flat[offs[layer]:offs[layer + 1]] = (rank + 1) * (layer + 1) + step
            gb.layer_done(layer)
        launched = list(gb.launched)
        gb.finish()
        results.append((launched, flat.numpy().copy()))
    out[rank] = [(l, a.tolist()) for l, a in results]
    dist.barrier()
    dist.destroy_process_group()


def test_two_ranks_sum_every_layer_bucket_by_bucket():
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(2, port, out), nprocs=2, start_method="spawn", join=True)
        res = dict(out)
    sizes = _layer_sizes(scale=64)
    offs = np.concatenate([[0], np.cumsum(sizes)])
    buckets = plan_buckets(sizes, 4 * sum(sizes) // 9)
    for step in range(2):
        for rank in (0, 1):
            launched, flat = res[rank][step]
            assert launched == list(range(len(buckets)))  # in backward order, each once
            flat = np.asarray(flat)
            for layer in range(len(sizes)):
                # rank 0 wrote (layer + 1) + step, rank 1 wrote 2 (layer + 1) + step
                expect = 3 * (layer + 1) + 2 * step
                assert np.all(flat[offs[layer]:offs[layer + 1]] == expect), (step, rank, layer)


def test_double_report_and_early_finish_are_errors():
    import torch
    from orthogonal_equivalence_cnp_b200.ddp import GradBuckets

    class _NoDist:  # the host logic only: no collective is issued by these calls
        class ReduceOp:
            SUM = None

    gb = GradBuckets.__new__(GradBuckets)
    gb.dist = _NoDist
    gb.flat, gb.sizes, gb.group = torch.zeros(10), [4, 6], None
    gb.offsets = [0, 4, 10]
    gb.buckets = [(1, 2), (0, 1)]
    gb.bucket_of = {1: 0, 0: 1}
    gb._reset()
    with pytest.raises(RuntimeError):
        gb.finish()  # nothing reported yet
