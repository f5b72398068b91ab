"""The N > 1 path of bench.py on CPU: two gloo ranks (world size 2, 127.0.0.1).

Each rank runs an independent replica on its own tokens (data parallel over tokens); the
timing is the max over ranks and the reported value counts the tokens of all ranks.
"""
import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import datetime

    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    r, w, _ = bench.dist_env()
    local_ms = 10.0 + 5.0 * rank                     # rank 1 is the slow one
    t_max = bench.max_over_ranks(local_ms, w)        # what rank 0 reports
    seed = bench.shard_seed(1002, r)
    # the exchange step: packed gradients (theta_R then theta_P, back to back) summed over ranks
    g = torch.arange(12, dtype=torch.float32).reshape(3, 4) * (rank + 1)
    bench.dp_allreduce(g, w)
    summed = g.clone()
    # the same collective steps on every rank, including after the reduction
    dist.barrier()
    out[rank] = (r, w, t_max, seed, summed.numpy().tolist())
    dist.destroy_process_group()


def test_two_ranks_max_over_ranks_and_token_shards():
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(2, port, out), nprocs=2, start_method="spawn", join=True)
        res = dict(out)
    assert res[0][:3] == (0, 2, 15.0) and res[1][:3] == (1, 2, 15.0)
    assert res[0][3] != res[1][3]  # each rank draws its own tokens
    expect = (np.arange(12, dtype=np.float32).reshape(3, 4) * 3).tolist()  # rank 0 (x1) + rank 1 (x2)
    assert res[0][4] == expect and res[1][4] == expect
    sys.path.insert(0, ROOT)
    import bench
    import poetx_inputs as I
    s = I.WORKLOADS["llama8b_attn_4096_b256_bf16"]
    # weak scaling: the value counts every rank's tokens over the slowest rank's time
    value = 2 * s.n_tokens * 100 / (15.0 / 1e3)
    assert value == pytest.approx(2 * 2048 * 100 / 0.015)
    assert bench.step_flops(s)["total"] == 2 * 2048 * 4096 * 4096 * 2 + 2 * 2048 * 256 * 8192 + 4 * 2048 * 256 * 8192 \
        + 32 * 3 * 256 ** 3 + 32 * 12 * 256 ** 3


def test_reference_arm_under_torchrun_two_ranks_prints_one_line():
    port = _free_port()
    env = dict(os.environ, OMP_NUM_THREADS="2", OPENBLAS_NUM_THREADS="2")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3",
           "--workload", "layer256_b32_f32"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, env=env, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"


def test_reference_arm_single_process_json_line():
    # N = 1 without torchrun: one JSON line with the contract's keys, the oracle as the arm.
    env = dict(os.environ, OMP_NUM_THREADS="2", OPENBLAS_NUM_THREADS="2")
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "2", "--warmup", "3",
           "--workload", "layer256_b32_f32"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, env=env, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "dtype", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["n_gpus"] == 1 and d["steps"] == 2 and d["warmup"] == 3
    assert d["value"] > 0 and d["higher_is_better"] is True and d["config"]["workload"] == "layer256_b32_f32"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
