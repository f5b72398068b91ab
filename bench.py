#!/usr/bin/env python
"""Benchmark of the POET-X layer step on B200: tokens/s and TFLOP/s against the bf16 roofline.

A step is one pass of the whole hot path over one batch of synthetic tokens: CNP forward of
both sides, layer forward, layer backward (including the CNP adjoint that writes the packed
gradients).  Default workload: the Llama-8B attention projection (4096 x 4096, b = 256, k = 3,
2048 tokens, bf16, fast mode), the single-layer configuration the POET-X pages time (SAI
replication review, "Reproducibility & code", first item).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl poetx|reference] [--workload NAME]

Multi-GPU (torchrun, one process per GPU): each rank runs an independent replica of the layer on
its own tokens (data parallel, weak scaling); no collective is on the timed path.  Timing: CUDA
events around each step on the launching stream, an L2 flush (256 MiB write) between steps
outside the timed intervals, barrier + synchronize around the timed region, max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import poetx_inputs as I  # noqa: E402

DEFAULT_WORKLOAD = "llama8b_attn_4096_b256_bf16"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}
METRIC = "POET-X linear fwd+bwd tokens/s & TFLOP/s (4096², b=256) vs bf16 roofline"


# ------------------------------------------------------------------------------ work model
def step_flops(s: I.LayerShape) -> dict:
    """Algorithmic FLOPs of one step (what the method must compute; W0 is frozen, no dW0).

    fwd = 2N d_in d_out + 2N b (d_in + d_out); bwd = 2N d_in d_out + 4N b (d_in + d_out)
    (+ 2N d_in d_out + 2N b d_in recomputed in mem mode); CNP fwd = nb k b^3 (each power of a
    skew block is symmetric or skew, so half of each product is needed); CNP adjoint = nb 2k 2b^3."""
    N, di, do, b, k = s.n_tokens, s.d_in, s.d_out, s.b, s.k
    nb = s.nb_in + s.nb_out
    fwd = 2 * N * di * do + 2 * N * b * (di + do)
    bwd = 2 * N * di * do + 4 * N * b * (di + do)
    if s.mode == "mem":
        bwd += 2 * N * di * do + 2 * N * b * di
    cnp = nb * k * b ** 3 + nb * 2 * k * 2 * b ** 3
    return {"fwd": fwd, "bwd": bwd, "cnp": cnp, "total": fwd + bwd + cnp}


# DRAM bytes (read + write) of one W0' launch, from one ncu capture of this kernel build on the
# bench workload (mean of two forward and two adjoint launches).  Only valid for that workload
# and that kernel build; None otherwise.
W_GEMM_TRAFFIC = {"llama8b_attn_4096_b256_bf16": 52.478e6 + 0.899e6}


def w_gemm_flops(s: I.LayerShape) -> int:
    """Algorithmic FLOPs of one launch of the dominant kernel, the W0' GEMM (Z = V W0'^T or
    dV = dZ W0'); for bf16 and b = 256 that launch also applies the block factor on its output
    side (Y'_i = Z_i Q_R,i^T: 2 N d_out b more; dU_i = dV_i Q_P,i: 2 N d_in b more).  Returned
    per launch, averaged over the forward and the backward launch."""
    f = 2 * s.n_tokens * s.d_in * s.d_out
    if s.dtype == "bf16" and s.b == 256:
        f += s.n_tokens * s.b * (s.d_in + s.d_out)
    return f


def read_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        d["source"] = "measured"
        return d
    return dict(FALLBACK_PEAKS)


# --------------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""
    QUERY = ("uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, period_ms: int = 100):
        self.period_ms = period_ms
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="poetx_clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits", f"-lms", str(self.period_ms),
                 "-f", self.path], stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self, uuid: str) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9 or (uuid and not parts[0].lower().endswith(uuid.lower())):
                    continue
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower().startswith("active")})
        pw = [float(r[3]) for r in rows if r[3].replace(".", "").isdigit()]
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows), "power_w_max": max(pw) if pw else None}


def gpu_uuid(dev) -> str:
    import torch
    try:
        return str(torch.cuda.get_device_properties(dev).uuid).replace("GPU-", "")
    except Exception:
        return ""


def count_step_launches(P, layer, X, dY) -> int:
    """Kernels the library launches in one step (counted on a directly launched step)."""
    import torch
    n0 = P.poetx_launch_count()
    layer.step(X, dY)
    torch.cuda.synchronize()
    return P.poetx_launch_count() - n0


# ---------------------------------------------------------------------------- distributed
def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def max_over_ranks(value: float, world: int, device=None) -> float:
    """Max of a per-rank scalar over all ranks (identity for one rank)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def dp_allreduce(grad, world: int) -> None:
    """The exchange step of data-parallel training: sum the packed theta gradients of all ranks
    in place (theta_R and theta_P are stored back to back, so one collective moves both)."""
    if world <= 1:
        return
    import torch.distributed as dist
    dist.all_reduce(grad, op=dist.ReduceOp.SUM)


def shard_seed(base_seed: int, rank: int) -> int:
    """Each rank draws its own tokens (the layer state is shared by construction)."""
    return base_seed + 7919 * rank


# ------------------------------------------------------------------------------ CPU oracle
def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [d.get("num_threads", 0) for d in threadpool_info() if d.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def oracle_step(inp: I.LayerInputs, W0p, n_tok: int):
    """The float64 oracle's layer step on the first n_tok tokens (CNP, forward, backward + CNP
    adjoint); W0' is layer state, absorbed once by the caller (as on the GPU)."""
    import oracle as O
    s = inp.shape
    X, dY = inp.X[:n_tok], inp.dY[:n_tok]
    Q_R, Q_P = O.cnp(inp.theta_R, s.b, s.k), O.cnp(inp.theta_P, s.b, s.k)
    O.forward_chain(X, W0p, Q_R, Q_P, inp.pi_L, inp.pi_R)
    O.backward_chain(X, dY, W0p, inp.theta_R, inp.theta_P, inp.pi_L, inp.pi_R, s.b, s.k)


def measure_xq(s, src, X, dY, flush, stream, world, dev, use_graph, Kx):
    """POET-XQ beside POET-Xmem on the same layer state: one mem-mode layer with the bf16 W0' and
    one with W0' quantised to int8 codes and per-row scales (the W0' GEMMs dequantise in shared
    memory).  Each step is captured and timed like the headline step (L2 flushed between steps,
    outside the intervals), then replayed once more with the library's per-launch events to get
    the W0' GEMM launch times."""
    import torch

    import orthogonal_equivalence_cnp_b200 as P
    from orthogonal_equivalence_cnp_b200.layer import PoetxLayer, make_desc
    res = {}
    for name in ("mem_bf16", "xq"):
        L = PoetxLayer(make_desc(s.d_in, s.d_out, s.b, s.k, "bf16", "mem"), s.n_tokens, device=dev)
        L.W0p.copy_(src.W0p)
        L.theta.copy_(src.theta)
        L.perm_L.copy_(src.perm_L)
        L.perm_R.copy_(src.perm_R)
        if name == "xq":
            L.quantize()
        for _ in range(3):
            L.step(X, dY)
        torch.cuda.synchronize()
        g = None
        if use_graph:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                L.step(X, dY)
        e0 = [torch.cuda.Event(enable_timing=True) for _ in range(Kx)]
        e1 = [torch.cuda.Event(enable_timing=True) for _ in range(Kx)]
        for i in range(Kx):
            flush.zero_()
            e0[i].record(stream)
            if g is not None:
                g.replay()
            else:
                L.step(X, dY)
            e1[i].record(stream)
        torch.cuda.synchronize()
        res[f"{name}_ms_per_step"] = round(max_over_ranks(sum(e0[i].elapsed_time(e1[i]) for i in range(Kx)),
                                                          world, dev) / Kx, 4)
        prof = {}
        for i in range(min(Kx, 50)):
            flush.zero_()
            P.poetx_profile_enable(True)
            L.step(X, dY)
            P.poetx_profile_enable(False)
            torch.cuda.synchronize()
            for k, (n, ms) in P.poetx_profile_summary().items():
                c = prof.get(k, (0, 0.0))
                prof[k] = (c[0] + n, c[1] + ms)
        for cls, tag in (("w_gemm", "w_gemm_launch_ms"), ("w_gemm_adj", "w_gemm_adj_launch_ms")):
            n, ms = prof.get(cls, (0, 0.0))
            res[f"{name}_{tag}"] = round(ms / max(n, 1), 4)
        st, det = P.poetx_device_status()
        if st != 0:
            raise RuntimeError(f"device-side timeout in the POET-XQ measurement ({det:#x})")
        del g, L
    res["w0p_bytes_bf16"] = 2 * s.d_out * s.d_in
    res["w0p_bytes_xq"] = s.d_out * s.d_in + 4 * s.d_out
    res["xq_over_mem_bf16_time"] = round(res["xq_ms_per_step"] / res["mem_bf16_ms_per_step"], 3)
    res["what"] = ("POET-Xmem step (CNP, forward, backward with recompute) with W0' in bf16 vs. int8 codes + "
                   "per-row fp32 scales dequantised inside the W0' GEMMs (three W0' launches per step: forward, "
                   "recompute, adjoint)")
    return res


def cpu_baseline(inp: I.LayerInputs, budget_s: float = 20.0) -> dict:
    import oracle as O
    W0p = O.absorb(inp.W0, inp.pi_L, inp.pi_R)
    n = inp.X.shape[0]
    t0 = time.perf_counter()
    oracle_step(inp, W0p, n)
    t1 = time.perf_counter()
    reps, total = 1, t1 - t0
    while total + (t1 - t0) <= budget_s and reps < 5:
        t2 = time.perf_counter()
        oracle_step(inp, W0p, n)
        total += time.perf_counter() - t2
        reps += 1
    return {"value": reps * n / total, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"{reps} full oracle step(s) of the workload ({n} tokens each, float64 numpy), "
                      f"{total:.1f} s"}


# ------------------------------------------------------------------------------ main arm
def run_poetx(args):
    import torch
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)

    import orthogonal_equivalence_cnp_b200 as P
    from orthogonal_equivalence_cnp_b200.layer import PoetxLayer, make_desc

    s = I.WORKLOADS[args.workload]
    seed = I.WORKLOAD_SEEDS[args.workload]
    state = I.make_layer(s, seed, with_activations=False)
    acts = I.make_layer(s, shard_seed(seed, rank))
    layer = PoetxLayer(make_desc(s.d_in, s.d_out, s.b, s.k, s.dtype, s.mode), s.n_tokens, device=dev)
    layer.load_state(state.W0, state.theta_R, state.theta_P, state.pi_L, state.pi_R)
    X, dY = layer.to_dev(acts.X), layer.to_dev(acts.dY)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    for _ in range(args.warmup):
        layer.step(X, dY)
        dp_allreduce(layer.grad, world)
    torch.cuda.synchronize()
    st, det = P.poetx_device_status()
    if st != 0:
        raise RuntimeError(f"device-side timeout during warm-up ({det:#x})")

    K = args.steps
    # One step captured into a CUDA graph and replayed: launch-bound sequences of short kernels
    # run without host overhead between them (every kernel of the step is one of ours).
    graph = None
    if not args.no_graph:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            layer.step(X, dY)
        graph.replay()
        torch.cuda.synchronize()

    def run_step():
        if graph is not None:
            graph.replay()
        else:
            layer.step(X, dY)
        dp_allreduce(layer.grad, world)  # N > 1: the packed gradients are summed over ranks

    ev0 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ev1 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    clocks = ClockSampler()
    clocks.start()
    time.sleep(0.3)
    barrier()
    torch.cuda.synchronize()
    launches0 = P.poetx_launch_count()
    step_launches = count_step_launches(P, layer, X, dY) if graph is not None else None
    for i in range(K):
        flush.zero_()
        ev0[i].record(stream)
        run_step()
        ev1[i].record(stream)
    torch.cuda.synchronize()
    barrier()
    launches = P.poetx_launch_count() - launches0 if graph is None else step_launches * K
    clk = clocks.stop(gpu_uuid(dev))
    times = [ev0[i].elapsed_time(ev1[i]) for i in range(K)]
    t_ms = max_over_ranks(sum(times), world, dev)
    st, det = P.poetx_device_status()
    if st != 0:
        raise RuntimeError(f"device-side timeout in the timed region ({det:#x})")

    # Live per-kernel durations: a graph of one step captured with the library's CUDA-event pair
    # around every launch, replayed K times (separate pass, so the headline timing carries no
    # bookkeeping); per-class device time is read back after each replay.
    P.poetx_profile_enable(True)
    if graph is not None:
        pgraph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(pgraph):
            layer.step(X, dY)
    P.poetx_profile_enable(False)
    prof = {}
    for i in range(K):
        flush.zero_()
        if graph is not None:
            pgraph.replay()
        else:
            P.poetx_profile_enable(True)
            layer.step(X, dY)
            P.poetx_profile_enable(False)
        torch.cuda.synchronize()
        for k, (n, ms) in P.poetx_profile_summary().items():
            c = prof.get(k, (0, 0.0))
            prof[k] = (c[0] + n, c[1] + ms)
    if graph is not None:
        del pgraph

    # End to end through the public API with host buffers, as a training loop runs it: every step
    # copies its X and dY from pinned host memory and reads its result (the packed gradients of
    # theta_R and theta_P) back to pinned host memory.  The copies run on their own streams so
    # that step i+1's inputs cross PCIe while step i computes (device inputs double-buffered, one
    # captured step per buffer; the gradients are staged on the device before their read-back).
    # The L2 flush runs before every step's compute, inside the timed interval.
    hX = torch.from_numpy(acts.X).to(layer.dtype).pin_memory()
    hdY = torch.from_numpy(acts.dY).to(layer.dtype).pin_memory()
    h_gR = torch.empty(layer.g_R.shape, dtype=torch.float32).pin_memory()
    h_gP = torch.empty(layer.g_P.shape, dtype=torch.float32).pin_memory()
    Xb = [torch.empty_like(X) for _ in range(2)]
    dYb = [torch.empty_like(dY) for _ in range(2)]
    gRs = [torch.empty_like(layer.g_R) for _ in range(2)]
    gPs = [torch.empty_like(layer.g_P) for _ in range(2)]
    egraphs = []
    if graph is not None:
        for j in range(2):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                layer.step(Xb[j], dYb[j])
            egraphs.append(g)
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    Ke = K
    ev_in = [torch.cuda.Event() for _ in range(Ke)]
    ev_done = [torch.cuda.Event() for _ in range(Ke)]
    ev_read = [torch.cuda.Event() for _ in range(Ke)]
    t_beg, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def h2d(i):
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(ev_done[i - 2])  # step i-2 no longer reads this buffer
            Xb[i % 2].copy_(hX, non_blocking=True)
            dYb[i % 2].copy_(hdY, non_blocking=True)
            ev_in[i].record(s_in)

    barrier()
    torch.cuda.synchronize()
    t_beg.record(stream)
    s_in.wait_stream(stream)
    s_out.wait_stream(stream)
    h2d(0)
    for i in range(Ke):
        if i + 1 < Ke:
            h2d(i + 1)
        stream.wait_event(ev_in[i])
        if i >= 2:
            stream.wait_event(ev_read[i - 2])  # the staged gradients of step i-2 have been read
        flush.zero_()
        if egraphs:
            egraphs[i % 2].replay()
        else:
            layer.step(Xb[i % 2], dYb[i % 2])
        dp_allreduce(layer.grad, world)
        gRs[i % 2].copy_(layer.g_R)
        gPs[i % 2].copy_(layer.g_P)
        ev_done[i].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_done[i])
            h_gR.copy_(gRs[i % 2], non_blocking=True)
            h_gP.copy_(gPs[i % 2], non_blocking=True)
            ev_read[i].record(s_out)
    stream.wait_stream(s_in)
    stream.wait_stream(s_out)
    t_end.record(stream)
    torch.cuda.synchronize()
    barrier()
    te_ms = max_over_ranks(t_beg.elapsed_time(t_end), world, dev)
    del egraphs
    h2d = hX.numel() * hX.element_size() + hdY.numel() * hdY.element_size()
    d2h = h_gR.numel() * 4 + h_gP.numel() * 4
    if not np.array_equal(h_gR.numpy(), layer.g_R.cpu().numpy()):
        raise RuntimeError("end-to-end read-back differs from the device gradients")

    # The optimiser on the packed theta (AdamW, both sides in one launch): HBM bound, 28 bytes per
    # parameter (theta, g, m, v read; theta, m, v written).  Timed per launch with CUDA events,
    # L2 flushed before each launch, on the layer's own state (the trained theta is not reused).
    adam = P.poetx_adamw_cfg(1e-3, 0.5, 0.9, 0.999, 1e-8, 0.0)
    th_save = layer.theta.clone()
    n_par = layer.theta.numel()
    Ko = min(K, 200)
    oe0 = [torch.cuda.Event(enable_timing=True) for _ in range(Ko)]
    oe1 = [torch.cuda.Event(enable_timing=True) for _ in range(Ko)]
    for _ in range(3):
        P.poetx_adamw_step(adam, n_par, 1, layer.theta, layer.grad, layer.m, layer.v)
    clean = torch.ones(64 * 1024 * 1024, dtype=torch.int32, device=dev)  # 256 MiB, never written again
    for i in range(Ko):
        flush.zero_()
        clean.sum()  # reading clean data evicts the flush's dirty lines before the timed launch
        oe0[i].record(stream)
        P.poetx_adamw_step(adam, n_par, i + 1, layer.theta, layer.grad, layer.m, layer.v)
        oe1[i].record(stream)
    torch.cuda.synchronize()
    opt_ms = statistics.median(oe0[i].elapsed_time(oe1[i]) for i in range(Ko))
    del clean
    layer.theta.copy_(th_save)
    P.poetx_adamw_reset(n_par, layer.m, layer.v)
    torch.cuda.synchronize()

    # Comparator: the same step in the weight-centric order (form W = R W0 P first, then dense
    # products), captured and timed the same way (L2 flushed between steps, outside the interval).
    wc_ms = fp_ms = None

    def time_variant(fn):
        """A comparator step captured and timed like the headline step (L2 flushed between steps,
        outside the intervals)."""
        fn(X, dY)
        torch.cuda.synchronize()
        vgraph = None
        if graph is not None:
            vgraph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(vgraph):
                fn(X, dY)
        Kc = min(K, 200)
        we0 = [torch.cuda.Event(enable_timing=True) for _ in range(Kc)]
        we1 = [torch.cuda.Event(enable_timing=True) for _ in range(Kc)]
        for i in range(Kc):
            flush.zero_()
            we0[i].record(stream)
            if vgraph is not None:
                vgraph.replay()
            else:
                fn(X, dY)
            we1[i].record(stream)
        torch.cuda.synchronize()
        del vgraph
        return max_over_ranks(sum(we0[i].elapsed_time(we1[i]) for i in range(Kc)), world, dev) / Kc

    if args.comparator:
        wc_ms = time_variant(layer.wc_step)
        if s.mode == "fast":
            fp_ms = time_variant(layer.fourperm_step)

    xq = None
    if args.xq and s.dtype == "bf16" and s.d_in % 256 == 0 and s.d_out % 256 == 0:
        xq = measure_xq(s, layer, X, dY, flush, stream, world, dev, graph is not None, min(K, 200))

    fl = step_flops(s)
    value = world * s.n_tokens * K / (t_ms / 1e3)
    tflops = world * fl["total"] * K / (t_ms / 1e3) / 1e12
    peaks = read_peaks()
    # Both W0' launches of the step: the forward one (alone on the GPU) and the adjoint one (which
    # shares the GPU with theta_R's gradient GEMM on the side stream); the roofline uses their
    # average duration.
    fcnt, fms = prof["w_gemm"]
    acnt, ams = prof.get("w_gemm_adj", (0, 0.0))
    wcnt, wms = fcnt + acnt, fms + ams
    w_avg_ms = wms / max(wcnt, 1)
    achieved = w_gemm_flops(s) / (w_avg_ms / 1e3) / 1e12
    peak = float(peaks["bf16_tflops"])
    total_prof_ms = sum(v[1] for v in prof.values())
    # The CNP against HBM: algorithmic bytes per launch (forward: theta read, bf16 Q written;
    # adjoint: G = dL/dQ read as fp32, theta read, packed gradients written).
    nbt, Pk = s.nb_in + s.nb_out, s.b * (s.b - 1) // 2
    cnp_bytes = {"cnp_gemm": nbt * (4 * Pk + 2 * s.b * s.b), "cnp_adj": nbt * (4 * s.b * s.b + 8 * Pk)}
    cnp = {}
    for cls, tag in (("cnp_gemm", "fwd"), ("cnp_adj", "adj")):
        n_c, ms_c = prof.get(cls, (0, 0.0))
        if n_c:
            us = 1e3 * ms_c / n_c
            cnp[f"{tag}_us"] = round(us, 2)
            cnp[f"{tag}_bytes"] = cnp_bytes[cls]
            cnp[f"{tag}_hbm_frac"] = round(cnp_bytes[cls] / (us * 1e-6) / 1e9 / float(peaks["hbm_gbs"]), 4)
    cnp["note"] = ("per-launch CUDA-event times inside the replayed step; algorithmic bytes; both sides of the "
                   "layer in one launch each")
    out = {
        "metric": METRIC,
        "value": round(value, 1),
        "unit": "tokens/s",
        "tflops": round(tflops, 2),
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": round(t_ms / K, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": s.dtype,
        "data": "synthetic (seeded numpy draws, see poetx_inputs.py)",
        "config": {"workload": args.workload, "d_in": s.d_in, "d_out": s.d_out, "b": s.b, "k": s.k,
                   "n_tokens_per_gpu": s.n_tokens, "mode": s.mode,
                   "step": "CNP fwd (R,P) + forward + backward incl. CNP adjoint",
                   "l2": "flushed between steps (256 MiB write outside the timed intervals)",
                   "launch": "CUDA graph of one step, replayed" if graph is not None else "direct launches",
                   "parallelism": (f"dp{world}: data parallel over tokens, replicas plus an NCCL all-reduce of the "
                                   f"packed theta gradients ({4 * layer.grad.numel()} bytes) every step"
                                   if world > 1 else "dp1 (one replica; the gradient all-reduce needs N > 1)"),
                   "algorithmic_gflop_per_step": round(fl["total"] / 1e9, 2)},
        "roofline": {"bound": "tensor",
                     "kernel": "w0_gemm (Z = V W0'^T with Y' = BD_R Z; dV = dZ W0' with dU = BD_P^T dV)",
                     "achieved": round(achieved, 1), "peak": peak, "unit": "TFLOP/s",
                     "frac": round(achieved / peak, 4), "traffic": W_GEMM_TRAFFIC.get(args.workload),
                     "traffic_source": "ncu dram__bytes_read.sum + dram__bytes_write.sum, mean of two forward and "
                                       "two adjoint launches of this kernel build on this workload",
                     "peak_source": f"{peaks['source']} bf16_tflops (burst)",
                     "frac_of_sustained": round(achieved / float(peaks["bf16_tflops_sustained"]), 4),
                     "launch_ms": round(w_avg_ms, 4), "launches": wcnt,
                     "forward_launch_ms": round(fms / max(fcnt, 1), 4),
                     "adjoint_launch_ms": round(ams / max(acnt, 1), 4),
                     "forward_frac": round(w_gemm_flops(s) / (fms / max(fcnt, 1) / 1e3) / 1e12 / peak, 4)},
        "step_roofline": {"t_flop_us": round(fl["total"] / (peak * 1e12) * 1e6, 1),
                          "frac": round((fl["total"] / (peak * 1e12)) / (t_ms / K / 1e3), 4)},
        "cnp": cnp,
        "kernel_share": {k: round(v[1] / total_prof_ms, 4) for k, v in prof.items() if v[0]},
        "kernel_ms_per_step": {k: round(v[1] / K, 4) for k, v in prof.items() if v[0]},
        "gpu_launches": int(launches),
        "comparator": (None if wc_ms is None else
                       {"weight_centric_ms_per_step": round(wc_ms, 4), "input_centric_ms_per_step": round(t_ms / K, 4),
                        "input_centric_speedup": round(wc_ms / (t_ms / K), 3),
                        "what": "same layer step with W = R W0 P formed first (original POET order): "
                                "T = W0' BD_P, M = BD_R T, W permuted to the original basis, Y = X W^T; "
                                "dX = dY W, dW = dY^T X, dM, gradients of Q from dM, CNP adjoint",
                        "four_permutation_ms_per_step": None if fp_ms is None else round(fp_ms, 4),
                        "two_permutation_speedup": None if fp_ms is None else round(fp_ms / (t_ms / K), 3),
                        "four_permutation_what": "same step with none of the permutations absorbed: R and P around "
                                                 "the original W0, four activation permutations per pass"}),
        "xq": xq,
        "optimizer": {"kernel": "adamw_kernel (packed theta_R + theta_P, one launch)", "params": int(n_par),
                      "us_per_launch": round(opt_ms * 1e3, 2),
                      "achieved": round(28 * n_par / (opt_ms / 1e3) / 1e9, 1), "unit": "GB/s",
                      "peak": float(peaks["hbm_gbs"]), "frac": round(28 * n_par / (opt_ms / 1e3) / 1e9 / float(peaks["hbm_gbs"]), 4),
                      "note": "median of per-launch CUDA-event times; before each launch 256 MiB written then "
                              "256 MiB of other data read, so L2 holds no operand and no dirty line; not part "
                              "of the step"},
        "e2e": {"value": round(world * s.n_tokens * Ke / (te_ms / 1e3), 1), "unit": "tokens/s",
                "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
                "ms_per_step": round(te_ms / Ke, 4),
                "protocol": "pinned X, dY in and packed theta gradients out every step; Y and dX stay "
                            "on the device (a training loop hands them to the neighbouring layers there); "
                            "copies on their own streams overlap the previous/next step; L2 flushed before "
                            "every step inside the interval"},
        "clocks": clk,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(acts)
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# -------------------------------------------------------------------------- stacked workloads
def run_stack(args):
    """A whole Llama-shaped stack as one step: one CNP launch over every block of every linear
    (the 13B stack, b = 512, runs it per transformer block: its CNP goes through the GEMM
    kernels and their scratch), then the forward of all linears in order, then the backward of
    all linears in reverse order (each with its CNP adjoint); the 13B stack's step ends with the
    merge of every linear (fresh permutations, theta reset to zero).  Weights, parameters,
    permutations and activations are seeded draws made on the device (torch's generator; the
    host-side draws of the single-layer workloads would need tens of GB of host memory), with the
    distributions of the single-layer workloads.  Inputs are far larger than L2."""
    import torch

    import orthogonal_equivalence_cnp_b200 as P
    from orthogonal_equivalence_cnp_b200.layer import make_desc
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)
    cfg, nblk, shapes_fn = I.STACKS[args.workload]
    layers = I.stack_layers(args.workload)
    sh0 = layers[0][1]
    N, b, k = sh0.n_tokens, sh0.b, sh0.k
    bf = torch.bfloat16
    gen = torch.Generator(device=dev)

    def randn(shape, std, seed, dtype=bf):
        gen.manual_seed(seed)
        return (torch.randn(shape, generator=gen, device=dev, dtype=torch.float32) * std).to(dtype)

    def randperm(n, seed):
        gen.manual_seed(seed)
        return torch.randperm(n, generator=gen, device=dev).to(torch.int32)

    descs = [make_desc(sh.d_in, sh.d_out, sh.b, sh.k, sh.dtype, sh.mode) for _, sh, _ in layers]
    nb_of = [sh.nb_out + sh.nb_in for _, sh, _ in layers]
    off = np.concatenate([[0], np.cumsum(nb_of)]).astype(int)
    nb_total = int(off[-1])
    Pk = b * (b - 1) // 2
    theta = randn((nb_total, Pk), sh0.theta_std, 17 + cfg, torch.float32)
    grad = torch.empty_like(theta)
    Q = torch.empty(nb_total, b, b, dtype=bf, device=dev)
    W = [randn((sh.d_out, sh.d_in), sh.w_std, seed) for _, sh, seed in layers]
    perms = [[randperm(sh.d_out, seed + 1), randperm(sh.d_in, seed + 2)] for _, sh, seed in layers]
    new_perms = [[randperm(sh.d_out, seed + 10001), randperm(sh.d_in, seed + 10002)] for _, sh, seed in layers]
    dims_in = sorted({sh.d_in for _, sh, _ in layers})
    dims_out = sorted({sh.d_out for _, sh, _ in layers})
    X = {d: randn((N, d), 1.0, 7 + d) for d in dims_in}
    dX = {d: torch.empty(N, d, dtype=bf, device=dev) for d in dims_in}
    dY = {d: randn((N, d), 1.0, 11 + d) for d in dims_out}
    Y = {d: torch.empty(N, d, dtype=bf, device=dev) for d in dims_out}
    fast = sh0.mode == "fast"
    saved = [torch.empty(N * (sh.d_in + sh.d_out), dtype=bf, device=dev) if fast else None for _, sh, _ in layers]
    ws_bytes = max(P.poetx_workspace_size(d, N) for d in descs)
    per_block = len(layers) // nblk
    cnp_chunks = [(0, nb_total)] if b <= 256 else [(int(off[i]), int(off[i + per_block]) - int(off[i]))
                                                   for i in range(0, len(layers), per_block)]
    ws_bytes = max(ws_bytes, max(P.poetx_cnp_blocks_workspace_size(descs[0], n) for _, n in cnp_chunks))
    ws = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)
    merge = cfg == 5
    stream = torch.cuda.current_stream()
    buckets = None
    if world > 1:  # the packed gradients of each run of layers are summed while the layers below run
        from orthogonal_equivalence_cnp_b200.ddp import GradBuckets
        buckets = GradBuckets(grad.view(-1), [n * Pk for n in nb_of])

    def sl(t, i):  # slice of the flat block arrays for linear i: R side, then P side
        _, sh, _ = layers[i]
        a, m = int(off[i]), sh.nb_out
        return t[a:a + m], t[a + m:a + m + sh.nb_in]

    def cnp():
        for a, n in cnp_chunks:
            P.poetx_cnp_blocks(descs[0], n, theta[a:a + n], Q[a:a + n], ws)

    def fwd_bwd():
        for i, (_, sh, _) in enumerate(layers):
            QR, QP = sl(Q, i)
            P.poetx_forward(descs[i], N, X[sh.d_in], W[i], perms[i][0], perms[i][1], QR, QP, Y[sh.d_out], saved[i], ws)
        for i in reversed(range(len(layers))):
            _, sh, _ = layers[i]
            QR, QP = sl(Q, i)
            tR, tP = sl(theta, i)
            gR, gP = sl(grad, i)
            P.poetx_backward(descs[i], N, dY[sh.d_out], X[sh.d_in], W[i], perms[i][0], perms[i][1], QR, QP, tR, tP,
                             saved[i], dX[sh.d_in], gR, gP, ws)
            if buckets is not None:
                buckets.layer_done(i)
        if buckets is not None:
            buckets.finish()

    def do_merge():
        for i in range(len(layers)):
            QR, QP = sl(Q, i)
            tR, tP = sl(theta, i)
            P.poetx_merge(descs[i], W[i], QR, QP, perms[i][0], perms[i][1], new_perms[i][0], new_perms[i][1], tR, tP,
                          ws)
            perms[i], new_perms[i] = new_perms[i], perms[i]

    def step():
        cnp()
        fwd_bwd()
        if merge:
            do_merge()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st, det = P.poetx_device_status()
    if st != 0:
        raise RuntimeError(f"device-side timeout during warm-up ({det:#x})")
    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K)]
    clocks = ClockSampler()
    clocks.start()
    time.sleep(0.3)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    n0 = P.poetx_launch_count()
    for i in range(K):
        ev[i][0].record(stream)
        cnp()
        ev[i][1].record(stream)
        fwd_bwd()
        ev[i][2].record(stream)
        if merge:
            do_merge()
        ev[i][3].record(stream)
    torch.cuda.synchronize()
    launches = P.poetx_launch_count() - n0
    clk = clocks.stop(gpu_uuid(dev))
    st, det = P.poetx_device_status()
    if st != 0:
        raise RuntimeError(f"device-side timeout in the timed region ({det:#x})")
    t_step = max_over_ranks(sum(ev[i][0].elapsed_time(ev[i][3]) for i in range(K)), world, dev) / K
    t_cnp = sum(ev[i][0].elapsed_time(ev[i][1]) for i in range(K)) / K
    t_fb = sum(ev[i][1].elapsed_time(ev[i][2]) for i in range(K)) / K
    t_merge = sum(ev[i][2].elapsed_time(ev[i][3]) for i in range(K)) / K
    fl = sum(step_flops(sh)["total"] for _, sh, _ in layers)
    f_merge = sum(4 * sh.b * sh.d_in * sh.d_out for _, sh, _ in layers) if merge else 0
    peaks = read_peaks()
    peak, hbm = float(peaks["bf16_tflops_sustained"]), float(peaks["hbm_gbs"])
    cnp_bytes = nb_total * (4 * Pk + 2 * b * b)
    out = {
        "metric": METRIC,
        "value": round(world * N / (t_step / 1e3), 1),
        "unit": "tokens/s",
        "tflops": round(world * (fl + f_merge) / (t_step / 1e3) / 1e12, 2),
        "n_gpus": world, "steps": K, "warmup": args.warmup, "ms_per_step": round(t_step, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded draws on the device, torch generator)",
        "config": {"workload": args.workload, "linears": len(layers), "blocks": nb_total, "b": b, "k": k,
                   "n_tokens_per_gpu": N, "mode": sh0.mode,
                   "step": "one CNP launch over all blocks + forward of every linear + backward of every linear"
                           + (" + merge of every linear" if merge else ""),
                   "l2": "inputs larger than L2", "launch": "direct launches",
                   "parallelism": (f"dp{world}: replicas on their own tokens; packed gradients summed over the "
                                   f"ranks in buckets of consecutive layers during the backward pass"
                                   if world > 1 else "dp1"),
                   "algorithmic_gflop_per_step": round(fl / 1e9, 1),
                   "merge_gflop_per_step": round(f_merge / 1e9, 1)},
        "step_roofline": {"t_flop_ms": round(fl / (peak * 1e12) * 1e3, 2),
                          "frac": round(fl / (peak * 1e12) / ((t_step - t_merge) / 1e3), 4),
                          "peak": peak, "peak_source": f"{peaks['source']} bf16_tflops_sustained",
                          "note": "fwd + bwd + CNP FLOPs over the step time less the merge"},
        "cnp": {"launches_per_step": len(cnp_chunks), "ms": round(t_cnp, 3), "blocks": nb_total,
                "bytes": cnp_bytes, "hbm_frac": round(cnp_bytes / (t_cnp / 1e3) / 1e9 / hbm, 4)},
        "fwd_bwd_ms": round(t_fb, 3),
        "merge_ms": round(t_merge, 3) if merge else None,
        "gpu_launches": int(launches),
        "clocks": clk,
    }
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ------------------------------------------------------------------------- reference arm
def run_reference(args):
    """The float64 oracle on the host cores.  Each step is a bounded sample of the workload, scaled
    to it: for every linear of the sample, the activation part of the step (forward chain and the
    backward chain up to G = dL/dQ) on the first n tokens, and the CNP forward and adjoint of one
    block per side; the step time of the whole workload is estimated as the sum over the sample's
    linears of t_act * N / n + t_cnp * (blocks of both sides) / 2, which the reported tokens/s
    divides N by.  A single-layer workload is its own sample; a stacked workload's sample is its
    first transformer block (7 linears), scaled by the number of blocks (extrapolated).  n is
    chosen so that all steps take about two minutes."""
    import oracle as O
    rank, world, _ = dist_env()
    if rank != 0:
        return
    if args.workload in I.STACKS:
        _, nblk, _ = I.STACKS[args.workload]
        chosen = I.stack_layers(args.workload)
        chosen = [(sh, seed) for _, sh, seed in chosen[:len(chosen) // nblk]]
        scale = nblk
    else:
        chosen, scale = [(I.WORKLOADS[args.workload], I.WORKLOAD_SEEDS[args.workload])], 1
    n_full = chosen[0][0].n_tokens
    n_cap = 256 if args.workload in I.STACKS else n_full  # host draws of the stacks' token rows stay small
    prepared = []
    for sh, seed in chosen:
        inp = I.make_layer(sh, seed, n_tokens=min(n_full, n_cap))
        W0p = O.absorb(inp.W0, inp.pi_L, inp.pi_R)  # layer state, outside the timing
        Q_R, Q_P = O.cnp(inp.theta_R[:1], sh.b, sh.k), O.cnp(inp.theta_P[:1], sh.b, sh.k)
        Q_R = np.repeat(Q_R, sh.nb_out, axis=0)  # every block's Q has the same cost; one is computed
        Q_P = np.repeat(Q_P, sh.nb_in, axis=0)
        _, G_R, _ = O.backward_chain_G(inp.X[:8], inp.dY[:8], W0p, Q_R, Q_P, inp.pi_L, inp.pi_R, sh.b)
        prepared.append((sh, inp, W0p, Q_R, Q_P, G_R))

    def sample_step(n_tok):
        """Returns (raw activation seconds, raw CNP seconds, the step estimate for the workload)."""
        ra = rc = est = 0.0
        for sh, inp, W0p, Q_R, Q_P, G_R in prepared:
            X, dY = inp.X[:n_tok], inp.dY[:n_tok]
            t0 = time.perf_counter()
            O.forward_chain(X, W0p, Q_R, Q_P, inp.pi_L, inp.pi_R)
            O.backward_chain_G(X, dY, W0p, Q_R, Q_P, inp.pi_L, inp.pi_R, sh.b)
            t1 = time.perf_counter()
            for th in (inp.theta_R[:1], inp.theta_P[:1]):  # one block per side: CNP forward + adjoint
                O.cnp(th, sh.b, sh.k)
                O.cnp_grad(th, G_R[:1], sh.b, sh.k)
            t2 = time.perf_counter()
            ra += t1 - t0
            rc += t2 - t1
            est += (t1 - t0) * n_full / n_tok + (t2 - t1) * (sh.nb_in + sh.nb_out) / 2
        return ra, rc, est * scale

    ra, rc, _ = sample_step(8)
    budget = 120.0 / max(1, args.steps + args.warmup)
    n_tok = 8
    n_max = min(n_full, n_cap)
    while n_tok * 2 <= n_max and ra * (n_tok * 2) / 8 + rc <= budget:
        n_tok *= 2
    for _ in range(args.warmup):
        sample_step(n_tok)
    t_step = 0.0
    for _ in range(args.steps):
        t_step += sample_step(n_tok)[2]
    t_step /= args.steps  # whole-workload step, estimated
    value = n_full / t_step
    fl = sum(step_flops(sh)["total"] for sh, *_ in prepared) * scale
    what = (f"{len(prepared)} linears of the first of {scale} transformer blocks, extrapolated x{scale}"
            if scale > 1 else "the layer")
    sample = (f"per step: {what}: forward + backward activation chain on the first {n_tok} of {n_full} tokens and "
              f"the CNP forward + adjoint of 1 block per side, float64 numpy; scaled to the full step as "
              f"t_act*{n_full}/{n_tok} + t_cnp*(blocks of both sides)/2 per linear")
    s0 = prepared[0][0]
    out = {
        "impl": "reference",
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(1e3 * t_step, 2),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic (seeded numpy draws, see poetx_inputs.py)",
        "config": {"workload": args.workload, "d_in": s0.d_in, "d_out": s0.d_out, "b": s0.b, "k": s0.k,
                   "n_tokens_per_gpu": n_full, "mode": s0.mode,
                   "algorithmic_gflop_per_step": round(fl / 1e9, 2)},
        "cpu_baseline": {"value": round(value, 2), "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 2), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", choices=["poetx", "reference"], default="poetx")
    ap.add_argument("--workload", choices=sorted(I.WORKLOADS) + sorted(I.STACKS), default=DEFAULT_WORKLOAD)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-xq", dest="xq", action="store_false",
                    help="skip timing the POET-XQ (int8 W0') mem-mode step beside the bf16 mem-mode step")
    ap.add_argument("--no-comparator", dest="comparator", action="store_false",
                    help="skip timing the weight-centric comparator")
    ap.add_argument("--no-graph", action="store_true", help="launch every step directly instead of replaying a CUDA graph")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    elif args.workload in I.STACKS:
        run_stack(args)
    else:
        run_poetx(args)


if __name__ == "__main__":
    main()
