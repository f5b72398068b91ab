"""Seeded synthetic inputs for the POET-X layer (shared by the oracle side and the CUDA side).

This module draws random numbers and rounds them to the storage type; it holds none of the
method's arithmetic.  Both the float64 oracle (``oracle/``) and the CUDA library's tests and
benchmark consume exactly the arrays returned here, so a parity comparison always starts from
bit-identical inputs.

Workloads are Llama-shaped synthetic POET-X linear layers.  The shapes, block sizes, Neumann
order and value distributions follow the workloads the POET-X pages measure: the single-layer
fwd+bwd benchmark at hidden size 4096, sequence 2048 and block size 256 (SAI replication
review of POET-X, "Reproducibility & code", first item; paper Fig. 3), the Llama-8B/13B
stacks of the memory tables (agidaily.cc article, Table 9 paragraph), and b in {256, 512}
(replication review, "Summary" and "Weaknesses").  No dataset is involved: the pages'
C4/t5-base pretraining data is for end-to-end training, which is outside this library.

Draw order for one layer with ``numpy.random.default_rng(seed)`` (PCG64):
    pi_L = permutation(d_out); pi_R = permutation(d_in);
    theta_R ~ N(0, theta_std^2) [nb_out, b(b-1)/2]; theta_P likewise [nb_in, b(b-1)/2];
    W0 ~ N(0, w_std^2) [d_out, d_in]; X ~ N(0, 1) [N, d_in]; dY ~ N(0, 1) [N, d_out].
All draws are float64, cast to float32; for bf16 workloads W0, X and dY are then rounded to
the nearest bfloat16 (round-to-nearest-even) and kept as float32 arrays holding exactly
representable values.  The packed skew parameters always stay float32.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional

import numpy as np


@dataclasses.dataclass(frozen=True)
class LayerShape:
    d_in: int
    d_out: int
    b: int
    k: int
    n_tokens: int
    dtype: str          # "f32" or "bf16": storage type of W0', activations and Q
    mode: str           # "fast" or "mem"
    theta_std: float
    w_std: float

    @property
    def nb_in(self) -> int:
        return self.d_in // self.b

    @property
    def nb_out(self) -> int:
        return self.d_out // self.b

    @property
    def n_packed(self) -> int:
        return self.b * (self.b - 1) // 2


def _shape(d_in, d_out, b, n, dtype, mode, theta_std, w_std, k=3):
    return LayerShape(d_in=d_in, d_out=d_out, b=b, k=k, n_tokens=n, dtype=dtype, mode=mode,
                      theta_std=theta_std, w_std=w_std)


# Single-layer workloads.  Seeds are 1000 + workload number.
WORKLOADS: Dict[str, LayerShape] = {
    # fp32 correctness layer: 256x256, b=32 (8 blocks per side), k=3, 64 tokens.
    "layer256_b32_f32": _shape(256, 256, 32, 64, "f32", "fast", 0.01, 1.0 / 16.0),
    # Llama-8B attention projection: 4096x4096, b=256, 2048 tokens, bf16, fast mode.
    "llama8b_attn_4096_b256_bf16": _shape(4096, 4096, 256, 2048, "bf16", "fast", 0.005, 0.02),
    # Llama-8B MLP up-projection: 4096->14336, 8192 tokens, bf16, mem mode, b=256 or 512.
    "llama8b_up_4096x14336_b256_bf16_mem": _shape(4096, 14336, 256, 8192, "bf16", "mem", 0.005, 0.02),
    "llama8b_up_4096x14336_b512_bf16_mem": _shape(4096, 14336, 512, 8192, "bf16", "mem", 0.005, 0.02),
}

WORKLOAD_SEEDS: Dict[str, int] = {
    "layer256_b32_f32": 1001,
    "llama8b_attn_4096_b256_bf16": 1002,
    "llama8b_up_4096x14336_b256_bf16_mem": 1003,
    "llama8b_up_4096x14336_b512_bf16_mem": 1003,
}


def llama8b_stack_shapes(n_tokens: int = 2048) -> List[LayerShape]:
    """The 7 linears of one Llama-8B-shaped block (GQA 32q/8kv heads of 128): q,k,v,o,gate,up,down."""
    h, kv, ff = 4096, 1024, 14336
    dims = [(h, h), (h, kv), (h, kv), (h, h), (h, ff), (h, ff), (ff, h)]
    return [_shape(di, do, 256, n_tokens, "bf16", "fast", 0.005, 0.02) for (di, do) in dims]


def llama13b_stack_shapes(n_tokens: int = 4096) -> List[LayerShape]:
    """The 7 linears of one Llama-13B-shaped block: q,k,v,o 5120^2, gate/up 5120->13824, down back."""
    h, ff = 5120, 13824
    dims = [(h, h), (h, h), (h, h), (h, h), (h, ff), (h, ff), (ff, h)]
    return [_shape(di, do, 512, n_tokens, "bf16", "mem", 0.005, 0.02) for (di, do) in dims]


def round_to_bf16(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even); returns float32 values."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    bias = np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))
    r = ((u + bias) >> np.uint64(16)) << np.uint64(16)
    return r.astype(np.uint32).view(np.float32).reshape(a.shape)


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """Upper 16 bits of float32 values that are exactly representable in bfloat16."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32)
    if np.any(u & np.uint32(0xFFFF)):
        raise ValueError("values are not bfloat16-representable")
    return (u >> np.uint32(16)).astype(np.uint16)


@dataclasses.dataclass
class LayerInputs:
    shape: LayerShape
    seed: int
    pi_L: np.ndarray      # int32 [d_out]
    pi_R: np.ndarray      # int32 [d_in]
    theta_R: np.ndarray   # float32 [nb_out, b(b-1)/2]
    theta_P: np.ndarray   # float32 [nb_in,  b(b-1)/2]
    W0: np.ndarray        # float32 [d_out, d_in] (bf16-representable for bf16 layers)
    X: Optional[np.ndarray]   # float32 [N, d_in]
    dY: Optional[np.ndarray]  # float32 [N, d_out]


def _store(a: np.ndarray, dtype: str) -> np.ndarray:
    a = a.astype(np.float32)
    return round_to_bf16(a) if dtype == "bf16" else a


def make_layer(shape: LayerShape, seed: int, n_tokens: Optional[int] = None,
               with_activations: bool = True) -> LayerInputs:
    """Draw one layer's inputs in the documented order.

    ``n_tokens`` overrides the workload's token count (the first rows of the full draw are NOT
    a prefix of a smaller draw; each token count is its own seeded workload).
    """
    n = shape.n_tokens if n_tokens is None else int(n_tokens)
    rng = np.random.default_rng(seed)
    pi_L = rng.permutation(shape.d_out).astype(np.int32)
    pi_R = rng.permutation(shape.d_in).astype(np.int32)
    theta_R = rng.normal(0.0, shape.theta_std, (shape.nb_out, shape.n_packed)).astype(np.float32)
    theta_P = rng.normal(0.0, shape.theta_std, (shape.nb_in, shape.n_packed)).astype(np.float32)
    W0 = _store(rng.normal(0.0, shape.w_std, (shape.d_out, shape.d_in)), shape.dtype)
    X = dY = None
    if with_activations:
        X = _store(rng.normal(0.0, 1.0, (n, shape.d_in)), shape.dtype)
        dY = _store(rng.normal(0.0, 1.0, (n, shape.d_out)), shape.dtype)
    return LayerInputs(shape, seed, pi_L, pi_R, theta_R, theta_P, W0, X, dY)


def make_theta(shape: LayerShape, seed: int):
    """theta_R, theta_P of make_layer(shape, seed) (the same draws), without W0 or activations."""
    rng = np.random.default_rng(seed)
    rng.permutation(shape.d_out)
    rng.permutation(shape.d_in)
    theta_R = rng.normal(0.0, shape.theta_std, (shape.nb_out, shape.n_packed)).astype(np.float32)
    theta_P = rng.normal(0.0, shape.theta_std, (shape.nb_in, shape.n_packed)).astype(np.float32)
    return theta_R, theta_P


# Stacked workloads: layer l of stack config c (4: the 32-block Llama-8B stack, 5: the 40-block
# Llama-13B stack) is drawn with seed 1000 + 100 c + l; the layers of a block are q,k,v,o,gate,
# up,down in that order.
STACKS = {
    "llama8b_stack_32x7_b256_bf16": (4, 32, llama8b_stack_shapes),
    "llama13b_stack_40x7_b512_bf16_mem": (5, 40, llama13b_stack_shapes),
}


def stack_layers(name: str):
    """[(layer index, LayerShape, seed)] of every linear of a stacked workload."""
    config, nblocks, shapes = STACKS[name]
    per_block = shapes()
    out = []
    for blk in range(nblocks):
        for j, sh in enumerate(per_block):
            l = blk * len(per_block) + j
            out.append((l, sh, 1000 + 100 * config + l))
    return out


def make_workload(name: str, n_tokens: Optional[int] = None, with_activations: bool = True) -> LayerInputs:
    return make_layer(WORKLOADS[name], WORKLOAD_SEEDS[name], n_tokens, with_activations)


def fresh_permutations(shape: LayerShape, seed: int):
    """The new permutations a merge re-absorbs: drawn from default_rng(seed + 10000)."""
    rng = np.random.default_rng(seed + 10000)
    return (rng.permutation(shape.d_out).astype(np.int32),
            rng.permutation(shape.d_in).astype(np.int32))


def small_shape(d_in: int, d_out: int, b: int, k: int, n_tokens: int, dtype: str = "f32",
                mode: str = "fast", theta_std: float = 0.05, w_std: float = 0.1) -> LayerShape:
    """A small layer for unit tests (sizes chosen by the test)."""
    return _shape(d_in, d_out, b, n_tokens, dtype, mode, theta_std, w_std, k=k)
