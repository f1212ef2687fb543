"""Seeded synthetic inputs for the q4gsw linear layer.

This module draws random tensors and names shapes; it holds none of the
layer's arithmetic (no packing, no dequantisation, no products).  Tests, the
smoke check and the benchmark use it to feed the same inputs to the CUDA
library and to the CPU oracle.

Draw order for one shape (numpy ``default_rng(seed)``, PCG64):
  1. x      = standard_normal((M, K), float32) -> float16
  2. codes  = integers(0, 16, (N, K), uint8)
  3. scales = per-workload distribution, shape [K/group_size, N] -> float16
  4. d_out  = standard_normal((M, N), float32) * sigma -> float16

The workloads are the layer shapes of a 1B-class decoder (hidden 2048,
32 query heads and 8 key/value heads of width 64, MLP 8192) and an 8B-class
layer (hidden 4096, MLP 14336).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np


@dataclass(frozen=True)
class Shape:
    name: str
    M: int
    N: int
    K: int
    group_size: int
    seed: int
    scales: str = "uniform"         # "uniform" -> U[0.005, 0.02]; "loguniform" -> logU[1e-3, 5e-2]
    dout_sigma: float = 1.0
    directions: tuple = ("fwd",)    # subset of ("fwd", "bwd")
    splits: tuple = ()              # (Nq, Nk, Nv) for the fused Q/K/V projection


@dataclass
class Inputs:
    x: np.ndarray          # float16 [M, K]
    codes: np.ndarray      # uint8  [N, K], 0..15
    scales: np.ndarray     # float16 [G, N]
    d_out: np.ndarray      # float16 [M, N]
    shape: Shape = field(repr=False, default=None)


def tiny():
    return [Shape("tiny", 4, 64, 128, 32, seed=0, directions=("fwd", "bwd"))]


def decode():
    shapes = [(2048, 2048), (8192, 2048), (2048, 8192)]
    return [Shape(f"decode_N{N}_K{K}", 1, N, K, 32, seed=200 + i)
            for i, (N, K) in enumerate(shapes)]


def qkv():
    Nq, Nk, Nv = 2048, 512, 512
    return [Shape(f"qkv_M{M}", M, Nq + Nk + Nv, 2048, 32, seed=300 + i, splits=(Nq, Nk, Nv))
            for i, M in enumerate((128, 508, 512))]


def adapter():
    return [
        Shape("adapter_up_M512", 512, 8192, 2048, 32, seed=400, dout_sigma=1e-2, directions=("fwd", "bwd")),
        Shape("adapter_down_M512", 512, 2048, 8192, 32, seed=401, dout_sigma=1e-2, directions=("fwd", "bwd")),
    ]


SWEEP_M = (1, 4, 16, 64, 256, 1024, 4096)


def sweep():
    out = []
    for si, (N, K) in enumerate(((14336, 4096), (4096, 14336))):
        for mi, M in enumerate(SWEEP_M):
            out.append(Shape(f"sweep_M{M}_N{N}_K{K}", M, N, K, 128, seed=500 + si * len(SWEEP_M) + mi,
                             scales="loguniform", directions=("fwd", "bwd")))
    return out


def embedding():
    """Embedding gathers from a 1B-class table (vocabulary 32000 x 2048 features,
    gs 32): one decode token, a 512-token prompt and a 16384-token batch.  The
    token ids come from ``embedding_indices``."""
    return [Shape(f"embedding_T{T}_V32000_D2048", T, 32000, 2048, 32, seed=600 + i, directions=("emb",))
            for i, T in enumerate((1, 512, 16384))]


def embedding_indices(shape: Shape, T: int | None = None) -> np.ndarray:
    """Seeded token ids, int32 [T], uniform over the table's N rows (repeats allowed)."""
    T = shape.M if T is None else T
    return np.random.default_rng(shape.seed + 10_000).integers(0, shape.N, T, dtype=np.int32)


def all_shapes():
    return tiny() + decode() + qkv() + adapter() + sweep() + embedding()


def by_name(name: str) -> Shape:
    for s in all_shapes():
        if s.name == name:
            return s
    raise KeyError(name)


def make_inputs(shape: Shape, M: int | None = None) -> Inputs:
    """Draw the inputs of one shape.  ``M`` overrides the token count (same seed)."""
    M = shape.M if M is None else M
    rng = np.random.default_rng(shape.seed)
    x = rng.standard_normal((M, shape.K), dtype=np.float32).astype(np.float16)
    codes = rng.integers(0, 16, (shape.N, shape.K), dtype=np.uint8)
    G = shape.K // shape.group_size
    if shape.scales == "uniform":
        s = rng.uniform(0.005, 0.02, (G, shape.N))
    elif shape.scales == "loguniform":
        s = np.exp(rng.uniform(np.log(1e-3), np.log(5e-2), (G, shape.N)))
    else:
        raise ValueError(shape.scales)
    scales = s.astype(np.float16)
    d_out = (rng.standard_normal((M, shape.N), dtype=np.float32) * np.float32(shape.dout_sigma)).astype(np.float16)
    return Inputs(x=x, codes=codes, scales=scales, d_out=d_out, shape=shape)


def random_inputs(M: int, N: int, K: int, group_size: int, seed: int,
                  scales: str = "uniform", dout_sigma: float = 1.0) -> Inputs:
    """Inputs for an ad-hoc shape (edge cases, ragged sizes)."""
    return make_inputs(Shape(f"adhoc_M{M}_N{N}_K{K}_g{group_size}", M, N, K, group_size, seed,
                             scales=scales, dout_sigma=dout_sigma, directions=("fwd", "bwd")))


def integer_exact_inputs(M: int, N: int, K: int, group_size: int, seed: int) -> Inputs:
    """Inputs whose products and partial sums are all exact in fp32 and fp16.

    x and d_out take values in {-2, ..., 2}; every scale is a power of two in
    [2^-6, 2^-3], so each weight is an integer times 2^-6 with magnitude at most 1
    and every partial sum is a multiple of 2^-6 far below 2^18.
    """
    rng = np.random.default_rng(seed)
    x = rng.integers(-2, 3, (M, K)).astype(np.float16)
    codes = rng.integers(0, 16, (N, K), dtype=np.uint8)
    G = K // group_size
    scales = np.ldexp(1.0, rng.integers(-6, -2, (G, N))).astype(np.float16)
    d_out = rng.integers(-2, 3, (M, N)).astype(np.float16)
    return Inputs(x=x, codes=codes, scales=scales, d_out=d_out,
                  shape=Shape(f"intexact_M{M}_N{N}_K{K}", M, N, K, group_size, seed))
