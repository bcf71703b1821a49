"""Seeded synthetic inputs for the sign-weight linear layers.

This module only draws random numbers and rounds draws to the storage types the
workloads name (bf16 activations, fp32 weights and scales, +/-1 sign matrices).
It holds none of the method's arithmetic: no sign extraction, packing, SVID or
linear algebra.  Both the CUDA path and the fp64 oracle are fed from here, so
every comparison runs on identical inputs.

Workload shapes follow the 7B-class linear layers (hidden 4096, MLP 11008) that
stand in for the Llama2-7B / Llama3-8B weights evaluated in "Addition is almost
all you need: Compressing large language models with double binary
factorization" (Resultaten); those weights are not available, so every tensor
here is synthetic.  The outlier-channel recipe (6 channels, magnitude ~60)
follows the emergent-feature statistics on the LLM.int8() page
(hub.baai.ac.cn/view/22301, outlier-feature section).
"""
from __future__ import annotations

import numpy as np

# Stream ids: each array of a workload gets its own child stream of the seed,
# so drawing one array never shifts another.
_STREAM = {"x": 1, "w": 2, "sa": 3, "sb": 4, "a": 5, "m": 6, "b": 7, "perm": 8}


def rng(seed: int, stream: str) -> np.random.Generator:
    """PCG64 generator for (seed, named stream)."""
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(seed), _STREAM[stream]])))


def bf16_round(x: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Round fp32 values to bf16, round-to-nearest-even.

    Returns (bits, values): ``bits`` is the uint16 bf16 encoding, ``values`` the
    same numbers as float32 (exactly representable).  Inputs must be finite.
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    bias = 0x7FFF + ((u >> 16) & 1)
    bits = ((u + bias) >> 16).astype(np.uint16)
    values = (bits.astype(np.uint32) << 16).view(np.float32)
    return bits, values


def outlier_channels(K: int, seed: int = 5, count: int = 6) -> np.ndarray:
    """The fixed outlier feature dimensions: first ``count`` of a seeded permutation of K."""
    return rng(seed, "perm").permutation(K)[:count].astype(np.int64)


def activations(seed: int, M: int, K: int, outliers: bool = False,
                outlier_scale: float = 60.0) -> tuple[np.ndarray, np.ndarray]:
    """X ~ N(0,1) (M x K), optionally with the outlier channels scaled, rounded to bf16.

    Returns (bits uint16 [M,K], values float32 [M,K]).
    """
    x = rng(seed, "x").standard_normal((M, K), dtype=np.float32)
    if outliers and K > 0:
        x[:, outlier_channels(K)] *= np.float32(outlier_scale)
    return bf16_round(x)


def weights(seed: int, N: int, K: int, std: float = 0.02) -> np.ndarray:
    """W ~ N(0, std^2), fp32, N x K (out x in); ``std`` is the standard deviation."""
    return (rng(seed, "w").standard_normal((N, K), dtype=np.float32) * np.float32(std)).astype(np.float32)


def pm1(seed: int, rows: int, cols: int, stream: str) -> np.ndarray:
    """Random +/-1 matrix (Bernoulli 1/2), int8."""
    bits = rng(seed, stream).integers(0, 2, size=(rows, cols), dtype=np.int8)
    return (1 - 2 * bits).astype(np.int8)


def scales(seed: int, n: int, stream: str) -> np.ndarray:
    """Positive scale vector |N(0,1)| * 0.02 + 1e-3, fp32."""
    v = np.abs(rng(seed, stream).standard_normal(n, dtype=np.float32)) * np.float32(0.02)
    return (v + np.float32(1e-3)).astype(np.float32)


def dbf_factors(seed: int, N: int, r: int, K: int) -> dict:
    """Random DBF operands: S_A (N x r), S_B (r x K) as +/-1 int8; a(N), m(r), b(K) fp32."""
    return {
        "S_A": pm1(seed, N, r, "sa"),
        "S_B": pm1(seed, r, K, "sb"),
        "a": scales(seed, N, "a"),
        "m": scales(seed, r, "m"),
        "b": scales(seed, K, "b"),
    }


# The five workload configurations (sizes as named; seeds fixed per workload).
CONFIGS = {
    "onebit_tiny": dict(seed=0, M=[4], N=256, K=256),
    "onebit_decode": dict(seed=1, M=[1, 4, 16], N=4096, K=4096),
    "onebit_prefill": dict(seed=2, M=[2048], N=11008, K=4096),
    "dbf": dict(seed=3, M=[1, 512], N=4096, K=4096, r=2048),
    "sweep_outliers": dict(seed=4, M=[1, 16, 256, 4096],
                           shapes=[(4096, 4096), (4096, 11008), (11008, 4096)]),  # (K, N): K -> N
}
