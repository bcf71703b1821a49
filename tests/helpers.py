"""Shared test helpers: tolerance checks, cached oracle SVID, tensor conversion."""
from __future__ import annotations

import functools

import numpy as np

import oracle
from binary_weight_gemm_b200 import synth
from conftest import MAX_ABS_REL_TOL, REL_FRO_TOL


def gemm_errors(y_gpu, y_ref: np.ndarray) -> tuple[float, float]:
    """(relative Frobenius error, max |dY| / max |Y_ref|) of a GPU result against the fp64 oracle."""
    y = y_gpu.float().cpu().numpy().astype(np.float64) if hasattr(y_gpu, "cpu") else np.asarray(y_gpu, np.float64)
    ref = np.asarray(y_ref, dtype=np.float64)
    assert y.shape == ref.shape, (y.shape, ref.shape)
    nref = np.linalg.norm(ref)
    mref = np.abs(ref).max() if ref.size else 0.0
    if nref == 0.0:
        return float(np.linalg.norm(y)), float(np.abs(y).max() if y.size else 0.0)
    return float(np.linalg.norm(y - ref) / nref), float(np.abs(y - ref).max() / mref)


def assert_gemm_close(y_gpu, y_ref, rel_fro=REL_FRO_TOL, max_rel=MAX_ABS_REL_TOL, what=""):
    fro, mx = gemm_errors(y_gpu, y_ref)
    assert fro <= rel_fro, f"{what}: relative Frobenius error {fro:.3e} > {rel_fro}"
    assert mx <= max_rel, f"{what}: max |dY| / max |Y_ref| = {mx:.3e} > {max_rel}"
    return fro, mx


@functools.lru_cache(maxsize=8)
def oracle_svid(seed: int, N: int, K: int):
    """Oracle SVID (full SVD, fp64) of the seeded weight W(seed, N, K), cast to fp32 for both sides."""
    W = synth.weights(seed, N, K)
    a, b, s = oracle.svid_rank1(W)
    return W, a.astype(np.float32), b.astype(np.float32), s


def cosine(x: np.ndarray, y: np.ndarray) -> float:
    x = np.asarray(x, np.float64).ravel()
    y = np.asarray(y, np.float64).ravel()
    return float(x @ y / (np.linalg.norm(x) * np.linalg.norm(y)))


def header_functions(path: str) -> list[str]:
    """Names of the functions include/obgemm.h declares (lines starting with OB_API)."""
    import re
    names = []
    with open(path) as f:
        for line in f:
            m = re.match(r"^OB_API\s+[\w\s\*]+?\b(\w+)\s*\(", line)
            if m:
                names.append(m.group(1))
    return names
