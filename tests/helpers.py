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


CANARY_BYTE = 0xA5
CANARY_PAD = 4096  # bytes before and after; keeps the interior 256-byte aligned


class Guarded:
    """A CUDA tensor inside a larger allocation whose CANARY_PAD bytes on each side hold
    CANARY_BYTE, so that a kernel writing past either end of its output is caught
    (compute-sanitizer is not available; this is the stand-in for output buffers)."""

    def __init__(self, shape, dtype, device="cuda"):
        import torch
        nbytes = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        self._buf = torch.full((CANARY_PAD + nbytes + CANARY_PAD,), CANARY_BYTE, dtype=torch.uint8, device=device)
        self._n = nbytes
        self.t = self._buf[CANARY_PAD:CANARY_PAD + nbytes].view(dtype).view(shape)

    def check(self, what=""):
        head = self._buf[:CANARY_PAD]
        tail = self._buf[CANARY_PAD + self._n:]
        bad_h = int((head != CANARY_BYTE).sum())
        bad_t = int((tail != CANARY_BYTE).sum())
        assert bad_h == 0 and bad_t == 0, f"{what}: {bad_h} bytes before and {bad_t} bytes after the buffer overwritten"
