"""DBF oracle: the double-binary factorised weight and its linear layer, fp64.

Test infrastructure only (see the package docstring).  Source page: "Addition
is almost all you need: Compressing large language models with double binary
factorization" (gist.science), section "Methodologie: Double Binary
Factorization (DBF)".

Reading of the page's garbled broadcast notation (a ⊙ A ⊙ m^T)(B ⊙ b^T): with
S_A (N x r) and S_B (r x K) the two +/-1 matrices, the weight is

    W_hat = diag(a) · S_A · diag(m) · S_B · diag(b),

which is the only reading consistent with the page's inference chain
((((X ⊙ b^T) S_B^T) ⊙ m^T) S_A^T) ⊙ a^T.  The page stores a, m, b in FP16; the
workloads here use fp32 vectors, and the oracle computes in fp64.
"""
from __future__ import annotations

import numpy as np


def dbf_weight(S_A, S_B, a, m, b) -> np.ndarray:
    """W_hat = diag(a) S_A diag(m) S_B diag(b), explicit N x K float64 matrix."""
    S_A = np.asarray(S_A, dtype=np.float64)
    S_B = np.asarray(S_B, dtype=np.float64)
    a = np.asarray(a, dtype=np.float64)
    m = np.asarray(m, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    left = a[:, None] * S_A * m[None, :]          # diag(a) S_A diag(m), N x r
    right = S_B * b[None, :]                       # S_B diag(b), r x K
    return left @ right


def dbf_linear(X, S_A, S_B, a, m, b) -> np.ndarray:
    """Y = X · W_hat^T in the direct form (W_hat materialised), float64, M x N."""
    return np.asarray(X, dtype=np.float64) @ dbf_weight(S_A, S_B, a, m, b).T


def dbf_linear_chain(X, S_A, S_B, a, m, b) -> np.ndarray:
    """The page's inference order ((((X ⊙ b^T) S_B^T) ⊙ m^T) S_A^T) ⊙ a^T, float64.

    Equal to the direct form in exact arithmetic (pinned by the tests against
    dbf_linear); the GPU parity tests use it where r and K are large enough that
    materialising W_hat would cost seconds per case.
    """
    X = np.asarray(X, dtype=np.float64)
    T = (X * np.asarray(b, dtype=np.float64)[None, :]) @ np.asarray(S_B, dtype=np.float64).T
    T = T * np.asarray(m, dtype=np.float64)[None, :]
    return (T @ np.asarray(S_A, dtype=np.float64).T) * np.asarray(a, dtype=np.float64)[None, :]
