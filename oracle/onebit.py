"""OneBit oracle: sign extraction, bit packing, SVID and the linear layer, fp64.

Test infrastructure only (see the package docstring).  Source page: "1bit量化"
(blog.zerodtree.com), notes on "OneBit: Towards Extremely Low-bit Large
Language Models".

Readings where the page is silent (each recorded in the design notes):
* Sign(0): the page does not define it.  Sign(w) = -1 iff w < 0, so +0.0 and
  -0.0 both map to +1.  Proposition 2 needs only W = W_sign ⊙ |W|, which holds
  for any choice at zero.
* Bit layout: 32 signs per uint32, rows K-major, bit i of word w holds column
  32*w + i (least significant bit first); a set bit means -1.
* SVID split: a = sqrt(sigma1) * u1, b = sqrt(sigma1) * v1 with u1, v1 the
  leading singular pair of |W| taken nonnegative (|W| is a nonnegative matrix,
  so a nonnegative leading pair exists).
"""
from __future__ import annotations

import numpy as np


def sign_pm1(W: np.ndarray) -> np.ndarray:
    """W_sign = Sign(W) as float64 +/-1 ("rank-1 approximation": W = W_sign ⊙ |W|).

    -1 exactly where W < 0.  NaN has no sign and is rejected.
    """
    W = np.asarray(W)
    if np.isnan(W).any():
        raise ValueError("Sign(W) is undefined for NaN entries")
    return np.where(W < 0, -1.0, 1.0)


def pack_signs(W: np.ndarray) -> np.ndarray:
    """Packed W_sign: uint32 array (N, K/32); bit i of word w <-> column 32*w + i, 1 <=> -1.

    K must be a multiple of 32 (whole words per row).
    """
    W = np.asarray(W)
    if W.ndim != 2 or W.shape[1] % 32 != 0:
        raise ValueError("pack_signs needs a 2-D array with K a multiple of 32")
    N, K = W.shape
    negative = (sign_pm1(W) < 0).reshape(N, K // 32, 32)
    words = np.zeros((N, K // 32), dtype=np.uint64)
    for i in range(32):
        words |= negative[:, :, i].astype(np.uint64) << np.uint64(i)
    return words.astype(np.uint32)


def unpack_signs(P: np.ndarray, K: int) -> np.ndarray:
    """Inverse of ``pack_signs``: uint32 (N, K/32) -> float64 +/-1 (N, K)."""
    P = np.asarray(P, dtype=np.uint32)
    N, nw = P.shape
    if nw * 32 != K:
        raise ValueError("packed width does not match K")
    out = np.empty((N, K), dtype=np.float64)
    for i in range(32):
        bit = (P >> np.uint32(i)) & np.uint32(1)
        out[:, i::32] = np.where(bit == 1, -1.0, 1.0)
    return out


def rank1_svd(A: np.ndarray) -> tuple[np.ndarray, float, np.ndarray]:
    """Best rank-1 approximation u1 * sigma1 * v1^T of A by the SVD ("rank-1 approximation").

    Returns (u1, sigma1, v1) from LAPACK's thin SVD in float64.  For a matrix
    that is all zeros, returns zero vectors and sigma1 = 0.
    """
    A = np.asarray(A, dtype=np.float64)
    if not np.any(A):
        return np.zeros(A.shape[0]), 0.0, np.zeros(A.shape[1])
    U, s, Vt = np.linalg.svd(A, full_matrices=False)
    return U[:, 0].copy(), float(s[0]), Vt[0].copy()


def svid_rank1(W: np.ndarray) -> tuple[np.ndarray, np.ndarray, float]:
    """SVID of W: |W| ≈ a b^T by the rank-1 SVD of |W| ("rank-1 approximation").

    Returns (a, b, sigma1) in float64 with a = sqrt(sigma1) u1 >= 0 and
    b = sqrt(sigma1) v1 >= 0, so that W ≈ W_sign ⊙ (a b^T).
    """
    A = np.abs(np.asarray(W, dtype=np.float64))
    if np.isnan(A).any():
        raise ValueError("SVID is undefined for NaN entries")
    u, s, v = rank1_svd(A)
    # Singular vectors are defined up to a common sign; |W| >= 0 admits a
    # nonnegative leading pair, so orient it that way.
    if u.sum() + v.sum() < 0:
        u, v = -u, -v
    root = np.sqrt(s)
    return root * u, root * v, s


def onebit_weight(S: np.ndarray, a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """The approximated weight W_hat = W_sign ⊙ (a b^T), N x K, float64."""
    S = np.asarray(S, dtype=np.float64)
    return S * np.outer(np.asarray(a, dtype=np.float64), np.asarray(b, dtype=np.float64))


def onebit_linear(X: np.ndarray, S: np.ndarray, a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """Y = X · W_hat^T in the direct form (W_hat materialised), float64, M x N."""
    return np.asarray(X, dtype=np.float64) @ onebit_weight(S, a, b).T


def onebit_linear_packed(X: np.ndarray, P: np.ndarray, a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """``onebit_linear`` with W_sign given in the packed format."""
    X = np.asarray(X)
    return onebit_linear(X, unpack_signs(P, X.shape[1]), a, b)


def onebit_linear_prop1(X: np.ndarray, S: np.ndarray, a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """Proposition 1's factorised form [(X ⊙ b^T) W_sign^T] ⊙ a^T, float64.

    Used only to check Proposition 1 against the direct form.
    """
    X = np.asarray(X, dtype=np.float64)
    Xb = X * np.asarray(b, dtype=np.float64)[None, :]
    return (Xb @ np.asarray(S, dtype=np.float64).T) * np.asarray(a, dtype=np.float64)[None, :]


# Layer normalisation after the OneBit layer ("1bit量化", knowledge-distillation
# section: the student computes Y with Proposition 1 and then Z = LayerNorm(Y)).
# Reading (the page gives the name only): per token, i.e. per row of Y, over its
# N features; the biased variance; eps = 1e-5 inside the square root; no affine
# parameters (the page shows none).
LN_EPS = 1e-5


def layernorm(Y: np.ndarray, eps: float = LN_EPS) -> np.ndarray:
    """Z[m, :] = (Y[m, :] - mean) / sqrt(var + eps), mean and biased var over the row, fp64."""
    Y = np.asarray(Y, dtype=np.float64)
    mean = Y.mean(axis=1, keepdims=True)
    var = ((Y - mean) ** 2).mean(axis=1, keepdims=True)
    return (Y - mean) / np.sqrt(var + eps)


def onebit_linear_ln(X: np.ndarray, S: np.ndarray, a: np.ndarray, b: np.ndarray,
                     eps: float = LN_EPS) -> np.ndarray:
    """Z = LayerNorm(Y) with Y the OneBit layer in the direct form."""
    return layernorm(onebit_linear(X, S, a, b), eps)
