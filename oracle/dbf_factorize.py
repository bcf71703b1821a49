"""DBF factorisation oracle: W -> (S_A, S_B, a, m, b), fp64.

Test infrastructure only (see the package docstring).  Source page: "Addition is
almost all you need: Compressing large language models with double binary
factorization" (gist.science), section "Optimalisatie en Training" under
"Methodologie: Double Binary Factorization (DBF)".  The page names the ingredients
and nothing more: finding the best factorisation is NP-hard, so a heuristic is
used; it alternates between the two factors (alternating minimisation) with the
ADMM method; the binary constraints are met by a projection based on SVID (the
magnitudes approximated by a rank-1 decomposition).  It gives no initialisation,
penalty, schedule or stopping rule, and it weights the error by input and output
importance, which needs calibration data (out of scope here: unweighted).

The plainest reading, written out here (every choice is recorded in the design
notes):

* Structured set.  A matrix Z is "OneBit-structured" when Z = diag(u) S diag(v)
  with S a +/-1 matrix and u, v >= 0, i.e. Z = S ⊙ (u v^T).  The DBF weight is the
  product of two such matrices, Z_A (N x r) and Z_B (r x K):
      Z_A Z_B = diag(u_A) S_A diag(v_A ⊙ u_B) S_B diag(v_B),
  so a = u_A, m = v_A ⊙ u_B, b = v_B.
* SVID projection of a real matrix M onto that set: S = Sign(M) and u v^T the
  rank-1 SVID of |M| (the same construction as OneBit's, applied to a factor).
* Initialisation: the rank-r truncated SVD W ≈ U_r Σ_r V_r^T split evenly,
  A = U_r Σ_r^(1/2), B = Σ_r^(1/2) V_r^T (zero columns/rows past min(N, K)),
  then Z_A, Z_B their projections and the scaled duals zero.  Alternatively (the
  start a GPU can run without an SVD) a sketch: A = W Ω for a given K x r matrix Ω
  (random numbers drawn by the caller), B = argmin ||W - A B||^2 + eps ||B||^2 with
  eps = SKETCH_RIDGE * trace(A^T A) / r.  The ridge (a tenth of A^T A's mean
  eigenvalue) keeps the start well posed in fp32 when W Ω is rank-deficient, and on
  the weights tried it ends at a slightly lower error than smaller ridges or the SVD
  start.
* One sweep: `admm_iters` ADMM steps on the left factor with Z_B fixed, then as
  many on the right factor with Z_A fixed.  An ADMM step on the left factor for
  min ||W - A Z_B||_F^2 subject to A in the set, with the split A = Z_A and the
  scaled dual U_A, is
      A   <- argmin ||W - A Z_B||^2 + rho ||A - Z_A + U_A||^2
           = (W Z_B^T + rho (Z_A - U_A)) (Z_B Z_B^T + rho I)^-1
      Z_A <- SVID projection of A + U_A
      U_A <- U_A + A - Z_A
  and symmetrically on the right factor.  rho = rho_rel * trace(Gram) / r with the
  current Gram matrix of the fixed factor, so rho_rel is scale-free.
* The kept iterate is the best (smallest ||W - Z_A Z_B||_F) seen over the sweeps.
* Last, with the signs fixed, the scales are refitted by exact least squares, one
  vector at a time given the other two (a, then b, then m, `refit_rounds` times):
  every such step can only lower the error.

Parity status: the factorisation loop as a whole is a heuristic whose steps the
page does not give, so its result is "parity unpinned": the tests pin its parts
(the projection's closed-form error, the ADMM least-squares step and the scale
refits against a library least-squares solve, exact recovery of a weight that is
itself a rank-1 DBF, the monotone refit, the +/-1 constraint) and a property of
the whole (a better error than OneBit at the same bits on a low-rank weight).
"""
from __future__ import annotations

import numpy as np

from .dbf import dbf_weight
from .onebit import sign_pm1, svid_rank1


def svid_project(M: np.ndarray) -> tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Projection of M onto {S ⊙ u v^T}: S = Sign(M), u v^T the rank-1 SVID of |M|.

    Returns (S, u, v) in float64 with u, v >= 0; the projection is diag(u) S diag(v).
    """
    M = np.asarray(M, dtype=np.float64)
    u, v, _ = svid_rank1(M)
    return sign_pm1(M), u, v


def structured(S: np.ndarray, u: np.ndarray, v: np.ndarray) -> np.ndarray:
    """diag(u) S diag(v) as a dense float64 matrix."""
    return np.asarray(u, dtype=np.float64)[:, None] * np.asarray(S, dtype=np.float64) * \
        np.asarray(v, dtype=np.float64)[None, :]


def dbf_init(W: np.ndarray, r: int) -> tuple[np.ndarray, np.ndarray]:
    """A (N x r), B (r x K) from the rank-r truncated SVD of W, singular values split evenly."""
    W = np.asarray(W, dtype=np.float64)
    N, K = W.shape
    U, s, Vt = np.linalg.svd(W, full_matrices=False)
    q = min(r, s.size)
    A = np.zeros((N, r))
    B = np.zeros((r, K))
    root = np.sqrt(s[:q])
    A[:, :q] = U[:, :q] * root[None, :]
    B[:q, :] = root[:, None] * Vt[:q, :]
    return A, B


SKETCH_RIDGE = 0.1


def dbf_init_sketch(W: np.ndarray, omega: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """A = W Ω (N x r); B = (A^T A + eps I)^-1 A^T W with eps = SKETCH_RIDGE trace(A^T A) / r."""
    W = np.asarray(W, dtype=np.float64)
    A = W @ np.asarray(omega, dtype=np.float64)
    r = A.shape[1]
    G = A.T @ A
    eps = SKETCH_RIDGE * float(np.trace(G)) / r
    B = np.linalg.solve(G + eps * np.eye(r), A.T @ W)
    return A, B


def admm_left_step(W, ZB, ZA, UA, rho):
    """argmin_A ||W - A ZB||_F^2 + rho ||A - ZA + UA||_F^2 = (W ZB^T + rho (ZA - UA)) (ZB ZB^T + rho I)^-1."""
    r = ZB.shape[0]
    G = ZB @ ZB.T + rho * np.eye(r)
    R = W @ ZB.T + rho * (ZA - UA)
    return np.linalg.solve(G, R.T).T  # G is symmetric


def admm_right_step(W, ZA, ZB, UB, rho):
    """argmin_B ||W - ZA B||_F^2 + rho ||B - ZB + UB||_F^2 = (ZA^T ZA + rho I)^-1 (ZA^T W + rho (ZB - UB))."""
    r = ZA.shape[1]
    G = ZA.T @ ZA + rho * np.eye(r)
    R = ZA.T @ W + rho * (ZB - UB)
    return np.linalg.solve(G, R)


def refit_a(W, S_A, S_B, m, b):
    """The least-squares a given the rest: a_n = <W_n, R_n> / ||R_n||^2, R = S_A diag(m) S_B diag(b)."""
    R = dbf_weight(S_A, S_B, np.ones(S_A.shape[0]), m, b)
    den = (R * R).sum(axis=1)
    num = (np.asarray(W, dtype=np.float64) * R).sum(axis=1)
    return np.where(den > 0, num / np.where(den > 0, den, 1.0), 0.0)


def refit_b(W, S_A, S_B, a, m):
    """The least-squares b given the rest: b_k = <W[:, k], C[:, k]> / ||C[:, k]||^2, C = diag(a) S_A diag(m) S_B."""
    C = dbf_weight(S_A, S_B, a, m, np.ones(S_B.shape[1]))
    den = (C * C).sum(axis=0)
    num = (np.asarray(W, dtype=np.float64) * C).sum(axis=0)
    return np.where(den > 0, num / np.where(den > 0, den, 1.0), 0.0)


def refit_m(W, S_A, S_B, a, b):
    """The least-squares m given the rest.

    W_hat = sum_j m_j p_j q_j^T with p_j = a ⊙ S_A[:, j] and q_j = S_B[j, :] ⊙ b, so the
    normal equations are G m = h with G = (P^T P) ∘ (Q Q^T) and h_j = p_j^T W q_j
    (P = diag(a) S_A, Q = S_B diag(b)); solved in the least-squares sense.
    """
    P = np.asarray(a, dtype=np.float64)[:, None] * np.asarray(S_A, dtype=np.float64)
    Q = np.asarray(S_B, dtype=np.float64) * np.asarray(b, dtype=np.float64)[None, :]
    G = (P.T @ P) * (Q @ Q.T)
    h = np.einsum("nj,nk,jk->j", P, np.asarray(W, dtype=np.float64), Q)
    return np.linalg.lstsq(G, h, rcond=None)[0]


def dbf_error(W, S_A, S_B, a, m, b) -> float:
    """||W - diag(a) S_A diag(m) S_B diag(b)||_F."""
    return float(np.linalg.norm(np.asarray(W, dtype=np.float64) - dbf_weight(S_A, S_B, a, m, b)))


def dbf_factorize(W: np.ndarray, r: int, sweeps: int = 20, admm_iters: int = 3, rho_rel: float = 1.0,
                  refit_rounds: int = 2, omega: np.ndarray | None = None) -> dict:
    """Factorise W (N x K) as diag(a) S_A diag(m) S_B diag(b) with middle dimension r.

    omega: None for the truncated-SVD start, or a K x r matrix for the sketch start.
    Returns a dict with S_A (N x r, +/-1), S_B (r x K, +/-1), a (N), m (r), b (K), all
    float64; "history": ||W - Z_A Z_B||_F after every sweep; "best": the smallest of
    the start's error and them (the iterate kept); "error": the error after the scale
    refit.
    """
    W = np.asarray(W, dtype=np.float64)
    if W.ndim != 2 or r < 1:
        raise ValueError("W must be a matrix and r >= 1")
    A, B = dbf_init(W, r) if omega is None else dbf_init_sketch(W, omega)
    pa = svid_project(A)
    pb = svid_project(B)
    ZA, ZB = structured(*pa), structured(*pb)
    UA, UB = np.zeros_like(ZA), np.zeros_like(ZB)
    best = (float(np.linalg.norm(W - ZA @ ZB)), pa, pb)
    history = []
    for _ in range(sweeps):
        for _ in range(admm_iters):
            rho = rho_rel * float(np.trace(ZB @ ZB.T)) / r
            A = admm_left_step(W, ZB, ZA, UA, rho)
            pa = svid_project(A + UA)
            ZA = structured(*pa)
            UA = UA + A - ZA
        for _ in range(admm_iters):
            rho = rho_rel * float(np.trace(ZA.T @ ZA)) / r
            B = admm_right_step(W, ZA, ZB, UB, rho)
            pb = svid_project(B + UB)
            ZB = structured(*pb)
            UB = UB + B - ZB
        err = float(np.linalg.norm(W - ZA @ ZB))
        history.append(err)
        if err < best[0]:
            best = (err, pa, pb)
    _, (S_A, uA, vA), (S_B, uB, vB) = best
    a, m, b = uA, vA * uB, vB
    for _ in range(refit_rounds):
        a = refit_a(W, S_A, S_B, m, b)
        b = refit_b(W, S_A, S_B, a, m)
        m = refit_m(W, S_A, S_B, a, b)
    return {"S_A": S_A, "S_B": S_B, "a": a, "m": m, "b": b, "history": history, "best": best[0],
            "error": dbf_error(W, S_A, S_B, a, m, b)}
