"""Pins of the DBF factorisation oracle (oracle/dbf_factorize.py), CPU only.

The factorisation loop is a heuristic the page names but does not spell out
("Addition is almost all you need: ...", gist.science, "Optimalisatie en
Training": alternating minimisation with ADMM and an SVID-based projection), so the
loop as a whole is parity unpinned.  Its parts are pinned here against closed
forms and library least-squares solves, and the whole against exact recovery and
a property: a better error than OneBit at equal bits on a low-rank weight.
"""
import numpy as np
import pytest

import oracle
from oracle import dbf_factorize as F


def _rng(seed):
    return np.random.default_rng(seed)


def _pm1(rng, shape):
    return np.where(rng.standard_normal(shape) < 0, -1.0, 1.0)


def test_projection_error_closed_form():
    # With S = Sign(M) and u v^T >= 0, ||M - S ⊙ u v^T|| = || |M| - u v^T ||, and for the
    # rank-1 SVD of |M| that is ||M||^2 - sigma_1(|M|)^2 (Eckart-Young).  sigma_1^2 comes
    # from the symmetric eigensolver of |M|^T |M|, not from an SVD.
    for seed in range(20):
        rng = _rng(seed)
        M = rng.standard_normal((7, 5)) * rng.uniform(0.1, 3.0)
        S, u, v = F.svid_project(M)
        Z = F.structured(S, u, v)
        lam = np.linalg.eigvalsh(np.abs(M).T @ np.abs(M))[-1]
        assert np.linalg.norm(M - Z) ** 2 == pytest.approx(np.linalg.norm(M) ** 2 - lam, rel=1e-9, abs=1e-12)
        assert np.all((u >= 0)) and np.all(v >= 0)
        assert np.array_equal(np.sign(Z[Z != 0]), S[Z != 0])


def test_projection_is_best_scaling_for_its_signs():
    # No nearby nonnegative (u', v') does better with the same signs.
    rng = _rng(40)
    M = rng.standard_normal((6, 8))
    S, u, v = F.svid_project(M)
    best = np.linalg.norm(M - F.structured(S, u, v))
    for _ in range(300):
        du = np.abs(u + 0.05 * rng.standard_normal(u.shape))
        dv = np.abs(v + 0.05 * rng.standard_normal(v.shape))
        assert np.linalg.norm(M - F.structured(S, du, dv)) >= best - 1e-12


@pytest.mark.parametrize("rho", [0.0, 0.37, 5.0])
def test_admm_steps_solve_regularised_least_squares(rho):
    # Row by row (left) and column by column (right), the regularised problem is an ordinary
    # least-squares problem on a stacked system; solve that with lstsq and compare.
    rng = _rng(50)
    N, r, K = 6, 4, 9
    W = rng.standard_normal((N, K))
    ZA, UA = rng.standard_normal((N, r)), 0.1 * rng.standard_normal((N, r))
    ZB, UB = rng.standard_normal((r, K)), 0.1 * rng.standard_normal((r, K))
    A = F.admm_left_step(W, ZB, ZA, UA, rho)
    for n in range(N):
        D = np.vstack([ZB.T, np.sqrt(rho) * np.eye(r)])
        t = np.concatenate([W[n], np.sqrt(rho) * (ZA - UA)[n]])
        assert np.allclose(A[n], np.linalg.lstsq(D, t, rcond=None)[0], atol=1e-10)
    B = F.admm_right_step(W, ZA, ZB, UB, rho)
    for k in range(K):
        D = np.vstack([ZA, np.sqrt(rho) * np.eye(r)])
        t = np.concatenate([W[:, k], np.sqrt(rho) * (ZB - UB)[:, k]])
        assert np.allclose(B[:, k], np.linalg.lstsq(D, t, rcond=None)[0], atol=1e-10)


def test_scale_refits_are_least_squares():
    rng = _rng(60)
    N, r, K = 5, 3, 7
    W = rng.standard_normal((N, K))
    SA, SB = _pm1(rng, (N, r)), _pm1(rng, (r, K))
    a, m, b = rng.uniform(0.5, 2, N), rng.uniform(0.5, 2, r), rng.uniform(0.5, 2, K)
    # a: one scalar per row; b: one per column; m: the vectorised design, one column per channel.
    R = SA @ np.diag(m) @ SB @ np.diag(b)
    a_ref = np.array([np.linalg.lstsq(R[n][:, None], W[n], rcond=None)[0][0] for n in range(N)])
    assert np.allclose(F.refit_a(W, SA, SB, m, b), a_ref, atol=1e-12)
    C = np.diag(a) @ SA @ np.diag(m) @ SB
    b_ref = np.array([np.linalg.lstsq(C[:, k][:, None], W[:, k], rcond=None)[0][0] for k in range(K)])
    assert np.allclose(F.refit_b(W, SA, SB, a, m), b_ref, atol=1e-12)
    D = np.stack([np.outer(a * SA[:, j], SB[j] * b).ravel() for j in range(r)], axis=1)
    m_ref = np.linalg.lstsq(D, W.ravel(), rcond=None)[0]
    assert np.allclose(F.refit_m(W, SA, SB, a, b), m_ref, atol=1e-10)


def test_scale_refits_never_raise_the_error():
    rng = _rng(70)
    N, r, K = 12, 5, 10
    W = rng.standard_normal((N, K))
    SA, SB = _pm1(rng, (N, r)), _pm1(rng, (r, K))
    a, m, b = rng.uniform(0.1, 2, N), rng.uniform(0.1, 2, r), rng.uniform(0.1, 2, K)
    e = F.dbf_error(W, SA, SB, a, m, b)
    for _ in range(4):
        a = F.refit_a(W, SA, SB, m, b)
        e1 = F.dbf_error(W, SA, SB, a, m, b)
        b = F.refit_b(W, SA, SB, a, m)
        e2 = F.dbf_error(W, SA, SB, a, m, b)
        m = F.refit_m(W, SA, SB, a, b)
        e3 = F.dbf_error(W, SA, SB, a, m, b)
        assert e1 <= e + 1e-12 and e2 <= e1 + 1e-12 and e3 <= e2 + 1e-12
        e = e3


@pytest.mark.parametrize("refit_rounds", [0, 2])
def test_exact_recovery_of_a_rank1_dbf_weight(refit_rounds):
    # W = diag(a) s_A m s_B^T diag(b) is a DBF weight with r = 1; its truncated SVD is
    # exact and so is the projection of each factor, so the factorisation returns W.
    for seed in range(5):
        rng = _rng(80 + seed)
        N, K = 9, 13
        W = oracle.dbf_weight(_pm1(rng, (N, 1)), _pm1(rng, (1, K)), rng.uniform(0.2, 2, N), rng.uniform(0.5, 2, 1),
                              rng.uniform(0.2, 2, K))
        res = F.dbf_factorize(W, 1, sweeps=3, refit_rounds=refit_rounds)
        W_hat = oracle.dbf_weight(res["S_A"], res["S_B"], res["a"], res["m"], res["b"])
        assert np.linalg.norm(W - W_hat) <= 1e-10 * np.linalg.norm(W)
        assert res["error"] <= 1e-10 * np.linalg.norm(W)


def test_sketch_start_recovers_a_rank1_dbf_weight():
    # For a rank-1 W, A = W Ω = w c^T and A^T A = |w|^2 c c^T has the single eigenvalue
    # lambda = trace(A^T A); the ridge fit then gives A B = W lambda / (lambda + eps) with
    # eps = SKETCH_RIDGE lambda / r, i.e. W / (1 + SKETCH_RIDGE / r) exactly.  The ADMM
    # sweeps remove that shrink: the factorisation returns W.
    for seed in range(5):
        rng = _rng(85 + seed)
        N, K, r = 9 + seed, 13, 4
        W = oracle.dbf_weight(_pm1(rng, (N, 1)), _pm1(rng, (1, K)), rng.uniform(0.2, 2, N), rng.uniform(0.5, 2, 1),
                              rng.uniform(0.2, 2, K))
        A, B = F.dbf_init_sketch(W, rng.standard_normal((K, r)))
        assert np.allclose(A @ B, W / (1 + F.SKETCH_RIDGE / r), rtol=1e-10, atol=1e-12)
        res = F.dbf_factorize(W, r, sweeps=3, refit_rounds=0, omega=rng.standard_normal((K, r)))
        assert res["error"] <= 1e-10 * np.linalg.norm(W)


def test_sketch_start_solves_the_ridge_least_squares():
    rng = _rng(86)
    W, omega = rng.standard_normal((8, 11)), rng.standard_normal((11, 3))
    A, B = F.dbf_init_sketch(W, omega)
    assert np.allclose(A, W @ omega)
    eps = F.SKETCH_RIDGE * np.trace(A.T @ A) / 3
    for k in range(11):
        D = np.vstack([A, np.sqrt(eps) * np.eye(3)])
        t = np.concatenate([W[:, k], np.zeros(3)])
        assert np.allclose(B[:, k], np.linalg.lstsq(D, t, rcond=None)[0], atol=1e-10)


def test_sketch_start_beats_onebit_on_a_low_rank_weight():
    # 128 x 128 at r = 64: the same bits as OneBit, and r a multiple of the packed word.
    rng = _rng(0)
    N = K = 128
    W = rng.standard_normal((N, 8)) @ rng.standard_normal((8, K)) * 0.01 + 0.001 * rng.standard_normal((N, K))
    r = 64
    a, b, _ = oracle.svid_rank1(W)
    e_onebit = np.linalg.norm(W - oracle.onebit_weight(oracle.sign_pm1(W), a, b))
    res = F.dbf_factorize(W, r, omega=np.random.default_rng(1).standard_normal((K, r)) / np.sqrt(K))
    assert res["error"] < 0.6 * e_onebit


def test_result_invariants():
    rng = _rng(90)
    N, K, r = 20, 28, 11
    W = rng.standard_normal((N, K))
    res = F.dbf_factorize(W, r, sweeps=8)
    assert res["S_A"].shape == (N, r) and res["S_B"].shape == (r, K)
    assert res["a"].shape == (N,) and res["m"].shape == (r,) and res["b"].shape == (K,)
    assert set(np.unique(res["S_A"])) <= {-1.0, 1.0} and set(np.unique(res["S_B"])) <= {-1.0, 1.0}
    assert len(res["history"]) == 8
    assert res["best"] <= min(res["history"]) + 1e-12
    assert res["error"] <= res["best"] + 1e-12  # the refit starts from the kept iterate
    assert res["error"] == pytest.approx(
        np.linalg.norm(W - oracle.dbf_weight(res["S_A"], res["S_B"], res["a"], res["m"], res["b"])), rel=1e-12)
    assert res["error"] < np.linalg.norm(W)


def test_middle_dimension_above_min_side():
    # r > min(N, K): the SVD fills min(N, K) channels and the rest start at zero.
    rng = _rng(100)
    W = rng.standard_normal((10, 14))
    res = F.dbf_factorize(W, 16, sweeps=5)
    assert res["S_A"].shape == (10, 16) and res["S_B"].shape == (16, 14)
    assert np.isfinite(res["error"]) and res["error"] < np.linalg.norm(W)


def test_beats_onebit_at_equal_bits_on_a_low_rank_weight():
    # At r = N K / (N + K) the two sign matrices hold as many bits as OneBit's one.  On a
    # weight of rank 8 plus small noise the factorisation must do clearly better.
    rng = _rng(0)
    N, K = 96, 128
    W = rng.standard_normal((N, 8)) @ rng.standard_normal((8, K)) * 0.01 + 0.001 * rng.standard_normal((N, K))
    r = N * K // (N + K)
    a, b, _ = oracle.svid_rank1(W)
    e_onebit = np.linalg.norm(W - oracle.onebit_weight(oracle.sign_pm1(W), a, b))
    res = F.dbf_factorize(W, r)
    assert res["error"] < 0.6 * e_onebit
