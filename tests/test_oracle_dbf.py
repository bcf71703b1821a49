"""Pins for the DBF oracle (CPU only).

Source page: "Addition is almost all you need: Compressing large language
models with double binary factorization" (gist.science), section
"Methodologie: Double Binary Factorization (DBF)".
"""
import numpy as np
import pytest

import oracle
from binary_weight_gemm_b200 import synth


def test_dbf_golden(golden):
    g = golden("dbf_2x2.json")
    args = [np.array(g[k], dtype=np.float64) for k in ("S_A", "S_B", "a", "m", "b")]
    X = np.array(g["X"])
    np.testing.assert_array_equal(oracle.dbf_weight(*args), g["W_hat"])
    np.testing.assert_array_equal(oracle.dbf_linear(X, *args), g["Y"])
    np.testing.assert_array_equal(oracle.dbf_linear_chain(X, *args), g["Y"])


def test_dbf_chain_equals_direct():
    for seed in range(20):
        rng = np.random.default_rng(seed)
        M, N, r, K = (int(v) for v in rng.integers(1, 10, 4))
        X = rng.standard_normal((M, K))
        S_A = np.where(rng.random((N, r)) < 0.5, -1.0, 1.0)
        S_B = np.where(rng.random((r, K)) < 0.5, -1.0, 1.0)
        a, m, b = rng.standard_normal(N), rng.standard_normal(r), rng.standard_normal(K)
        d = oracle.dbf_linear(X, S_A, S_B, a, m, b)
        c = oracle.dbf_linear_chain(X, S_A, S_B, a, m, b)
        assert np.linalg.norm(d - c) <= 1e-12 * max(1.0, np.linalg.norm(d))


def test_dbf_bruteforce_loops():
    # Y[i,n] = sum_k sum_j x_ik a_n SA_nj m_j SB_jk b_k by plain Python loops.
    rng = np.random.default_rng(8)
    M, N, r, K = 2, 3, 4, 5
    X = rng.standard_normal((M, K))
    S_A = np.where(rng.random((N, r)) < 0.5, -1.0, 1.0)
    S_B = np.where(rng.random((r, K)) < 0.5, -1.0, 1.0)
    a, m, b = rng.standard_normal(N), rng.standard_normal(r), rng.standard_normal(K)
    Y = oracle.dbf_linear(X, S_A, S_B, a, m, b)
    for i in range(M):
        for n in range(N):
            acc = 0.0
            for k in range(K):
                for j in range(r):
                    acc += X[i, k] * a[n] * S_A[n, j] * m[j] * S_B[j, k] * b[k]
            assert Y[i, n] == pytest.approx(acc, rel=1e-12, abs=1e-13)


def test_dbf_r1_reduces_to_onebit():
    # r = 1: W_hat = diag(a) s_A m0 s_B^T diag(b) = (s_A s_B^T) ⊙ (a (m0 b)^T),
    # the OneBit form with sign matrix s_A s_B^T and input scale m0*b.
    rng = np.random.default_rng(12)
    N, K = 7, 9
    sA = np.where(rng.random(N) < 0.5, -1.0, 1.0)
    sB = np.where(rng.random(K) < 0.5, -1.0, 1.0)
    a, b = rng.uniform(0.1, 1, N), rng.uniform(0.1, 1, K)
    m0 = 0.37
    X = rng.standard_normal((4, K))
    y_dbf = oracle.dbf_linear(X, sA[:, None], sB[None, :], a, np.array([m0]), b)
    y_ob = oracle.onebit_linear(X, np.outer(sA, sB), a, m0 * b)
    assert np.linalg.norm(y_dbf - y_ob) <= 1e-13 * np.linalg.norm(y_ob)


def test_dbf_one_hot_input():
    # X = e_k  =>  Y[:, n] = a_n * sum_j SA_nj m_j SB_jk * b_k.
    f = synth.dbf_factors(3, 6, 32, 64)
    X = np.eye(64)[[0, 33, 63]]
    Y = oracle.dbf_linear(X, f["S_A"], f["S_B"], f["a"], f["m"], f["b"])
    for row, k in enumerate([0, 33, 63]):
        col = f["S_A"].astype(np.float64) @ (f["m"].astype(np.float64) * f["S_B"][:, k])
        np.testing.assert_allclose(Y[row], f["a"] * col * f["b"][k], rtol=1e-13)
