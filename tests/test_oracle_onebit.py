"""Pins for the OneBit oracle (CPU only).

Each test ties the oracle to something other than itself: hand-computed worked
examples (tests/golden), closed forms, special cases with a known answer,
brute force on tiny inputs, and the inequalities the page proves (Lemma 1,
Proposition 2).  Source page: "1bit量化" (blog.zerodtree.com).
"""
import itertools
import math

import numpy as np
import pytest

import oracle
from binary_weight_gemm_b200 import synth

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


# ---------------------------------------------------------------- sign + packing

def _golden_pack_matrix(spec):
    K = spec["K"]
    rows = []
    for row in spec["rows"]:
        r = np.full(K, row["fill"], dtype=np.float32)
        for col, val in row["set"].items():
            r[int(col)] = np.float32(float(val))
        rows.append(r)
    return np.stack(rows), [[int(w, 16) for w in row["words"]] for row in spec["rows"]]


def test_pack_golden_words(golden):
    W, words = _golden_pack_matrix(golden("pack_words.json"))
    P = oracle.pack_signs(W)
    assert P.dtype == np.uint32
    assert P.tolist() == words


def test_sign_of_zero_and_specials():
    W = np.array([-0.0, 0.0, 1e-45, -1e-45, np.inf, -np.inf], dtype=np.float32)
    assert oracle.sign_pm1(W).tolist() == [1.0, 1.0, 1.0, -1.0, 1.0, -1.0]


def test_sign_rejects_nan():
    with pytest.raises(ValueError):
        oracle.pack_signs(np.array([[np.nan] + [1.0] * 31], dtype=np.float32))


def test_pack_single_negative_position():
    # A lone negative at (n, k) must set exactly bit k%32 of word (n, k//32):
    # catches a reversed bit order, swapped row/word indexing and polarity.
    rng = np.random.default_rng(11)
    N, K = 7, 96
    for _ in range(40):
        n, k = int(rng.integers(N)), int(rng.integers(K))
        W = np.ones((N, K), dtype=np.float32)
        W[n, k] = -1.0
        P = oracle.pack_signs(W)
        expect = np.zeros((N, K // 32), dtype=np.uint32)
        expect[n, k // 32] = np.uint32(1) << np.uint32(k % 32)
        assert np.array_equal(P, expect)


def test_pack_unpack_roundtrip():
    W = synth.weights(0, 37, 160)
    P = oracle.pack_signs(W)
    assert P.shape == (37, 5)
    assert np.array_equal(oracle.unpack_signs(P, 160), np.where(W < 0, -1.0, 1.0))


def test_pack_matches_bit_arithmetic_brute_force():
    # Pure-Python construction of each word from its 32 signs.
    W = synth.weights(3, 4, 64)
    P = oracle.pack_signs(W)
    for n in range(4):
        for w in range(2):
            word = 0
            for i in range(32):
                if float(W[n, 32 * w + i]) < 0:
                    word += 2 ** i
            assert int(P[n, w]) == word


def test_pack_rejects_ragged_k():
    with pytest.raises(ValueError):
        oracle.pack_signs(np.ones((2, 33), dtype=np.float32))


# ---------------------------------------------------------------- SVID

def test_svid_golden_rank1(golden):
    g = golden("svid_2x2.json")
    a, b, s = oracle.svid_rank1(np.array(g["W"]))
    assert s == pytest.approx(g["sigma1"], rel=1e-14)
    np.testing.assert_allclose(a, g["a"], rtol=1e-13)
    np.testing.assert_allclose(b, g["b"], rtol=1e-13)
    What = oracle.onebit_weight(oracle.sign_pm1(np.array(g["W"])), a, b)
    np.testing.assert_allclose(What, g["W_hat"], rtol=1e-13)


def test_svid_golden_nonsquare_closed_form(golden):
    g = golden("svid_3x2_diag.json")
    W = np.array(g["W"])
    a, b, s = oracle.svid_rank1(W)
    assert a.shape == (3,) and b.shape == (2,)
    assert s == pytest.approx(g["sigma1"], rel=1e-14)
    np.testing.assert_allclose(a, g["a"], atol=1e-14)
    np.testing.assert_allclose(b, g["b"], atol=1e-14)
    err = np.sum((np.abs(W) - np.outer(a, b)) ** 2)
    assert err == pytest.approx(g["err_fro2"], rel=1e-13)
    np.testing.assert_allclose(oracle.onebit_weight(oracle.sign_pm1(W), a, b), g["W_hat"], atol=1e-14)


def test_svid_exact_when_magnitudes_rank1():
    # W = S0 ⊙ (p q^T) with p, q > 0: |W| = p q^T is rank 1, so SVID is exact,
    # W_hat == W, and the OneBit layer equals the dense layer X W^T.
    rng = np.random.default_rng(5)
    N, K = 9, 13
    p = rng.uniform(0.5, 2.0, N)
    q = rng.uniform(0.5, 2.0, K)
    S0 = np.where(rng.random((N, K)) < 0.5, -1.0, 1.0)
    W = S0 * np.outer(p, q)
    a, b, s = oracle.svid_rank1(W)
    np.testing.assert_allclose(np.outer(a, b), np.outer(p, q), rtol=1e-12)
    assert s == pytest.approx(np.linalg.norm(p) * np.linalg.norm(q), rel=1e-13)
    What = oracle.onebit_weight(oracle.sign_pm1(W), a, b)
    np.testing.assert_allclose(What, W, rtol=1e-12)
    X = rng.standard_normal((3, K))
    np.testing.assert_allclose(oracle.onebit_linear(X, oracle.sign_pm1(W), a, b), X @ W.T,
                               rtol=1e-11, atol=1e-12)


def test_svid_nonnegative_vectors():
    for seed in range(10):
        W = synth.weights(seed, 17, 23)
        a, b, _ = oracle.svid_rank1(W)
        assert a.shape == (17,) and b.shape == (23,)
        assert (a >= 0).all() and (b >= 0).all()


def test_svid_closed_form_error_against_eigenvalues():
    # Proposition 2's closed form ||A - a b^T||_F^2 = ||A||_F^2 - sigma1^2, with
    # sigma1^2 taken independently as the top eigenvalue of A^T A (eigvalsh).
    for seed in range(8):
        W = synth.weights(seed, 12 + seed, 20)
        A = np.abs(W.astype(np.float64))
        a, b, s = oracle.svid_rank1(W)
        lam = np.linalg.eigvalsh(A.T @ A).max()
        assert s * s == pytest.approx(lam, rel=1e-10)
        err = np.sum((A - np.outer(a, b)) ** 2)
        assert err == pytest.approx(np.sum(A * A) - lam, rel=1e-9)


def test_svid_eckart_young_bruteforce_3x3():
    # No rank-1 (a, b) beats the oracle's error on 3x3 inputs.  For a given
    # direction a, the best b is the least-squares fit A^T a / |a|^2; search a
    # over a dense grid of the sphere, then refine random restarts.
    from scipy.optimize import minimize

    def err(A, avec):
        nrm = float(avec @ avec)
        if nrm == 0.0:
            return float(np.sum(A * A))
        bvec = A.T @ avec / nrm
        return float(np.sum((A - np.outer(avec, bvec)) ** 2))

    th = np.linspace(0, math.pi, 61)
    ph = np.linspace(0, 2 * math.pi, 121)
    dirs = np.array([[math.sin(t) * math.cos(p), math.sin(t) * math.sin(p), math.cos(t)]
                     for t, p in itertools.product(th, ph)])
    rng = np.random.default_rng(2024)
    for trial in range(12):
        W = rng.standard_normal((3, 3))
        A = np.abs(W)
        a, b, _ = oracle.svid_rank1(W)
        best_oracle = float(np.sum((A - np.outer(a, b)) ** 2))
        grid_errs = [err(A, d) for d in dirs]
        grid_best = min(grid_errs)
        assert grid_best >= best_oracle - 1e-9
        # Refining the best grid direction reaches the oracle's error.
        start = dirs[int(np.argmin(grid_errs))]
        res = minimize(lambda v: err(A, v), start, method="Nelder-Mead",
                       options={"xatol": 1e-12, "fatol": 1e-15, "maxiter": 4000})
        assert res.fun >= best_oracle - 1e-9
        assert res.fun <= best_oracle + 1e-8
        for _ in range(5):
            res = minimize(lambda v: err(A, v), rng.standard_normal(3), method="Nelder-Mead",
                           options={"xatol": 1e-12, "fatol": 1e-14, "maxiter": 4000})
            assert res.fun >= best_oracle - 1e-9


def test_lemma1_sigma1_abs_dominates():
    # Lemma 1: sigma1(|W|) >= sigma1(W), with equality for nonnegative W.
    for seed in range(100):
        rng = np.random.default_rng(seed)
        W = rng.standard_normal((int(rng.integers(2, 9)), int(rng.integers(2, 9))))
        _, s_abs, _ = oracle.rank1_svd(np.abs(W))
        _, s, _ = oracle.rank1_svd(W)
        assert s_abs >= s - 1e-12
        # sigma1 is the operator 2-norm (independent routine).
        assert s == pytest.approx(np.linalg.norm(W, 2), rel=1e-12)
    P = np.abs(np.random.default_rng(1).standard_normal((5, 4)))
    assert oracle.rank1_svd(P)[1] == pytest.approx(oracle.rank1_svd(np.abs(P))[1], rel=1e-14)


def test_proposition2_svid_beats_plain_rank1():
    # Proposition 2: ||W - W_sign ⊙ a~ b~^T||_F^2 <= ||W - a b^T||_F^2, where
    # a b^T is the rank-1 SVD of W itself; and the SVID error equals the rank-1
    # error of |W| (sign mask does not change squared magnitudes).
    for seed in range(50):
        rng = np.random.default_rng(100 + seed)
        W = rng.standard_normal((int(rng.integers(2, 12)), int(rng.integers(2, 12))))
        a, b, _ = oracle.svid_rank1(W)
        svid_err = np.sum((W - oracle.onebit_weight(oracle.sign_pm1(W), a, b)) ** 2)
        u, s, v = oracle.rank1_svd(W)
        plain_err = np.sum((W - s * np.outer(u, v)) ** 2)
        assert svid_err <= plain_err + 1e-12
        assert svid_err == pytest.approx(np.sum((np.abs(W) - np.outer(a, b)) ** 2), rel=1e-12)


def test_svid_all_zero():
    a, b, s = oracle.svid_rank1(np.zeros((4, 3)))
    assert s == 0.0 and not a.any() and not b.any()


# ---------------------------------------------------------------- linear layer

def test_linear_golden(golden):
    g = golden("onebit_linear_2x2.json")
    X, S, a, b = (np.array(g[k]) for k in ("X", "S", "a", "b"))
    np.testing.assert_array_equal(oracle.onebit_weight(S, a, b), g["W_hat"])
    np.testing.assert_array_equal(oracle.onebit_linear(X, S, a, b), g["Y"])
    np.testing.assert_array_equal(oracle.onebit_linear_prop1(X, S, a, b), g["Y"])


def test_linear_bruteforce_loops():
    # Y[i,j] = sum_k x_ik s_jk a_j b_k, by plain Python loops (proof of Prop. 1).
    rng = np.random.default_rng(7)
    M, N, K = 3, 5, 4
    X = rng.standard_normal((M, K))
    S = np.where(rng.random((N, K)) < 0.5, -1.0, 1.0)
    a, b = rng.standard_normal(N), rng.standard_normal(K)
    Y = oracle.onebit_linear(X, S, a, b)
    for i in range(M):
        for j in range(N):
            acc = 0.0
            for k in range(K):
                acc += X[i, k] * S[j, k] * a[j] * b[k]
            assert Y[i, j] == pytest.approx(acc, rel=1e-13, abs=1e-14)


def test_proposition1_direct_equals_factored():
    for seed in range(20):
        rng = np.random.default_rng(seed)
        M, N, K = (int(v) for v in rng.integers(1, 9, 3))
        X = rng.standard_normal((M, K))
        S = np.where(rng.random((N, K)) < 0.5, -1.0, 1.0)
        a, b = rng.standard_normal(N), rng.standard_normal(K)
        d = oracle.onebit_linear(X, S, a, b)
        f = oracle.onebit_linear_prop1(X, S, a, b)
        assert np.linalg.norm(d - f) <= 1e-12 * max(1.0, np.linalg.norm(d))


def test_linear_one_hot_rows_pick_columns():
    # X = e_k  =>  Y[:, n] = a_n * s_nk * b_k : pins the K/N orientation.
    rng = np.random.default_rng(3)
    N, K = 6, 64
    W = rng.standard_normal((N, K)).astype(np.float32)
    P = oracle.pack_signs(W)
    a, b = rng.uniform(0.1, 1, N), rng.uniform(0.1, 1, K)
    X = np.eye(K)[[0, 7, 31, 32, 63]]
    Y = oracle.onebit_linear_packed(X, P, a, b)
    for row, k in enumerate([0, 7, 31, 32, 63]):
        expect = a * np.where(W[:, k] < 0, -1.0, 1.0) * b[k]
        np.testing.assert_allclose(Y[row], expect, rtol=1e-15)


def test_linear_all_plus_signs():
    rng = np.random.default_rng(4)
    X = rng.standard_normal((3, 32))
    a, b = rng.standard_normal(5), rng.standard_normal(32)
    Y = oracle.onebit_linear(X, np.ones((5, 32)), a, b)
    np.testing.assert_allclose(Y, np.outer(X @ b, a), rtol=1e-12)


def test_linear_packed_equals_unpacked():
    W = synth.weights(9, 10, 96)
    _, x = synth.activations(9, 4, 96)
    a, b, _ = oracle.svid_rank1(W)
    y1 = oracle.onebit_linear_packed(x, oracle.pack_signs(W), a, b)
    y2 = oracle.onebit_linear(x, oracle.sign_pm1(W), a, b)
    np.testing.assert_array_equal(y1, y2)


# ---------------------------------------------------------------- LayerNorm after the layer

def test_layernorm_golden(golden):
    g = golden("layernorm_4.json")
    np.testing.assert_allclose(oracle.layernorm(np.array(g["Y"]), eps=g["eps"]), np.array(g["Z"]),
                               rtol=0, atol=1e-15)


@pytest.mark.parametrize("M,N", [(1, 2), (3, 7), (16, 4096), (5, 11008)])
def test_layernorm_matches_torch(M, N):
    import torch
    Y = np.random.default_rng(M * N).standard_normal((M, N)) * 3.0 + 0.7
    ref = torch.nn.functional.layer_norm(torch.from_numpy(Y), (N,), eps=1e-5).numpy()
    np.testing.assert_allclose(oracle.layernorm(Y, eps=1e-5), ref, rtol=1e-12, atol=1e-12)


def test_layernorm_invariants():
    rng = np.random.default_rng(3)
    Y = rng.standard_normal((6, 300)) * rng.uniform(0.1, 10, (6, 1)) + rng.uniform(-5, 5, (6, 1))
    var = Y.var(axis=1)
    Z = oracle.layernorm(Y, eps=1e-5)
    np.testing.assert_allclose(Z.mean(axis=1), 0.0, atol=1e-13)
    np.testing.assert_allclose(Z.var(axis=1), var / (var + 1e-5), rtol=1e-12)
    # eps = 0: invariant under a positive per-row scale and a per-row shift.
    alpha, beta = rng.uniform(0.5, 4, (6, 1)), rng.uniform(-3, 3, (6, 1))
    np.testing.assert_allclose(oracle.layernorm(alpha * Y + beta, eps=0.0), oracle.layernorm(Y, eps=0.0),
                               rtol=1e-10, atol=1e-12)


def test_layernorm_degenerate_rows():
    # One feature, or a constant row: y - mean = 0 everywhere, so Z = 0.
    assert not oracle.layernorm(np.array([[3.0], [-2.0]])).any()
    assert not oracle.layernorm(np.full((2, 5), 7.25)).any()


def test_onebit_linear_ln_golden(golden):
    # The 2 x 2 worked example gives Y = [-18, -57]: LayerNorm over two features is +/-1
    # up to eps (mean -37.5, variance 19.5^2).
    g = golden("onebit_linear_2x2.json")
    Z = oracle.onebit_linear_ln(np.array(g["X"]), np.array(g["S"]), np.array(g["a"]), np.array(g["b"]))
    np.testing.assert_allclose(Z, [[1.0, -1.0]], rtol=1e-7)
