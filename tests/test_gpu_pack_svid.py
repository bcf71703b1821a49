"""GPU parity: sign packing (bit-exact) and SVID (cosine >= 0.9999) against the oracle."""
import numpy as np
import pytest
import torch

import oracle
from binary_weight_gemm_b200 import synth
from conftest import SVID_COS_TOL
from helpers import cosine, oracle_svid

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ops():
    from binary_weight_gemm_b200 import build
    build.build()
    from binary_weight_gemm_b200 import ops as _ops
    torch.cuda.init()
    return _ops


def _pack_gpu(ops, W):
    P = ops.ob_pack_signs(torch.from_numpy(np.ascontiguousarray(W)).cuda())
    torch.cuda.synchronize()
    return P.cpu().numpy().view(np.uint32)


# ---------------------------------------------------------------- packing

def test_pack_golden_words(ops, golden):
    spec = golden("pack_words.json")
    K = spec["K"]
    rows, words = [], []
    for row in spec["rows"]:
        r = np.full(K, row["fill"], dtype=np.float32)
        for col, val in row["set"].items():
            r[int(col)] = np.float32(float(val))
        rows.append(r)
        words.append([int(w, 16) for w in row["words"]])
    assert _pack_gpu(ops, np.stack(rows)).tolist() == words
    assert ops.ob_last_device_error() == 0


@pytest.mark.parametrize("N,K", [(1, 32), (7, 96), (256, 256), (129, 4096), (4096, 4096), (11008, 4096),
                                 (4096, 11008)])
def test_pack_bit_exact(ops, N, K):
    W = synth.weights(N + K, N, K)
    assert np.array_equal(_pack_gpu(ops, W), oracle.pack_signs(W))


def test_pack_nan_sets_device_error(ops):
    W = np.ones((4, 64), dtype=np.float32)
    W[2, 17] = np.nan
    P = _pack_gpu(ops, W)
    assert ops.ob_last_device_error() == 4  # OB_ERR_NAN
    assert ops.ob_last_device_error() == 0  # cleared by the read
    assert P[2, 0] == 0  # NaN packs as +1


def test_pack_empty(ops):
    P = ops.ob_pack_signs(torch.empty((0, 64), dtype=torch.float32, device="cuda"))
    assert P.shape == (0, 2)


# ---------------------------------------------------------------- SVID

def _svid_gpu(ops, W, **kw):
    a, b, s, iters, st = ops.ob_svid_rank1(torch.from_numpy(np.ascontiguousarray(W)).cuda(), **kw)
    torch.cuda.synchronize()
    return a.cpu().numpy(), b.cpu().numpy(), float(s.cpu()[0]), iters, st


@pytest.mark.parametrize("seed,N,K", [(0, 256, 256), (7, 300, 512), (8, 1024, 96), (9, 64, 2048)])
def test_svid_matches_oracle(ops, seed, N, K):
    W = synth.weights(seed, N, K)
    a_ref, b_ref, s_ref = oracle.svid_rank1(W)
    a, b, s, iters, st = _svid_gpu(ops, W)
    assert st == 0 and iters >= 1
    assert (a >= 0).all() and (b >= 0).all()
    assert cosine(a, a_ref) >= SVID_COS_TOL
    assert cosine(b, b_ref) >= SVID_COS_TOL
    prod_err = np.linalg.norm(np.outer(a, b) - np.outer(a_ref, b_ref)) / np.linalg.norm(np.outer(a_ref, b_ref))
    assert prod_err <= 1e-4
    assert s == pytest.approx(s_ref, rel=1e-5)


def test_svid_full_size_decode_weight(ops):
    W, a_ref, b_ref, s_ref = oracle_svid(1, 4096, 4096)
    a, b, s, _, st = _svid_gpu(ops, W)
    assert st == 0
    assert cosine(a, a_ref) >= SVID_COS_TOL and cosine(b, b_ref) >= SVID_COS_TOL
    assert s == pytest.approx(s_ref, rel=1e-5)


@pytest.mark.parametrize("N,K", [(11008, 4096), (4096, 11008)])
def test_svid_full_size_fixed_point(ops, N, K):
    # At the 7B MLP shapes, check the defining property instead of a full SVD:
    # |W| b = sigma a and |W|^T a = sigma b with a, b >= 0.  For the positive
    # matrix |W|^T |W| the only nonnegative eigenvector is the leading one.
    W = synth.weights(2, N, K)
    a, b, s, _, st = _svid_gpu(ops, W)
    assert st == 0 and (a >= 0).all() and (b >= 0).all()
    A = np.abs(W.astype(np.float64))
    a64, b64 = a.astype(np.float64), b.astype(np.float64)
    assert np.linalg.norm(A @ b64 - s * a64) <= 1e-4 * np.linalg.norm(s * a64)
    assert np.linalg.norm(A.T @ a64 - s * b64) <= 1e-4 * np.linalg.norm(s * b64)
    # closed form: ||A - a b^T||^2 = ||A||^2 - sigma^2 (Proposition 2's derivation)
    err = np.sum(A * A) - 2 * (a64 @ A @ b64) + (a64 @ a64) * (b64 @ b64)
    assert err == pytest.approx(np.sum(A * A) - s * s, rel=1e-4)


def test_svid_exact_rank1_magnitudes(ops):
    rng = np.random.default_rng(5)
    p = rng.uniform(0.5, 2.0, 200).astype(np.float32)
    q = rng.uniform(0.5, 2.0, 160).astype(np.float32)
    W = (np.where(rng.random((200, 160)) < 0.5, -1, 1) * np.outer(p, q)).astype(np.float32)
    a, b, s, _, st = _svid_gpu(ops, W)
    assert st == 0
    np.testing.assert_allclose(np.outer(a, b), np.abs(W), rtol=2e-5)


def test_svid_all_zero_and_nan(ops):
    a, b, s, _, st = _svid_gpu(ops, np.zeros((64, 128), dtype=np.float32))
    assert st == 0 and s == 0.0 and not a.any() and not b.any()
    W = synth.weights(3, 64, 128)
    W[5, 5] = np.nan
    _, _, _, _, st = _svid_gpu(ops, W, check=False)
    assert st == 4  # OB_ERR_NAN


def test_svid_not_converged_reports(ops):
    W = synth.weights(4, 128, 128)
    a, b, s, iters, st = _svid_gpu(ops, W, max_iters=1, tol=1e-12, check=False)
    assert st == 5 and iters == 1  # OB_ERR_NOT_CONVERGED, last iterate written
    assert np.isfinite(a).all() and np.isfinite(b).all()
