"""GPU checks of dbf_factorize (the DBF factorisation) against the fp64 oracle.

The factorisation loop is a heuristic the page names without steps ("Addition is
almost all you need: ...", gist.science, "Optimalisatie en Training"), so parity is
to properties, not digits: exact recovery of a weight that is itself a rank-1 DBF,
the error the outputs actually give (recomputed by the oracle from the packed signs
and the scales), a better error than OneBit at equal bits on a low-rank weight and
closeness to the oracle's own run from the same start matrix, and the packed signs
feeding dbf_linear.  Every test also reads the device error word, so a build with
OB_DEBUG_BOUNDS=1 (device-side index checks) fails here on any refused access.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import dbf_factorize as F
from binary_weight_gemm_b200 import synth
from helpers import assert_gemm_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ops():
    from binary_weight_gemm_b200 import build
    build.build()
    from binary_weight_gemm_b200 import ops as _ops
    torch.cuda.init()
    return _ops


def _cuda(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()


def _factors(res, N, K, r):
    SA = oracle.unpack_signs(res["SA_packed"].cpu().numpy().view(np.uint32), r)
    SB = oracle.unpack_signs(res["SB_packed"].cpu().numpy().view(np.uint32), K)
    a, m, b = (res[k].double().cpu().numpy() for k in ("a", "m", "b"))
    assert SA.shape == (N, r) and SB.shape == (r, K)
    return SA, SB, a, m, b


def _pm1(rng, shape):
    return np.where(rng.standard_normal(shape) < 0, -1.0, 1.0)


def test_exact_recovery_of_a_rank1_dbf_weight(ops):
    rng = np.random.default_rng(85)
    N, K, r = 40, 64, 32
    W = oracle.dbf_weight(_pm1(rng, (N, 1)), _pm1(rng, (1, K)), rng.uniform(0.2, 2, N), rng.uniform(0.5, 2, 1),
                          rng.uniform(0.2, 2, K))
    omega = rng.standard_normal((K, r)) / np.sqrt(K)
    res = ops.dbf_factorize(_cuda(W), r, _cuda(omega), sweeps=3)
    assert ops.ob_last_device_error() == 0
    SA, SB, a, m, b = _factors(res, N, K, r)
    nW = np.linalg.norm(W)
    assert np.linalg.norm(W - oracle.dbf_weight(SA, SB, a, m, b)) <= 1e-3 * nW
    assert res["error"] <= 1e-3 * nW and res["best"] <= 1e-3 * nW


def test_low_rank_weight_against_the_oracle_and_onebit(ops):
    # 128 x 128 at r = 64: the same bits as OneBit.
    rng = np.random.default_rng(0)
    N = K = 128
    W = rng.standard_normal((N, 8)) @ rng.standard_normal((8, K)) * 0.01 + 0.001 * rng.standard_normal((N, K))
    r = 64
    omega = np.random.default_rng(1).standard_normal((K, r)) / np.sqrt(K)
    res = ops.dbf_factorize(_cuda(W), r, _cuda(omega))
    assert ops.ob_last_device_error() == 0
    SA, SB, a, m, b = _factors(res, N, K, r)
    nW = np.linalg.norm(W)
    e = np.linalg.norm(W - oracle.dbf_weight(SA, SB, a, m, b))
    assert e == pytest.approx(res["error"], rel=1e-3)          # the reported error is the outputs' error
    assert res["error"] <= res["best"] * (1 + 1e-4)             # the refit does not raise it
    assert res["best"] <= min(res["history"]) * (1 + 1e-6)
    ua, ub, _ = oracle.svid_rank1(W)
    e_onebit = np.linalg.norm(W - oracle.onebit_weight(oracle.sign_pm1(W), ua, ub))
    assert e < 0.6 * e_onebit
    ref = F.dbf_factorize(W, r, omega=omega)
    assert e <= 1.15 * ref["error"]                             # the oracle's run from the same start
    assert e / nW < 0.3


def test_factors_feed_dbf_linear(ops):
    rng = np.random.default_rng(7)
    N, K, r = 96, 160, 64
    W = synth.weights(7, N, K).astype(np.float64)
    omega = rng.standard_normal((K, r)) / np.sqrt(K)
    res = ops.dbf_factorize(_cuda(W), r, _cuda(omega), sweeps=4)
    assert ops.ob_last_device_error() == 0
    SA, SB, a, m, b = _factors(res, N, K, r)
    assert np.all(np.isfinite(a)) and np.all(np.isfinite(m)) and np.all(np.isfinite(b))
    xb, x = synth.activations(7, 5, K)
    X = torch.from_numpy(np.ascontiguousarray(xb.view(np.int16))).cuda().view(torch.bfloat16)
    Y = ops.dbf_linear(X, res["SB_packed"], res["m"], res["SA_packed"], res["a"], res["b"])
    torch.cuda.synchronize()
    assert_gemm_close(Y, oracle.dbf_linear(x, SA, SB, a, m, b), what="dbf_linear on factorised weights")
